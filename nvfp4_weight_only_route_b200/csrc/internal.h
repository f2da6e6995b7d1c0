// internal.h -- layer handle, workspace carving and kernel launchers of libtfmoe.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/tfmoe.h"

namespace tfmoe {

// Tile geometry of the repacked NVFP4 weights: 128 rows x 64 reduction
// elements per tile; a tile holds 4096 code bytes laid out as
// [half of the 64 columns][128 rows][16 bytes], then its 512 scale bytes as
// [128 rows][4 blocks of 16].
constexpr int kTileRows = 128;
constexpr int kTileK = 64;
constexpr int kTileCodeBytes = kTileRows * kTileK / 2;   // 4096
constexpr int kTileScaleBytes = kTileRows * kTileK / 16; // 512

// Default crossover: experts routed to at most this many tokens use the GEMV regime.
constexpr int kDefaultGemvMaxTokens = 1 << 30;

struct Workspace {
    float *logits = nullptr;        // [maxT][E]
    int32_t *ids = nullptr;         // [maxT][k]
    float *topk_w = nullptr;        // [maxT][k]
    int32_t *counts = nullptr;      // [E]
    int32_t *offsets = nullptr;     // [E+1]
    int32_t *perm = nullptr;        // [maxP]
    int32_t *inv = nullptr;         // [maxP]
    int32_t *regime = nullptr;      // [E]
    int32_t *gemv_list = nullptr;   // [E]   experts in the GEMV regime, ascending
    int32_t *mma_list = nullptr;    // [E]   experts in the MMA regime, ascending
    int32_t *list_sizes = nullptr;  // [4]   n_gemv, n_mma, (reserved)
    int32_t *err_word = nullptr;    // [1]
    uint16_t *act = nullptr;        // [maxP][I] bf16
    float *y = nullptr;             // [maxP][H]
    uint16_t *x_stage = nullptr;    // [maxT][H] bf16, for forward_host
    uint16_t *out_stage = nullptr;  // [maxT][H] bf16, for forward_host
};

struct Weights {
    uint16_t *router_w = nullptr;   // [E][H] bf16
    float *router_bias = nullptr;   // [E]
    uint8_t *gu_codes = nullptr;    // [E][2I/128][H/64] tiles (gate row j -> 2j, up row j -> 2j+1)
    uint8_t *gu_scales = nullptr;
    uint8_t *d_codes = nullptr;     // [E][H/128][I/64] tiles
    uint8_t *d_scales = nullptr;
    float *gate_global = nullptr;   // [E]
    float *up_global = nullptr;     // [E]
    float *down_global = nullptr;   // [E]
};

struct Layer {
    tfmoe_layer_desc desc{};
    int device = 0;
    int num_sms = 0;
    int gemv_max_tokens = kDefaultGemvMaxTokens;
    bool loaded = false;
    void *ws_block = nullptr;
    size_t ws_bytes = 0;
    void *w_block = nullptr;
    size_t w_bytes = 0;
    Workspace ws;
    Weights w;
    int32_t last_launches = 0;
    int gemv_grid_gu = 0, gemv_grid_down = 0;
    // per-stage profiling (tfmoe_profile_enable)
    bool profiling = false;
    cudaEvent_t prof_ev[TFMOE_STAGE_COUNT][2] = {};
    bool prof_used[TFMOE_STAGE_COUNT] = {};
    float prof_ms[TFMOE_STAGE_COUNT] = {};
    int32_t prof_calls[TFMOE_STAGE_COUNT] = {};
};

// Records the start/end events of one stage when profiling is on.
struct StageTimer {
    Layer &L;
    int stage;
    cudaStream_t s;
    StageTimer(Layer &l, int st, cudaStream_t str) : L(l), stage(st), s(str) {
        if (L.profiling) cudaEventRecord(L.prof_ev[stage][0], s);
    }
    ~StageTimer() {
        if (L.profiling) { cudaEventRecord(L.prof_ev[stage][1], s); L.prof_used[stage] = true; }
    }
};

// Launchers. Each returns cudaGetLastError() after its launches and adds
// the number of kernels it enqueued to *launches.
cudaError_t launch_router(Layer &L, const uint16_t *x, int T, cudaStream_t s, int *launches);
cudaError_t launch_permute(Layer &L, int T, cudaStream_t s, int *launches);
cudaError_t launch_gemv(Layer &L, const uint16_t *x, int T, cudaStream_t s, int *launches);
cudaError_t launch_combine(Layer &L, int T, uint16_t *out, cudaStream_t s, int *launches);
cudaError_t launch_repack(const Layer &L, const tfmoe_weights &src, cudaStream_t s);
cudaError_t gemv_setup(Layer &L);

// Sets the thread-local message returned by tfmoe_last_error() and returns st.
tfmoe_status record_error(tfmoe_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
tfmoe_status record_ok();

}  // namespace tfmoe
