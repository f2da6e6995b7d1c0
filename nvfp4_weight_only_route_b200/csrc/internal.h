// internal.h -- layer handle, workspace carving and kernel launchers of libtfmoe.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/tfmoe.h"

namespace tfmoe {

// Tile geometry of the repacked NVFP4 weights: 128 rows x 64 reduction
// elements per tile. Codes: 4096 bytes per tile laid out as
// [half of the 64 columns][128 rows][16 bytes], tiles ordered
// [expert][row tile][column tile]. Scales: one 512-byte slab per tile, ordered
// like the tiles, holding [128 rows][4 bytes] (the E4M3 scales of the row's
// four 16-column blocks of the tile).
constexpr int kTileRows = 128;
constexpr int kTileK = 64;
constexpr int kTileCodeBytes = kTileRows * kTileK / 2;   // 4096
constexpr int kTileScaleBytes = kTileRows * kTileK / 16; // 512

// Byte offset of the scale slab of row tile `row_tile_index` (= expert * RT + rt), column tile `kt`.
__host__ __device__ __forceinline__ size_t scale_offset(size_t row_tile_index, int KT, int kt) {
    return (row_tile_index * (size_t)KT + (size_t)kt) * kTileScaleBytes;
}

// Largest reduction length (hidden or intermediate) the library supports: a GEMV task
// stages the scales of all its column tiles with one tensor copy, whose box
// extent is limited to 256 tiles.
constexpr int kMaxReduction = 256 * kTileK;

// Built-in crossover between the regimes (measured on B200): for batches of at most
// kSmallBatchTokens tokens every expert stays in the GEMV regime (the tensor-core
// regime's extra launches cost more than they save); above that, experts routed to at
// most kDefaultGemvMaxTokens tokens use the GEMV regime.
constexpr int kSmallBatchTokens = 16;
constexpr int kDefaultGemvMaxTokens = 2;

// Router for T > 16 (tensor-core approximation + exact candidates): the largest top_k,
// and the candidate experts one token's list holds (beyond it the token takes every expert
// exactly).
constexpr int kRouterMaxK = 32;
constexpr int kRouterMaxCand = 64;

// Batches with more than this many (token, expert) pairs build the plan with a
// multi-CTA scan instead of one CTA.
constexpr int kLargePlanPairs = 4096;
// Tokens per segment of the multi-CTA plan: the router's last kernel writes each segment's
// expert histogram (one CTA of warps per segment, one warp per token).
constexpr int kPlanSegTokens = 8;

// Tokens per tensor-core tile (the MMA N dimension): up to kMmaTileTokens with one CTA
// per SM, or up to kMmaSmallTileTokens with two CTAs per SM when a batch averages at most
// kMmaSmallMaxAvgTokens tokens per expert.
constexpr int kMmaTileTokens = 256;
constexpr int kMmaSmallTileTokens = 64;
constexpr int kMmaSmallMaxAvgTokens = 64;
__host__ __device__ constexpr size_t max_mma_entries(size_t P, size_t E) { return P / kMmaSmallTileTokens + E + 1; }

struct Workspace {
    float *logits = nullptr;        // [maxT][E]
    float *xnorm = nullptr;         // [maxT] upper bound of ||x_t||_2 (router, T > 16)
    int32_t *xexp = nullptr;        // [maxT] smallest | largest << 16 exponent field of x_t's nonzero elements
    int32_t *cand_cnt = nullptr;    // [maxT] router candidates per token, -1 = every expert
    uint16_t *cand = nullptr;       // [maxT][kRouterMaxCand] router candidate experts
    int32_t *ids = nullptr;         // [maxT][k]
    float *topk_w = nullptr;        // [maxT][k]
    int32_t *counts = nullptr;      // [E]
    int32_t *offsets = nullptr;     // [E+1]
    int32_t *perm = nullptr;        // [maxP]
    int32_t *inv = nullptr;         // [maxP]
    int32_t *regime = nullptr;      // [E]
    int32_t *gemv_list = nullptr;   // [E]   experts in the GEMV regime, ascending
    int32_t *mma_list = nullptr;    // [E]   experts in the MMA regime, ascending
    int32_t *list_sizes = nullptr;  // [4]   n_gemv, n_mma, n_mma_entries, (reserved)
    int32_t *err_word = nullptr;    // [1]
    int32_t *route_counter = nullptr; // [1] arrivals of the fused routing kernel (left at 0)
    int32_t *seg_cnt = nullptr;     // [ceil(maxT/8)][E] per-segment expert counts (large-batch plan)
    int32_t *seg_base = nullptr;    // [ceil(maxT/8)][E] per-segment first ranks
    int32_t *plan_tot = nullptr;    // [E]
    int32_t *plan_counter = nullptr; // [1] arrivals of the plan scan (left at 0)
    int32_t *mma_entries = nullptr; // [max_mma_entries][4] token tiles of the MMA regime
    uint16_t *x_perm = nullptr;     // [maxP][H] f16 activation rows (times 2^sh) in permuted order (MMA regime)
    float *row_inv = nullptr;       // [maxP] 2^-sh of each x_perm row
    uint16_t *act = nullptr;        // [maxP][I] bf16
    uint16_t *xq = nullptr;         // [maxT][H] f16: x times a power of two per 16 elements (GEMV regime)
    float *xq_inv = nullptr;        // [maxT][H/16] the inverse powers of two
    uint16_t *aq = nullptr;         // [maxP][I] f16: act times a power of two per 16 elements (GEMV regime)
    float *aq_inv = nullptr;        // [maxP][I/16]
    float *y = nullptr;             // [maxP][H]
    uint16_t *x_stage = nullptr;    // [maxT][H] bf16, for forward_host
    uint16_t *out_stage = nullptr;  // [maxT][H] bf16, for forward_host
};

struct Weights {
    uint16_t *router_w = nullptr;   // [E][H] bf16
    float4 *router_cst = nullptr;   // [E] router bound constants {bias, C_e, B_e, 0} (router_tc.cu)
    int32_t *router_wexp = nullptr; // [2] smallest and largest exponent field of the router weights' nonzero elements
    float *router_bias = nullptr;   // [E]
    // Expert-slot arrays hold the E routed experts, then the shared expert's m = Is/I slots.
    uint8_t *gu_codes = nullptr;    // [E+m][2I/128][H/64] tiles (gate row j -> 2j, up row j -> 2j+1)
    uint8_t *gu_scales = nullptr;
    uint8_t *d_codes = nullptr;     // [E+m][H/128][I/64] tiles
    uint8_t *d_scales = nullptr;
    float *gate_global = nullptr;   // [E+m]
    float *up_global = nullptr;     // [E+m]
    float *down_global = nullptr;   // [E+m]
};

struct Layer {
    tfmoe_layer_desc desc{};
    int device = 0;
    int num_sms = 0;
    int gemv_max_tokens = 0;        // the descriptor's value; <= 0 = the built-in crossover
    bool loaded = false;
    void *ws_block = nullptr;
    size_t ws_bytes = 0;
    void *w_block = nullptr;
    size_t w_bytes = 0;
    Workspace ws;
    Weights w;
    int32_t last_launches = 0;
    int32_t last_T = -1;            // T of the last successful forward (stage replays need it)
    bool last_use_mma = false, last_use_gemv = false;
    bool mma_small = false;         // the tensor-core regime of the current forward uses small tiles
    void *router_maps = nullptr;    // tensor map of the router weights (router_tc.cu)
    void *gemv_maps = nullptr;      // tensor maps of the GEMV regime's scale slabs
    void *mma_maps = nullptr;       // tensor maps of the MMA regime's token operands
    // per-stage profiling (tfmoe_profile_enable)
    bool profiling = false;
    bool plain_order = false;       // launch every kernel in plain stream order (stage replays)
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

// The shared expert runs as m = Is / I extra expert slots E..E+m-1 that every token takes
// with weight 1: the plan, the expert kernels and the combine see E+m slots and k+m slots
// per token; the router and top-k see the E routed experts and k.
inline int shared_slots(const Layer &L) {
    return L.desc.shared_intermediate > 0 ? L.desc.shared_intermediate / L.desc.intermediate : 0;
}
inline int expert_slots(const Layer &L) { return L.desc.num_experts + shared_slots(L); }
inline int token_slots(const Layer &L) { return L.desc.top_k + shared_slots(L); }

// Per-expert token count up to which the GEMV regime is used, for a batch of T tokens.
inline int gemv_threshold(const Layer &L, int T) {
    if (L.gemv_max_tokens > 0) return L.gemv_max_tokens;
    return T <= kSmallBatchTokens ? T : kDefaultGemvMaxTokens;
}

// Launchers. Each returns cudaGetLastError() after its launches and adds
// the number of kernels it enqueued to *launches.
cudaError_t launch_router(Layer &L, const uint16_t *x, int T, cudaStream_t s, int *launches);
cudaError_t launch_router_tc(Layer &L, const uint16_t *x, int T, bool gemv, int32_t *seg_cnt, cudaStream_t s,
                             int *launches);
cudaError_t launch_router_norms(const Layer &L, cudaStream_t s);
cudaError_t router_setup(Layer &L);
void router_teardown(Layer &L);
cudaError_t launch_permute(Layer &L, int T, cudaStream_t s, int *launches);
cudaError_t launch_gemv(Layer &L, const uint16_t *x, int T, cudaStream_t s, int *launches);
cudaError_t launch_gemv_gate_up(Layer &L, const uint16_t *x, int T, cudaStream_t s, int *launches);
cudaError_t launch_gemv_down(Layer &L, int T, cudaStream_t s, int *launches);
// Weighted combine into out; with residual, added before the rounding; with norm_w, also
// the RMS norm of out into out_norm (one CTA per token).
cudaError_t launch_combine(Layer &L, int T, uint16_t *out, cudaStream_t s, int *launches,
                           const uint16_t *residual = nullptr, const uint16_t *norm_w = nullptr,
                           uint16_t *out_norm = nullptr);
cudaError_t launch_repack(const Layer &L, const tfmoe_weights &src, cudaStream_t s);
cudaError_t gemv_setup(Layer &L);
void gemv_teardown(Layer &L);
cudaError_t mma_setup(Layer &L);
bool mma_use_small_tiles(const Layer &L, int T);
void mma_teardown(Layer &L);
cudaError_t launch_gather(Layer &L, const uint16_t *x, int T, cudaStream_t s, int *launches);
cudaError_t launch_mma_gate_up(Layer &L, cudaStream_t s, int *launches);
cudaError_t launch_mma_down(Layer &L, cudaStream_t s, int *launches);

// cuTensorMapEncodeTiled for a 2-D tensor (dim0 contiguous), resolved through the
// runtime's driver entry point so the library does not link the driver library.
CUresult encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType type, void *base, uint64_t dim0,
                              uint64_t dim1, uint64_t row_stride_bytes, uint32_t box0, uint32_t box1,
                              CUtensorMapSwizzle swizzle);

// Sets the thread-local message returned by tfmoe_last_error() and returns st.
tfmoe_status record_error(tfmoe_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
tfmoe_status record_ok();

}  // namespace tfmoe
