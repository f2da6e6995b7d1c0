// gemv.cu -- the decode regime of the NVFP4 grouped expert projections:
// bandwidth-bound GEMV on CUDA cores, no tensor cores.
//
// Decode reads each routed expert's 4-bit weights once per step, so its time
// is the weight bytes over HBM bandwidth (DGX Spark GB10 bandwidth-budget
// page, section "Mechanism: decode is bandwidth-bound, prefill is
// compute-bound"); the expert up/down kernels are the largest share of decode
// GPU time in TensorFold issue #627 (comment with the RTX 4090 per-launch
// table). The kernel therefore streams the packed codes with 128-bit
// coalesced loads, stages the E4M3 block scales into shared memory with bulk
// (TMA) copies, keeps the few routed activation rows in shared memory as
// fp32, and reduces with warp shuffles.
//
// Work item: (expert in the GEMV list, block of 32 weight rows). A CTA of 8
// warps = 2 row groups of 16 rows x 4 splits of the reduction dimension.
// Lane l of a warp owns row (l % 16) of its group and half (l / 16) of every
// 64-column tile: 16 code bytes = 32 weights and 2 scale bytes per tile.
//
// Arithmetic per tile: w = E2M1 (exact in f16, widened to fp32),
// partial_b = sum of 16 w*x in fp32, acc += E4M3 scale_b * partial_b; the
// per-tensor scale multiplies the finished sum. Gate/up rows are interleaved
// (row 2j = gate j, 2j+1 = up j), so lanes l and l^1 hold G and U of the same
// j and the SwiGLU epilogue a = bf16(silu(G) * U) runs in registers.
#include "common.cuh"
#include "internal.h"

namespace tfmoe {
namespace {

constexpr int kRowsPerCta = 32;
constexpr int kKSplit = 4;
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTokGroup = 4;      // activation rows staged per pass
constexpr int kUnroll = 8;        // 64-column tiles loaded ahead per warp

enum class Proj { GateUp, Down };

template <Proj P>
struct GemvArgs {
    const uint8_t *codes;       // tiled codes of all experts
    const uint8_t *scales;      // tiled scales of all experts
    const float *glob0;         // gate (GateUp) or down (Down) per-tensor scale [E]
    const float *glob1;         // up (GateUp) or unused
    int R, K;                   // rows (2I or H) and reduction length (H or I)
    const int32_t *expert_list; // GEMV-regime experts
    const int32_t *list_size;   // [0] = number of GEMV experts
    const int32_t *offsets;     // [E+1]
    const int32_t *perm;        // [P] pair index of permuted row
    int top_k;
    const uint16_t *src;        // GateUp: x [T][H]; Down: act [P][I]
    uint16_t *act_out;          // GateUp output [P][I]
    float *y_out;               // Down output [P][H]
    int I;                      // intermediate size (GateUp output row length)
    int32_t *err_word;
};

__device__ __forceinline__ void decode32(const uint4 c, float w[32]) {
    const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const float2 f = f16x2_to_float2(e2m1x2_to_f16x2((words[q] >> (8 * b)) & 0xFFu));
            w[8 * q + 2 * b] = f.x;
            w[8 * q + 2 * b + 1] = f.y;
        }
    }
}

template <Proj P>
__global__ void __launch_bounds__(kThreads) gemv_kernel(const GemvArgs<P> a)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    // layout: xs[kTokGroup][K] fp32 | scales[32 rows][K/16] bytes | red | mbarrier
    float *xs = reinterpret_cast<float *>(smem_raw);
    uint8_t *sc = smem_raw + sizeof(float) * kTokGroup * a.K;
    const int KT = a.K / kTileK;
    float *red = reinterpret_cast<float *>(sc + kRowsPerCta * 4 * KT);   // [kKSplit][32 rows][kTokGroup]
    uint64_t *bar = reinterpret_cast<uint64_t *>(red + kKSplit * kRowsPerCta * kTokGroup);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rg = warp / kKSplit, ks = warp % kKSplit;
    const int half = lane >> 4, lrow = lane & 15;
    const int blocks_per_expert = a.R / kRowsPerCta;
    const int n_tasks = a.list_size[0] * blocks_per_expert;
    // contiguous task range per CTA
    const int per = (n_tasks + gridDim.x - 1) / gridDim.x;
    const int task_begin = blockIdx.x * per, task_end = min(n_tasks, task_begin + per);
    if (task_begin >= task_end) return;

    if (threadIdx.x == 0) { mbar_init(bar, 1); fence_mbar_init(); }
    __syncthreads();
    uint32_t phase = 0;
    const size_t tiles_per_row_tile = (size_t)KT;
    const size_t expert_tiles = (size_t)(a.R / kTileRows) * tiles_per_row_tile;

    for (int task = task_begin; task < task_end; ++task) {
        const int e = a.expert_list[task / blocks_per_expert];
        const int blk = task % blocks_per_expert;
        const int rt = blk / (kTileRows / kRowsPerCta), sub = blk % (kTileRows / kRowsPerCta);
        const int row_in_tile = sub * kRowsPerCta + rg * 16 + lrow;
        const uint8_t *tile0 = a.codes + ((size_t)e * expert_tiles + (size_t)rt * tiles_per_row_tile) * kTileCodeBytes;
        const uint8_t *stile0 = a.scales + ((size_t)e * expert_tiles + (size_t)rt * tiles_per_row_tile) * kTileScaleBytes;
        const int r_begin = a.offsets[e], m = a.offsets[e + 1] - r_begin;

        __syncthreads();   // previous task done with sc / xs / red
        // Stage this CTA's 32 rows of scales: 128 bytes per 64-column tile.
        if (threadIdx.x == 0) {
            mbar_arrive_expect_tx(bar, (uint32_t)(kRowsPerCta * 4 * KT));
            for (int kt = 0; kt < KT; ++kt)
                bulk_g2s(sc + kt * kRowsPerCta * 4, stile0 + (size_t)kt * kTileScaleBytes + sub * kRowsPerCta * 4,
                         kRowsPerCta * 4, bar);
        }
        bool scales_ready = false;

        for (int g0 = 0; g0 < m; g0 += kTokGroup) {
            const int nt = min(kTokGroup, m - g0);
            if (g0 > 0) __syncthreads();
            // stage activation rows as fp32
            for (int i = threadIdx.x; i < nt * (a.K / 8); i += kThreads) {
                const int tt = i / (a.K / 8), c8 = (i % (a.K / 8)) * 8;
                const int r = r_begin + g0 + tt;
                const uint16_t *srow;
                if (P == Proj::GateUp) srow = a.src + (size_t)(a.perm[r] / a.top_k) * a.K;
                else srow = a.src + (size_t)r * a.K;
                const uint4 v = *reinterpret_cast<const uint4 *>(srow + c8);
                float4 lo, hi;
                lo.x = bf16_bits_to_float(v.x & 0xFFFFu); lo.y = bf16_bits_to_float(v.x >> 16);
                lo.z = bf16_bits_to_float(v.y & 0xFFFFu); lo.w = bf16_bits_to_float(v.y >> 16);
                hi.x = bf16_bits_to_float(v.z & 0xFFFFu); hi.y = bf16_bits_to_float(v.z >> 16);
                hi.z = bf16_bits_to_float(v.w & 0xFFFFu); hi.w = bf16_bits_to_float(v.w >> 16);
                *reinterpret_cast<float4 *>(xs + tt * a.K + c8) = lo;
                *reinterpret_cast<float4 *>(xs + tt * a.K + c8 + 4) = hi;
            }
            __syncthreads();
            if (!scales_ready) {
                mbar_wait_bounded(bar, phase, a.err_word);
                phase ^= 1;
                scales_ready = true;
            }

            float acc[kTokGroup];
#pragma unroll
            for (int t = 0; t < kTokGroup; ++t) acc[t] = 0.f;

            for (int kt0 = ks; kt0 < KT; kt0 += kKSplit * kUnroll) {
                uint4 cv[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int kt = kt0 + u * kKSplit;
                    if (kt < KT)
                        cv[u] = ldg_stream_v4(tile0 + (size_t)kt * kTileCodeBytes + half * 2048 + row_in_tile * 16);
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int kt = kt0 + u * kKSplit;
                    if (kt >= KT) break;
                    const uint32_t sbytes = *reinterpret_cast<const uint16_t *>(
                        sc + kt * kRowsPerCta * 4 + (rg * 16 + lrow) * 4 + half * 2);
                    const float2 s = f16x2_to_float2(e4m3x2_to_f16x2(sbytes));
                    float w[32];
                    decode32(cv[u], w);
                    const int col = kt * kTileK + half * 32;
#pragma unroll
                    for (int t = 0; t < kTokGroup; ++t) {
                        if (t < nt) {
                            const float4 *xp = reinterpret_cast<const float4 *>(xs + t * a.K + col);
                            float p0 = 0.f, p1 = 0.f;
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float4 xv = xp[q];
                                p0 = fmaf(w[4 * q], xv.x, p0);
                                p0 = fmaf(w[4 * q + 1], xv.y, p0);
                                p0 = fmaf(w[4 * q + 2], xv.z, p0);
                                p0 = fmaf(w[4 * q + 3], xv.w, p0);
                            }
#pragma unroll
                            for (int q = 4; q < 8; ++q) {
                                const float4 xv = xp[q];
                                p1 = fmaf(w[4 * q], xv.x, p1);
                                p1 = fmaf(w[4 * q + 1], xv.y, p1);
                                p1 = fmaf(w[4 * q + 2], xv.z, p1);
                                p1 = fmaf(w[4 * q + 3], xv.w, p1);
                            }
                            acc[t] = fmaf(s.x, p0, acc[t]);
                            acc[t] = fmaf(s.y, p1, acc[t]);
                        }
                    }
                }
            }
            // halves -> one value per row, then the K splits through shared memory
#pragma unroll
            for (int t = 0; t < kTokGroup; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 16);
            if (half == 0) {
#pragma unroll
                for (int t = 0; t < kTokGroup; ++t)
                    red[(ks * kRowsPerCta + rg * 16 + lrow) * kTokGroup + t] = acc[t];
            }
            __syncthreads();
            if (ks == 0) {
                // warps (rg, 0): lanes 0..15 finish rows of group rg; fixed summation order
                float tot[kTokGroup];
#pragma unroll
                for (int t = 0; t < kTokGroup; ++t) {
                    float v = 0.f;
#pragma unroll
                    for (int s2 = 0; s2 < kKSplit; ++s2) v += red[(s2 * kRowsPerCta + rg * 16 + lrow) * kTokGroup + t];
                    tot[t] = v;
                }
                const int grow = rt * kTileRows + row_in_tile;   // row of the projection
                if (P == Proj::GateUp) {
                    const bool is_up = (grow & 1) != 0;
                    const float gs = is_up ? a.glob1[e] : a.glob0[e];
#pragma unroll
                    for (int t = 0; t < kTokGroup; ++t) {
                        const float v = tot[t] * gs;
                        const float other = __shfl_xor_sync(0xffffffffu, v, 1);
                        if (t < nt && !is_up && half == 0) {
                            const float G = v, U = other;
                            const int j = grow >> 1;
                            const int r = r_begin + g0 + t;
                            a.act_out[(size_t)r * a.I + j] = float_to_bf16_bits_rn(silu_f32(G) * U);
                        }
                    }
                } else {
                    const float gs = a.glob0[e];
#pragma unroll
                    for (int t = 0; t < kTokGroup; ++t) {
                        if (t < nt && half == 0) {
                            const int r = r_begin + g0 + t;
                            a.y_out[(size_t)r * a.R + grow] = tot[t] * gs;
                        }
                    }
                }
            }
        }
        if (!scales_ready) {   // no tokens (cannot happen for a listed expert): keep the barrier phase in step
            mbar_wait_bounded(bar, phase, a.err_word);
            phase ^= 1;
        }
    }
}

template <Proj P>
size_t gemv_smem_bytes(int K) {
    return sizeof(float) * kTokGroup * (size_t)K + (size_t)kRowsPerCta * 4 * (K / kTileK) +
           sizeof(float) * kKSplit * kRowsPerCta * kTokGroup + 16;
}

template <Proj P>
int gemv_grid(int K, int num_sms) {
    const size_t smem = gemv_smem_bytes<P>(K);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_kernel<P>, kThreads, smem) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    return per_sm * num_sms;
}

}  // namespace

cudaError_t gemv_setup(Layer &L)
{
    const int H = L.desc.hidden, I = L.desc.intermediate;
    cudaError_t e1 = cudaFuncSetAttribute(gemv_kernel<Proj::GateUp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)gemv_smem_bytes<Proj::GateUp>(H));
    if (e1 != cudaSuccess) return e1;
    cudaError_t e2 = cudaFuncSetAttribute(gemv_kernel<Proj::Down>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)gemv_smem_bytes<Proj::Down>(I));
    if (e2 != cudaSuccess) return e2;
    L.gemv_grid_gu = gemv_grid<Proj::GateUp>(H, L.num_sms);
    L.gemv_grid_down = gemv_grid<Proj::Down>(I, L.num_sms);
    return cudaSuccess;
}

cudaError_t launch_gemv(Layer &L, const uint16_t *x, int T, cudaStream_t s, int *launches)
{
    (void)T;
    const int H = L.desc.hidden, I = L.desc.intermediate;
    GemvArgs<Proj::GateUp> gu{};
    gu.codes = L.w.gu_codes; gu.scales = L.w.gu_scales;
    gu.glob0 = L.w.gate_global; gu.glob1 = L.w.up_global;
    gu.R = 2 * I; gu.K = H; gu.expert_list = L.ws.gemv_list; gu.list_size = L.ws.list_sizes;
    gu.offsets = L.ws.offsets; gu.perm = L.ws.perm; gu.top_k = L.desc.top_k;
    gu.src = x; gu.act_out = L.ws.act; gu.I = I; gu.err_word = L.ws.err_word;
    {
        StageTimer timer(L, TFMOE_STAGE_GEMV_GATE_UP, s);
        gemv_kernel<Proj::GateUp><<<L.gemv_grid_gu, kThreads, gemv_smem_bytes<Proj::GateUp>(H), s>>>(gu);
    }

    GemvArgs<Proj::Down> dn{};
    dn.codes = L.w.d_codes; dn.scales = L.w.d_scales;
    dn.glob0 = L.w.down_global; dn.glob1 = nullptr;
    dn.R = H; dn.K = I; dn.expert_list = L.ws.gemv_list; dn.list_size = L.ws.list_sizes;
    dn.offsets = L.ws.offsets; dn.perm = L.ws.perm; dn.top_k = L.desc.top_k;
    dn.src = L.ws.act; dn.y_out = L.ws.y; dn.I = I; dn.err_word = L.ws.err_word;
    {
        StageTimer timer(L, TFMOE_STAGE_GEMV_DOWN, s);
        gemv_kernel<Proj::Down><<<L.gemv_grid_down, kThreads, gemv_smem_bytes<Proj::Down>(I), s>>>(dn);
    }
    *launches += 2;
    return cudaGetLastError();
}

}  // namespace tfmoe
