// gemv.cu -- the decode regime of the NVFP4 grouped expert projections:
// bandwidth-bound GEMV on CUDA cores, no tensor cores.
//
// Decode reads each routed expert's 4-bit weights once per step, so its time
// is the weight bytes over HBM bandwidth (DGX Spark GB10 bandwidth-budget
// page, section "Mechanism: decode is bandwidth-bound, prefill is
// compute-bound"); the expert up/down kernels are the largest share of decode
// GPU time in TensorFold issue #627 (comment with the RTX 4090 per-launch
// table). The kernel streams the packed codes with 128-bit coalesced loads
// (16 in flight per lane), stages the E4M3 block scales into shared memory
// with bulk (TMA) copies one task ahead, keeps the routed activation rows in
// shared memory, and combines the two half-rows with a warp shuffle.
//
// Work item: (expert in the GEMV list, block of 64 weight rows). A CTA of 4
// warps covers the 64 rows; lane l of warp w owns row 16w + (l % 16) and half
// (l / 16) of every 64-column tile (16 code bytes = 32 weights, 2 scale bytes)
// and accumulates across all tiles of the row.
//
// Inner products (per 16-element block b of a lane's 32 weights):
//   partial_b = sum of w*x in fp32, acc += scale_b * partial_b, and the
//   per-tensor scale multiplies the finished sum.
// Two forms, chosen at compile time:
//   kMathF32  : E2M1 -> f16 (exact) -> fp32, x in fp32, packed fp32x2 FMAs.
//   kMathF16  : E2M1 -> f16 (exact), x as f16 times a power of two per
//               32-element block (exact for every bf16 value within 2^28 of the
//               block's largest), single-rounding f16*f16+f32 FMAs; the block's
//               power of two is folded into the scale.
// Gate/up rows are interleaved (row 2j = gate j, 2j+1 = up j), so lanes l and
// l^1 hold G and U of the same j and the SwiGLU epilogue
// a = bf16(silu(G) * U) runs in registers.
#include "common.cuh"
#include "internal.h"

namespace tfmoe {
namespace {

constexpr int kRowsPerTask = 64;
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kTokGroup = 4;      // activation rows staged per pass
constexpr int kBatch = 8;         // 64-column tiles per load batch (two batches in flight per lane)
constexpr int kMathF32 = 0, kMathF16 = 1;
#ifndef TFMOE_GEMV_MATH
#define TFMOE_GEMV_MATH 1
#endif
constexpr int kMath = TFMOE_GEMV_MATH;

enum class Proj { GateUp, Down };

struct GemvArgs {
    const uint8_t *codes;       // tiled codes of all experts
    const uint8_t *scales;      // tiled scales of all experts
    const float *glob0;         // gate (GateUp) or down (Down) per-tensor scale [E]
    const float *glob1;         // up (GateUp)
    int R, K;                   // rows (2I or H) and reduction length (H or I)
    const int32_t *expert_list; // GEMV-regime experts
    const int32_t *list_size;   // [0] = number of GEMV experts
    const int32_t *offsets;     // [E+1]
    const int32_t *perm;        // [P] pair index of permuted row
    int top_k;
    const uint16_t *src;        // GateUp: x [T][H]; Down: act [P][I]
    uint16_t *act_out;          // GateUp output [P][I]
    float *y_out;               // Down output [P][H]
    int I;
    int32_t *err_word;
};

__device__ __forceinline__ uint32_t byte_of(uint32_t w, int b) { return (w >> (8 * b)) & 0xFFu; }

// fp32 x and weights widened to fp32; two interleaved fp32x2 accumulators per block.
__device__ __forceinline__ void dot_f32(const uint4 c, const float *xrow, float &p0, float &p1) {
    const uint32_t words[4] = {c.x, c.y, c.z, c.w};
    float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
    const float4 *xp = reinterpret_cast<const float4 *>(xrow);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 xa = xp[2 * q], xb = xp[2 * q + 1];
        const float2 w01 = f16x2_to_float2(e2m1x2_to_f16x2(byte_of(words[q], 0)));
        const float2 w23 = f16x2_to_float2(e2m1x2_to_f16x2(byte_of(words[q], 1)));
        const float2 w45 = f16x2_to_float2(e2m1x2_to_f16x2(byte_of(words[q], 2)));
        const float2 w67 = f16x2_to_float2(e2m1x2_to_f16x2(byte_of(words[q], 3)));
        float2 &acc = (q < 2) ? a0 : a1;
        acc = __ffma2_rn(w01, make_float2(xa.x, xa.y), acc);
        acc = __ffma2_rn(w23, make_float2(xa.z, xa.w), acc);
        acc = __ffma2_rn(w45, make_float2(xb.x, xb.y), acc);
        acc = __ffma2_rn(w67, make_float2(xb.z, xb.w), acc);
    }
    p0 = a0.x + a0.y;
    p1 = a1.x + a1.y;
}

__device__ __forceinline__ float fma_f16_f32(uint32_t w2, uint32_t x2, float acc) {
    asm("{\n\t.reg .f16 wl, wh, xl, xh;\n\t"
        "mov.b32 {wl, wh}, %1;\n\tmov.b32 {xl, xh}, %2;\n\t"
        "fma.rn.f32.f16 %0, wl, xl, %0;\n\tfma.rn.f32.f16 %0, wh, xh, %0;\n\t}"
        : "+f"(acc) : "r"(w2), "r"(x2));
    return acc;
}

// f16 x (block-scaled), weights as f16, mixed-precision FMAs.
__device__ __forceinline__ void dot_f16(const uint4 c, const uint16_t *xrow, float &p0, float &p1) {
    const uint32_t words[4] = {c.x, c.y, c.z, c.w};
    const uint4 *xp = reinterpret_cast<const uint4 *>(xrow);
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 xv = xp[q];     // 8 f16 x values for this word's 8 weights
        const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
        float &u = (q < 2) ? ((q & 1) ? b0 : a0) : ((q & 1) ? b1 : a1);
#pragma unroll
        for (int b = 0; b < 4; ++b) u = fma_f16_f32(e2m1x2_to_f16x2(byte_of(words[q], b)), xs[b], u);
    }
    p0 = a0 + b0;
    p1 = a1 + b1;
}

template <Proj P>
__device__ __forceinline__ const uint16_t *src_row(const GemvArgs &a, int r) {
    return (P == Proj::GateUp) ? a.src + (size_t)(__ldg(a.perm + r) / a.top_k) * a.K : a.src + (size_t)r * a.K;
}

// Stage activation rows [r0, r0 + nt) into shared memory in the kernel's math form.
template <Proj P>
__device__ __forceinline__ void stage_x(const GemvArgs &a, int r0, int nt, float *xs32, uint16_t *xs16, float *xinv) {
    const int K = a.K;
    if (kMath == kMathF32) {
        for (int i = threadIdx.x; i < nt * (K / 8); i += kThreads) {
            const int tt = i / (K / 8), c8 = (i % (K / 8)) * 8;
            const uint4 v = *reinterpret_cast<const uint4 *>(src_row<P>(a, r0 + tt) + c8);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
            float4 lo, hi;
            lo.x = bf16_bits_to_float(u[0] & 0xFFFFu); lo.y = bf16_bits_to_float(u[0] >> 16);
            lo.z = bf16_bits_to_float(u[1] & 0xFFFFu); lo.w = bf16_bits_to_float(u[1] >> 16);
            hi.x = bf16_bits_to_float(u[2] & 0xFFFFu); hi.y = bf16_bits_to_float(u[2] >> 16);
            hi.z = bf16_bits_to_float(u[3] & 0xFFFFu); hi.w = bf16_bits_to_float(u[3] >> 16);
            *reinterpret_cast<float4 *>(xs32 + tt * K + c8) = lo;
            *reinterpret_cast<float4 *>(xs32 + tt * K + c8 + 4) = hi;
        }
    } else {
        // one thread per (token, 32-element block): the power of two 2^sh that puts the
        // block's largest magnitude just below 2^15 makes every element an exact f16
        for (int i = threadIdx.x; i < nt * (K / 32); i += kThreads) {
            const int tt = i / (K / 32), b = i % (K / 32);
            const uint16_t *srow = src_row<P>(a, r0 + tt) + b * 32;
            uint4 v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] = *reinterpret_cast<const uint4 *>(srow + 8 * q);
            uint32_t emax = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t u[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) emax = max(emax, max((u[j] >> 7) & 0xFFu, (u[j] >> 23) & 0xFFu));
            }
            int sh = 14 - ((int)emax - 127);
            sh = max(-120, min(120, sh));
            const float up = __int_as_float((127 + sh) << 23);       // exact powers of two
            xinv[tt * (K / 32) + b] = __int_as_float((127 - sh) << 23);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t u[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
                uint32_t ow[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const __half lo = __float2half_rn(bf16_bits_to_float(u[j] & 0xFFFFu) * up);
                    const __half hi = __float2half_rn(bf16_bits_to_float(u[j] >> 16) * up);
                    ow[j] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
                }
                *reinterpret_cast<uint4 *>(xs16 + tt * K + b * 32 + 8 * q) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
        }
    }
}

template <Proj P>
__global__ void __launch_bounds__(kThreads, 4) gemv_kernel(const GemvArgs a)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int K = a.K, KT = K / kTileK;
    // layout: x rows | x block scales (f16 form) | scales [2][KT][64][4] | mbarriers[2]
    uint8_t *p = smem_raw;
    float *xs32 = reinterpret_cast<float *>(p);
    uint16_t *xs16 = reinterpret_cast<uint16_t *>(p);
    p += (kMath == kMathF32) ? sizeof(float) * kTokGroup * K : sizeof(uint16_t) * kTokGroup * K;
    float *xinv = reinterpret_cast<float *>(p);
    if (kMath == kMathF16) p += sizeof(float) * kTokGroup * (K / 32);
    uint8_t *sc = p;
    const int sc_bytes = KT * kRowsPerTask * 4;
    p += 2 * (size_t)sc_bytes;
    uint64_t *bar = reinterpret_cast<uint64_t *>(p);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4, lrow = lane & 15;
    const int blocks_per_expert = a.R / kRowsPerTask;
    const int n_tasks = __ldg(a.list_size) * blocks_per_expert;
    if ((int)blockIdx.x >= n_tasks) return;
    const int RT = a.R / kTileRows;

    if (threadIdx.x == 0) { mbar_init(&bar[0], 1); mbar_init(&bar[1], 1); fence_mbar_init(); }
    __syncthreads();

    // the scales of a task (64 rows x all column tiles) are one contiguous span: one bulk copy
    auto issue_scales = [&](int task, int buf) {
        const int e = __ldg(a.expert_list + task / blocks_per_expert);
        const int blk = task % blocks_per_expert;
        const uint8_t *st = a.scales + scale_offset((size_t)e * RT + (blk >> 1), KT, blk & 1, 0);
        mbar_arrive_expect_tx(&bar[buf], (uint32_t)sc_bytes);
        bulk_g2s(sc + (size_t)buf * sc_bytes, st, (uint32_t)sc_bytes, &bar[buf]);
    };
    if (threadIdx.x == 0) issue_scales(blockIdx.x, 0);
    uint32_t phase0 = 0u, phase1 = 0u;
    int staged_e = -1, staged_g0 = -1;

    int it = 0;
    for (int task = blockIdx.x; task < n_tasks; task += gridDim.x, ++it) {
        const int buf = it & 1;
        const int e = __ldg(a.expert_list + task / blocks_per_expert);
        const int blk = task % blocks_per_expert;
        const int rt = blk >> 1, sub = blk & 1;
        const int row_in_tile = sub * kRowsPerTask + warp * 16 + lrow;
        const uint8_t *codes0 = a.codes + ((size_t)e * RT + rt) * KT * kTileCodeBytes + half * 2048 + row_in_tile * 16;
        const uint8_t *scl = sc + (size_t)buf * sc_bytes + (warp * 16 + lrow) * 4 + half * 2;
        const int r_begin = __ldg(a.offsets + e), m = __ldg(a.offsets + e + 1) - r_begin;

        __syncthreads();   // the previous task is done with x and with the other scale buffer
        if (threadIdx.x == 0 && task + (int)gridDim.x < n_tasks) issue_scales(task + gridDim.x, buf ^ 1);
        bool scales_ready = false;

        for (int g0 = 0; g0 < m; g0 += kTokGroup) {
            const int nt = min(kTokGroup, m - g0);
            // code loads of the first two batches go out before the activation staging
            uint4 cA[kBatch], cB[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                if (u < KT) cA[u] = ldg_stream_v4(codes0 + (size_t)u * kTileCodeBytes);
                if (kBatch + u < KT) cB[u] = ldg_stream_v4(codes0 + (size_t)(kBatch + u) * kTileCodeBytes);
            }
            if (e != staged_e || g0 != staged_g0) {
                if (g0 > 0) __syncthreads();
                stage_x<P>(a, r_begin + g0, nt, xs32, xs16, xinv);
                staged_e = e;
                staged_g0 = g0;
                __syncthreads();
            }
            if (!scales_ready) {
                mbar_wait_bounded(&bar[buf], buf ? phase1 : phase0, a.err_word);
                if (buf) phase1 ^= 1u; else phase0 ^= 1u;
                scales_ready = true;
            }

            float acc[kTokGroup];
#pragma unroll
            for (int t = 0; t < kTokGroup; ++t) acc[t] = 0.f;

            auto compute = [&](const uint4 (&cv)[kBatch], int kt0) {
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int kt = kt0 + u;
                    if (kt >= KT) break;
                    const uint32_t sbytes = *reinterpret_cast<const uint16_t *>(scl + kt * kRowsPerTask * 4);
                    const float2 s = f16x2_to_float2(e4m3x2_to_f16x2(sbytes));
                    const int col = kt * kTileK + half * 32;
#pragma unroll
                    for (int t = 0; t < kTokGroup; ++t) {
                        if (t < nt) {
                            float p0, p1;
                            if (kMath == kMathF32) {
                                dot_f32(cv[u], xs32 + t * K + col, p0, p1);
                                acc[t] = fmaf(s.x, p0, acc[t]);
                                acc[t] = fmaf(s.y, p1, acc[t]);
                            } else {
                                dot_f16(cv[u], xs16 + t * K + col, p0, p1);
                                const float xi = xinv[t * (K / 32) + (col >> 5)];
                                acc[t] = fmaf(s.x * xi, p0, acc[t]);
                                acc[t] = fmaf(s.y * xi, p1, acc[t]);
                            }
                        }
                    }
                }
            };
            for (int kt0 = 0; kt0 < KT; kt0 += 2 * kBatch) {
                compute(cA, kt0);
                if (kt0 + 2 * kBatch < KT) {
#pragma unroll
                    for (int u = 0; u < kBatch; ++u)
                        if (kt0 + 2 * kBatch + u < KT)
                            cA[u] = ldg_stream_v4(codes0 + (size_t)(kt0 + 2 * kBatch + u) * kTileCodeBytes);
                }
                if (kt0 + kBatch < KT) compute(cB, kt0 + kBatch);
                if (kt0 + 3 * kBatch < KT) {
#pragma unroll
                    for (int u = 0; u < kBatch; ++u)
                        if (kt0 + 3 * kBatch + u < KT)
                            cB[u] = ldg_stream_v4(codes0 + (size_t)(kt0 + 3 * kBatch + u) * kTileCodeBytes);
                }
            }
#pragma unroll
            for (int t = 0; t < kTokGroup; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 16);
            const int grow = rt * kTileRows + row_in_tile;   // row of the projection
            if (P == Proj::GateUp) {
                const bool is_up = (grow & 1) != 0;
                const float gs = is_up ? __ldg(a.glob1 + e) : __ldg(a.glob0 + e);
#pragma unroll
                for (int t = 0; t < kTokGroup; ++t) {
                    const float v = acc[t] * gs;
                    const float other = __shfl_xor_sync(0xffffffffu, v, 1);
                    if (t < nt && !is_up && half == 0) {
                        const int r = r_begin + g0 + t;
                        a.act_out[(size_t)r * a.I + (grow >> 1)] = float_to_bf16_bits_rn(silu_f32(v) * other);
                    }
                }
            } else {
                const float gs = __ldg(a.glob0 + e);
#pragma unroll
                for (int t = 0; t < kTokGroup; ++t) {
                    if (t < nt && half == 0) {
                        const int r = r_begin + g0 + t;
                        a.y_out[(size_t)r * a.R + grow] = acc[t] * gs;
                    }
                }
            }
        }
        if (!scales_ready) {   // no tokens (cannot happen for a listed expert): keep the barrier phase in step
            mbar_wait_bounded(&bar[buf], buf ? phase1 : phase0, a.err_word);
            if (buf) phase1 ^= 1u; else phase0 ^= 1u;
        }
    }
}

size_t gemv_smem_bytes(int K) {
    size_t b = (kMath == kMathF32) ? sizeof(float) * kTokGroup * (size_t)K : sizeof(uint16_t) * kTokGroup * (size_t)K;
    if (kMath == kMathF16) b += sizeof(float) * kTokGroup * (size_t)(K / 32);
    b += 2 * (size_t)(K / kTileK) * kRowsPerTask * 4;   // double-buffered scales
    return b + 2 * sizeof(uint64_t);
}

template <Proj P>
int gemv_grid(int K, int num_sms) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_kernel<P>, kThreads, gemv_smem_bytes(K)) !=
            cudaSuccess || per_sm < 1)
        per_sm = 1;
    return per_sm * num_sms;
}

}  // namespace

cudaError_t gemv_setup(Layer &L)
{
    const int H = L.desc.hidden, I = L.desc.intermediate;
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<Proj::GateUp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)gemv_smem_bytes(H));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gemv_kernel<Proj::Down>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gemv_smem_bytes(I));
    if (e != cudaSuccess) return e;
    L.gemv_grid_gu = gemv_grid<Proj::GateUp>(H, L.num_sms);
    L.gemv_grid_down = gemv_grid<Proj::Down>(I, L.num_sms);
    return cudaSuccess;
}

static GemvArgs gate_up_args(const Layer &L, const uint16_t *x) {
    GemvArgs g{};
    g.codes = L.w.gu_codes; g.scales = L.w.gu_scales;
    g.glob0 = L.w.gate_global; g.glob1 = L.w.up_global;
    g.R = 2 * L.desc.intermediate; g.K = L.desc.hidden;
    g.expert_list = L.ws.gemv_list; g.list_size = L.ws.list_sizes;
    g.offsets = L.ws.offsets; g.perm = L.ws.perm; g.top_k = L.desc.top_k;
    g.src = x; g.act_out = L.ws.act; g.y_out = nullptr; g.I = L.desc.intermediate; g.err_word = L.ws.err_word;
    return g;
}

cudaError_t launch_gemv_gate_up(Layer &L, const uint16_t *x, cudaStream_t s, int *launches)
{
    StageTimer timer(L, TFMOE_STAGE_GEMV_GATE_UP, s);
    gemv_kernel<Proj::GateUp><<<L.gemv_grid_gu, kThreads, gemv_smem_bytes(L.desc.hidden), s>>>(gate_up_args(L, x));
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_gemv_down(Layer &L, cudaStream_t s, int *launches)
{
    StageTimer timer(L, TFMOE_STAGE_GEMV_DOWN, s);
    GemvArgs d = gate_up_args(L, nullptr);
    d.codes = L.w.d_codes; d.scales = L.w.d_scales;
    d.glob0 = L.w.down_global; d.glob1 = nullptr;
    d.R = L.desc.hidden; d.K = L.desc.intermediate;
    d.src = L.ws.act; d.act_out = nullptr; d.y_out = L.ws.y;
    gemv_kernel<Proj::Down><<<L.gemv_grid_down, kThreads, gemv_smem_bytes(L.desc.intermediate), s>>>(d);
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_gemv(Layer &L, const uint16_t *x, int T, cudaStream_t s, int *launches)
{
    (void)T;
    cudaError_t e = launch_gemv_gate_up(L, x, s, launches);
    if (e == cudaSuccess) e = launch_gemv_down(L, s, launches);
    return e;
}

}  // namespace tfmoe
