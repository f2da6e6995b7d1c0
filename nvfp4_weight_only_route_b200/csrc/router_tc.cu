// router_tc.cu -- router logits and top-k for batches of more than 16 tokens.
//
// The top-k ids must equal those of the exact logits, fp32(the fp64 sum of the exact
// bf16 products) + bias, ties to the lower expert index. Computing every logit that way
// costs fp64 arithmetic on all T x E x H products. Here the products go through the bf16
// tensor cores first (fp32 accumulation), and a rigorous bound on the error of each
// approximate logit decides which experts can still be in a token's top k; only those
// are recomputed exactly (fp64, in the same way as the exact kernels), and the top k is
// taken among them on the exact values.
//
// Bound. Let S = sum_h x_h w_h and A = sum_h |x_h w_h| <= ||x||_2 ||w||_2 (Cauchy-Schwarz).
// Every product of two bf16 values is exact in fp32; a sum of H of them accumulated in fp32
// in any order, each addition in error by at most two units in the last place of its
// result, is off by at most (H + 32) 2^-22 A. The exact logit is l = fl(fl(S) + b), the
// approximation v = fl(D + b); the three further fp32 roundings (of S, and of the two bias
// additions, each at most 2^-24 of a value below 1.01 A + |b|) add less than 2^-22 A +
// 2^-23 |b|, and forming lo = fl(v - eps), hi = fl(v + eps) less than another 2^-23 A +
// 2^-23 |b|. So with both norms rounded up,
//   eps(t, e) = (H + 34) 2^-22 ||x_t|| ||w_e|| + 2^-21 |b_e|
// (constants rounded up) bounds |v - l| with the margins for those steps: the exact
// logit lies in [lo_e, hi_e]. The k-th largest lo_e, L, is at most the k-th largest exact
// logit, so every expert of the true top k (ties included) has hi_e >= L. Those experts
// are the candidates. A token whose approximations are not finite, or that has more
// candidates than the list holds, takes the exact path over every expert.
//
// Kernels: xprep (the row norms of x and the exponent range of each row, and the GEMV
// regime's block-scaled x), the tensor-core kernel (approximate logits, candidate lists),
// refine (exact candidates, top k, softmax weights, the shared slots, the large-batch plan's
// segment histograms). At weight load, router_consts_kernel computes each expert's bound
// constants and the exponent range of the router weights.
#include <algorithm>
#include <new>

#include "common.cuh"
#include "internal.h"

namespace tfmoe {
namespace {

constexpr int kRtM = 128;           // tokens per CTA (MMA M)
constexpr int kRtStages = 4;
constexpr int kRtThreads = 256;     // warp 0: TMA, warp 1: TMEM + MMA issue, warps 4-7: epilogue
constexpr int kRtMaxN = 256;        // experts (MMA N, E rounded up to 16)

struct RtArgs {
    int T, H, E, n_pad;
    const float *xnorm;             // [T]  upper bound of ||x_t||_2
    const float4 *cst;              // [E]  {bias, C_e, B_e, 0}: eps(t, e) = fma(xnorm_t, C_e, B_e)
    float *logits;                  // [T][E] approximations; the exact pass overwrites candidates
    int32_t *cand_cnt;              // [T] number of candidates, or -1: every expert
    uint16_t *cand;                 // [T][kRouterMaxCand] candidate experts, ascending
    int32_t *err_word;
};

struct RtSmem {
    uint8_t a[kRtStages][kRtM * 128];        // 128 token rows x 64 bf16, 128-byte swizzle
    uint8_t b[kRtStages][kRtMaxN * 128];     // up to 256 expert rows x 64 bf16
    float4 cst[kRtMaxN];                     // the experts' {bias, C_e, B_e, 0}
    uint64_t full[kRtStages], empty[kRtStages], dfull;
    uint32_t tmem_base;
    int32_t abort_flag;
};

__device__ __forceinline__ uint64_t rt_desc_sw128(uint32_t saddr) {
    // K-major, 128-byte swizzle: start >> 4, leading offset 1 (unused), 1024 B between 8-row
    // groups, descriptor version 1, layout type 2 (SWIZZLE_128B)
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
// kind::f16 with A and B bf16, D fp32, M = 128, N given, both K-major.
__device__ __forceinline__ uint32_t rt_idesc(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kRtM >> 4) << 24);
}
__device__ __forceinline__ void rt_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u));
}
__device__ __forceinline__ void rt_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool rt_elect() {
    uint32_t pred = 0;
    asm volatile("{\n\t.reg .b32 rx;\n\t.reg .pred px;\n\telect.sync rx|px, %1;\n\t@px mov.s32 %0, 1;\n\t}"
                 : "+r"(pred) : "r"(0xffffffffu));
    return pred != 0;
}
// Warp-collective: every lane of the warp calls it at the same point (the __syncwarp makes sure
// lanes that took different branches before it have reconverged).
__device__ __forceinline__ void rt_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    __syncwarp();
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ bool rt_wait(uint64_t *bar, uint32_t parity, int32_t *abort_flag, int32_t *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        for (int i = 0; i < 4; ++i)
            if (mbar_try_wait_sleep(bar, parity)) return true;
        if (*reinterpret_cast<volatile int32_t *>(abort_flag)) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, DEV_ERR_WAIT_TIMEOUT);
            *reinterpret_cast<volatile int32_t *>(abort_flag) = 1;
            return false;
        }
    }
}

// One CTA per 128 tokens: approximate logits of all experts in tensor memory, then one
// epilogue thread per token finds its candidates. KMAX >= k is the length of the
// epilogue's register list of the largest lower bounds; its last entry is the threshold L
// (the KMAX-th largest lower bound: the k-th largest when KMAX = k, which the launcher
// uses up to k = 8, and a smaller, still valid threshold above that).
template <int KMAX>
__global__ void __launch_bounds__(kRtThreads, 1) router_tc_kernel(const __grid_constant__ CUtensorMap mx,
                                                                  const __grid_constant__ CUtensorMap mw,
                                                                  const RtArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    RtSmem &sm = *reinterpret_cast<RtSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * kRtM;
    const int KT = a.H / kTileK;
    const uint32_t ncols = a.n_pad <= 32 ? 32u : a.n_pad <= 64 ? 64u : a.n_pad <= 128 ? 128u : 256u;
    // the experts' bound constants, once per CTA (the epilogue reads them from shared memory)
    for (int e = threadIdx.x; e < a.n_pad; e += kRtThreads)
        sm.cst[e] = e < a.E ? __ldg(a.cst + e) : make_float4(0.f, 0.f, 0.f, 0.f);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kRtStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.dfull, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&sm.tmem_base)), "r"(ncols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            const uint32_t bytes = (uint32_t)kRtM * 128u + (uint32_t)a.n_pad * 128u;
            int issued = 0;
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % kRtStages;
                const uint32_t ph = (kt / kRtStages) & 1u;
                if (!rt_wait(&sm.empty[s], ph ^ 1u, &sm.abort_flag, a.err_word)) break;
                mbar_arrive_expect_tx(&sm.full[s], bytes);
                tma_load_2d(sm.a[s], &mx, kt * kTileK, t0, &sm.full[s]);
                tma_load_2d(sm.b[s], &mw, kt * kTileK, 0, &sm.full[s]);
                issued = kt + 1;
            }
            if (sm.abort_flag)          // let the copies already issued land (bounded)
                for (int j = std::max(0, issued - kRtStages); j < issued; ++j) {
                    const uint64_t tw = global_timer_ns();
                    while (!mbar_try_wait_sleep(&sm.full[j % kRtStages], (j / kRtStages) & 1u) &&
                           global_timer_ns() - tw < kWaitLimitNs / 4) {
                    }
                }
        }
    } else if (warp == 1) {
        const uint32_t idesc = rt_idesc(a.n_pad);
        const uint64_t ad0 = rt_desc_sw128(smem_u32(sm.a[0])), bd0 = rt_desc_sw128(smem_u32(sm.b[0]));
        for (int kt = 0; kt < KT; ++kt) {
            const int s = kt % kRtStages;
            const uint32_t ph = (kt / kRtStages) & 1u;
            if (!__all_sync(0xffffffffu, rt_wait(&sm.full[s], ph, &sm.abort_flag, a.err_word))) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            if (rt_elect()) {
                const uint64_t ad = ad0 + (uint64_t)(s * (kRtM * 128 >> 4));
                const uint64_t bd = bd0 + (uint64_t)(s * (kRtMaxN * 128 >> 4));
#pragma unroll
                for (int j = 0; j < 4; ++j)      // K = 16 per MMA: 32 bytes further along each row
                    rt_mma_ss(tmem, ad + 2u * j, bd + 2u * j, idesc, (kt | j) != 0);
                rt_commit(&sm.empty[s]);
            }
            __syncwarp();
        }
        // every MMA issued (or the loop gave up): dfull reports their completion
        if (rt_elect()) rt_commit(&sm.dfull);
        __syncwarp();
    } else if (warp >= 4) {
        const int q = (warp & 3) * 32 + lane;                     // token row = TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int t = t0 + q;
        const bool ok = rt_wait(&sm.dfull, 0, &sm.abort_flag, a.err_word);
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (__all_sync(0xffffffffu, ok)) {
            const int E = a.E;
            const float xn = (t < a.T) ? __ldg(a.xnorm + t) : 0.f;
            float *__restrict__ lrow = a.logits + (size_t)t * E;
            const float4 *cst = sm.cst;
            // pass 1: approximations, and L = the KMAX-th largest lower bound (top[] holds the
            // KMAX largest lower bounds seen, descending; an insertion is a compare-exchange
            // sweep, every index static so that the list stays in registers)
            float top[KMAX];
#pragma unroll
            for (int i = 0; i < KMAX; ++i) top[i] = -INFINITY;
            float kth = -INFINITY;
            bool finite = true;
            for (int c0 = 0; c0 < a.n_pad; c0 += 16) {
                uint32_t d[16];
                rt_ld16(tmem + lane_base + (uint32_t)c0, d);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int e = c0 + i;
                    if (e < E) {
                        const float4 c = cst[e];
                        const float v = __uint_as_float(d[i]) + c.x;
                        if (t < a.T) lrow[e] = v;
                        finite = finite && fabsf(v) <= 3.402823466e38f;
                        const float lo = v - fmaf(xn, c.y, c.z);
                        if (lo > kth) {
                            float cur = lo;
#pragma unroll
                            for (int r = 0; r < KMAX; ++r) {
                                const float hi = fmaxf(top[r], cur);
                                cur = fminf(top[r], cur);
                                top[r] = hi;
                            }
                            kth = top[KMAX - 1];
                        }
                    }
                }
            }
            // pass 2: the candidates, hi_e >= L, in ascending expert order. The tensor-memory
            // loads are warp-collective (.sync.aligned): the loop bounds stay warp-uniform and a
            // token with non-finite approximations only skips the arithmetic.
            int n = 0;
            const bool any_finite = __any_sync(0xffffffffu, finite);
            for (int c0 = 0; any_finite && c0 < a.n_pad; c0 += 16) {
                uint32_t d[16];
                rt_ld16(tmem + lane_base + (uint32_t)c0, d);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int e = c0 + i;
                    if (e < E && finite) {
                        const float4 c = cst[e];
                        const float v = __uint_as_float(d[i]) + c.x;
                        const float hi = v + fmaf(xn, c.y, c.z);
                        if (hi >= kth) {
                            if (n < kRouterMaxCand && t < a.T) a.cand[(size_t)t * kRouterMaxCand + n] = (uint16_t)e;
                            ++n;
                        }
                    }
                }
            }
            if (t < a.T) a.cand_cnt[t] = (finite && n <= kRouterMaxCand) ? n : -1;
        } else if (t < a.T) {
            a.cand_cnt[t] = -1;         // no approximation: the exact pass covers every expert
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        // the epilogue's wait on dfull covered the MMAs; on an abort wait for them here (bounded)
        if (lane == 0 && sm.abort_flag) mbar_wait_bounded(&sm.dfull, 0, a.err_word);
        __syncwarp();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols));
    }
}

// One warp per token: ||x_t||_2 (fp64 sum of squares, rounded up to fp32) and, for the
// GEMV regime, x in f16 with a power of two per 16-element block.
// The exponent field of a bf16 value folded into a running (smallest, largest) over nonzero
// values (a subnormal counts as 0, an infinity or NaN as 255).
__device__ __forceinline__ void exp_range(uint32_t b, uint32_t &emin, uint32_t &emax) {
    if (b & 0x7FFFu) {
        const uint32_t e = (b >> 7) & 0xFFu;
        emin = min(emin, e);
        emax = max(emax, e);
    }
}

// One warp per token: ||x_t||_2 (fp64 sum of squares, rounded up to fp32), the exponent range
// of x_t's nonzero elements, and, for the GEMV regime, x in f16 with a power of two per
// 16-element block.
__global__ void __launch_bounds__(256) xprep_kernel(const uint16_t *__restrict__ x, int T, int H,
                                                    float *__restrict__ xnorm, int32_t *__restrict__ xexp, uint16_t *xq,
                                                    float *xq_inv)
{
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= T) return;
    const uint16_t *row = x + (size_t)t * H;
    double ss = 0.0;
    uint32_t emin = 255u, emax = 0u;
    for (int c = lane * 8; c < H; c += 256) {
        const uint4 v = *reinterpret_cast<const uint4 *>(row + c);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const double lo = bf16_bits_to_float(u[j] & 0xFFFFu), hi = bf16_bits_to_float(u[j] >> 16);
            ss = fma(lo, lo, ss);
            ss = fma(hi, hi, ss);
            exp_range(u[j] & 0xFFFFu, emin, emax);
            exp_range(u[j] >> 16, emin, emax);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    emin = __reduce_min_sync(0xffffffffu, emin);
    emax = __reduce_max_sync(0xffffffffu, emax);
    if (lane == 0) {
        xnorm[t] = (float)(sqrt(ss) * (1.0 + 0x1p-18));
        xexp[t] = (int32_t)(emin | (emax << 16));
    }
    if (xq)
        for (int b = lane; b < H / 16; b += 32) {
            const size_t off = (size_t)t * H + (size_t)b * 16;
            xq_inv[off / 16] = block16_bf16_to_f16(x + off, xq + off);
        }
}

// Per router row (at weight load): ||w_e||_2 rounded up, and the bound's constants
// C_e = (H + 34) 2^-22 ||w_e|| and B_e = 2^-21 |b_e| + 2^-126, both rounded up (the
// factor 1 + 2^-18 also covers the rounding of the fma that forms eps).
__global__ void __launch_bounds__(256) router_consts_kernel(const uint16_t *__restrict__ w, const float *bias,
                                                            int E, int H, float4 *__restrict__ cst,
                                                            int32_t *__restrict__ wexp)
{
    const int e = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (e >= E) return;
    double ss = 0.0;
    uint32_t emin = 255u, emax = 0u;
    for (int c = lane; c < H; c += 32) {
        const uint16_t b = w[(size_t)e * H + c];
        const double v = bf16_bits_to_float(b);
        ss = fma(v, v, ss);
        exp_range(b, emin, emax);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    emin = __reduce_min_sync(0xffffffffu, emin);
    emax = __reduce_max_sync(0xffffffffu, emax);
    if (lane == 0) {
        atomicMin(wexp, (int32_t)emin);
        atomicMax(wexp + 1, (int32_t)emax);
        const double up = 1.0 + 0x1p-18;
        const double wn = sqrt(ss) * up;
        const float b = bias ? bias[e] : 0.f;
        cst[e] = make_float4(b, (float)(wn * (double)(H + 34) * 0x1p-22 * up),
                             (float)(fabs((double)b) * 0x1p-21 * up) + 0x1p-126f, 0.f);
    }
}

// Order-preserving key of a finite fp32 logit (-0 counts as +0); larger logit, larger key.
__device__ __forceinline__ uint32_t rt_key(float v) {
    uint32_t b = __float_as_uint(v);
    if ((b << 1) == 0u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One warp per token: exact logits of the candidates (every expert when cand_cnt is -1), the
// top k among them (ties to the lower expert index) and the softmax weights, then the m
// shared slots (experts E..E+m-1, weight 1) -- rows of k + m ids and weights; with seg_cnt,
// the expert-slot histogram of this CTA's 8 tokens for the multi-CTA plan.
constexpr int kRefTokens = kPlanSegTokens;
__global__ void __launch_bounds__(256) router_refine_kernel(
    const uint16_t *__restrict__ x, const uint16_t *__restrict__ wr, const float *__restrict__ bias, int T, int H,
    int E, int k, int m, float *__restrict__ logits, const int32_t *__restrict__ cand_cnt,
    const uint16_t *__restrict__ cand, int32_t *__restrict__ ids, float *__restrict__ wts, int32_t *err_word,
    int debug, int32_t *seg_cnt, const int32_t *__restrict__ xexp, const int32_t *__restrict__ wexp)
{
    __shared__ int32_t ids_s[kRefTokens * 32];
    __shared__ int32_t cnt_s[256];
    const int kx = k + m, ES = E + m;
    if (seg_cnt)
        for (int e = threadIdx.x; e < ES; e += blockDim.x) cnt_s[e] = 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kRefTokens + warp;
    if (t < T) {
        int n = __ldg(cand_cnt + t);
        const bool all = n < 0 || n > kRouterMaxCand;
        if (all) n = E;
        const uint16_t *xrow = x + (size_t)t * H;
        // Every product of a bf16 x element and a bf16 weight is exact in fp32 (16 significant
        // bits) when it lies in fp32's normal range: nonzero elements normal, and the exponent
        // fields with ex + ew in [128, 380] for every pair. Then the fp64 accumulation of the fp32
        // product, acc + (double)(x * w), rounds exactly like fma((double)x, (double)w, acc) and
        // needs one fp32 -> fp64 conversion instead of two.
        const int32_t xr = __ldg(xexp + t);
        const int xmin = xr & 0xFFFF, xmax = xr >> 16, wmin = __ldg(wexp), wmax = __ldg(wexp + 1);
        const bool fast = xmin >= 1 && wmin >= 1 && xmax <= 254 && wmax <= 254 && xmin + wmin >= 128 &&
                          xmax + wmax <= 380;
        // candidate j sits in lane j % 32, slot j / 32 (n <= 256)
        uint32_t key[8];
        int eid[8];
        float lv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) { key[i] = 0u; eid[i] = -1; lv[i] = 0.f; }
        for (int j = 0; j < n; ++j) {
            const int e = all ? j : min((int)__ldg(cand + (size_t)t * kRouterMaxCand + j), E - 1);
            const uint16_t *wrow = wr + (size_t)e * H;
            double acc = 0.0;
            if (fast) {
#pragma unroll 4
                for (int c = lane * 8; c < H; c += 256) {
                    const uint4 xv = *reinterpret_cast<const uint4 *>(xrow + c);
                    const uint4 wv = *reinterpret_cast<const uint4 *>(wrow + c);
                    const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w}, wu[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        acc += (double)__fmul_rn(bf16_bits_to_float(xu[i] & 0xFFFFu), bf16_bits_to_float(wu[i] & 0xFFFFu));
                        acc += (double)__fmul_rn(bf16_bits_to_float(xu[i] >> 16), bf16_bits_to_float(wu[i] >> 16));
                    }
                }
            } else {
#pragma unroll 4
                for (int c = lane * 8; c < H; c += 256) {
                    const uint4 xv = *reinterpret_cast<const uint4 *>(xrow + c);
                    const uint4 wv = *reinterpret_cast<const uint4 *>(wrow + c);
                    const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w}, wu[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        acc = fma((double)bf16_bits_to_float(xu[i] & 0xFFFFu), (double)bf16_bits_to_float(wu[i] & 0xFFFFu), acc);
                        acc = fma((double)bf16_bits_to_float(xu[i] >> 16), (double)bf16_bits_to_float(wu[i] >> 16), acc);
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            float l = (float)acc;
            if (bias) l = l + __ldg(bias + e);
            if (debug && !isfinite(l)) atomicOr(err_word, DEV_ERR_NONFINITE);
            if (lane == 0) logits[(size_t)t * E + e] = l;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (j == 32 * i + lane) { key[i] = rt_key(l); eid[i] = e; lv[i] = l; }
        }
        // top k: k rounds of a warp-wide max of the keys, then the lowest expert holding it
        uint32_t taken = 0;
        float sel_first = 0.f, my_sel = 0.f;
        int my_id = -1;
        for (int s = 0; s < k; ++s) {
            uint32_t bk = 0u;
            bool any = false;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (eid[i] >= 0 && !(taken & (1u << i)) && (!any || key[i] > bk)) { bk = key[i]; any = true; }
            const uint32_t mk = __reduce_max_sync(0xffffffffu, any ? bk : 0u);
            uint32_t mine = 0xffffffffu;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (eid[i] >= 0 && !(taken & (1u << i)) && key[i] == mk) mine = min(mine, (uint32_t)eid[i]);
            const uint32_t win = __reduce_min_sync(0xffffffffu, mine);
            float wv = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (eid[i] == (int)win) { taken |= 1u << i; wv = lv[i]; }
            wv = __shfl_sync(0xffffffffu, wv, __ffs(__ballot_sync(0xffffffffu, mine == win)) - 1);
            if (s == 0) sel_first = wv;
            if (lane == s) { my_sel = wv; my_id = (int)win; }
        }
        const float ex = (lane < k) ? expf(my_sel - sel_first) : 0.f;
        float den = ex;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        if (lane < kx) {
            const int id = lane < k ? my_id : E + lane - k;
            ids[(size_t)t * kx + lane] = id;
            wts[(size_t)t * kx + lane] = lane < k ? ex / den : 1.f;
            ids_s[warp * kx + lane] = id;
        }
    }
    if (!seg_cnt) return;
    __syncthreads();
    const int n = min(kRefTokens, T - (int)blockIdx.x * kRefTokens) * kx;
    for (int i = threadIdx.x; i < n; i += blockDim.x) atomicAdd(&cnt_s[ids_s[i]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < ES; e += blockDim.x) seg_cnt[(size_t)blockIdx.x * ES + e] = cnt_s[e];
}

}  // namespace

struct RouterMaps {
    CUtensorMap w;                  // router weights [E][H] bf16, box 64 x n_pad
};

cudaError_t router_setup(Layer &L)
{
    const int H = L.desc.hidden, E = L.desc.num_experts;
    RouterMaps *rm = new (std::nothrow) RouterMaps();
    if (!rm) return cudaErrorMemoryAllocation;
    const int n_pad = (E + 15) & ~15;
    if (encode_tensor_map_2d(&rm->w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L.w.router_w, (uint64_t)H, (uint64_t)E,
                             (uint64_t)H * 2, (uint32_t)kTileK, (uint32_t)n_pad, CU_TENSOR_MAP_SWIZZLE_128B) !=
        CUDA_SUCCESS) {
        delete rm;
        return cudaErrorInvalidValue;
    }
    L.router_maps = rm;
    const int bytes = (int)(sizeof(RtSmem) + 1024);
    const void *fns[] = {(const void *)router_tc_kernel<1>, (const void *)router_tc_kernel<2>,
                         (const void *)router_tc_kernel<3>, (const void *)router_tc_kernel<4>,
                         (const void *)router_tc_kernel<5>, (const void *)router_tc_kernel<6>,
                         (const void *)router_tc_kernel<7>, (const void *)router_tc_kernel<8>,
                         (const void *)router_tc_kernel<16>, (const void *)router_tc_kernel<kRouterMaxK>};
    cudaError_t e = cudaSuccess;
    for (const void *f : fns)
        if (e == cudaSuccess) e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    return e;
}

void router_teardown(Layer &L)
{
    delete static_cast<RouterMaps *>(L.router_maps);
    L.router_maps = nullptr;
}

cudaError_t launch_router_norms(const Layer &L, cudaStream_t s)
{
    // exponent range of the weights: smallest starts at 0x7F7F7F7F, largest at 0
    cudaError_t e = cudaMemsetAsync(L.w.router_wexp, 0x7F, sizeof(int32_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(L.w.router_wexp + 1, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    router_consts_kernel<<<(L.desc.num_experts + 7) / 8, 256, 0, s>>>(
        L.w.router_w, L.desc.has_router_bias ? L.w.router_bias : nullptr, L.desc.num_experts, L.desc.hidden,
        L.w.router_cst, L.w.router_wexp);
    return cudaGetLastError();
}

cudaError_t launch_router_tc(Layer &L, const uint16_t *x, int T, bool gemv, int32_t *seg_cnt, cudaStream_t s,
                             int *launches)
{
    const int H = L.desc.hidden, E = L.desc.num_experts, k = L.desc.top_k;
    const int n_pad = (E + 15) & ~15;
    CUtensorMap mx;
    if (encode_tensor_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<uint16_t *>(x), (uint64_t)H,
                             (uint64_t)T, (uint64_t)H * 2, (uint32_t)kTileK, (uint32_t)kRtM,
                             CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const float *bias = L.desc.has_router_bias ? L.w.router_bias : nullptr;
    {
        StageTimer timer(L, TFMOE_STAGE_ROUTER, s);
        xprep_kernel<<<(T + 7) / 8, 256, 0, s>>>(x, T, H, L.ws.xnorm, L.ws.xexp, gemv ? L.ws.xq : nullptr,
                                                 L.ws.xq_inv);
        RtArgs a{};
        a.T = T; a.H = H; a.E = E; a.n_pad = n_pad;
        a.xnorm = L.ws.xnorm;
        a.cst = L.w.router_cst;
        a.logits = L.ws.logits;
        a.cand_cnt = L.ws.cand_cnt;
        a.cand = L.ws.cand;
        a.err_word = L.ws.err_word;
        const CUtensorMap &mw = static_cast<const RouterMaps *>(L.router_maps)->w;
        const dim3 grid((T + kRtM - 1) / kRtM);
        const size_t smem = sizeof(RtSmem) + 1024;
        switch (k <= 8 ? k : k <= 16 ? 16 : 32) {
        case 1: router_tc_kernel<1><<<grid, kRtThreads, smem, s>>>(mx, mw, a); break;
        case 2: router_tc_kernel<2><<<grid, kRtThreads, smem, s>>>(mx, mw, a); break;
        case 3: router_tc_kernel<3><<<grid, kRtThreads, smem, s>>>(mx, mw, a); break;
        case 4: router_tc_kernel<4><<<grid, kRtThreads, smem, s>>>(mx, mw, a); break;
        case 5: router_tc_kernel<5><<<grid, kRtThreads, smem, s>>>(mx, mw, a); break;
        case 6: router_tc_kernel<6><<<grid, kRtThreads, smem, s>>>(mx, mw, a); break;
        case 7: router_tc_kernel<7><<<grid, kRtThreads, smem, s>>>(mx, mw, a); break;
        case 8: router_tc_kernel<8><<<grid, kRtThreads, smem, s>>>(mx, mw, a); break;
        case 16: router_tc_kernel<16><<<grid, kRtThreads, smem, s>>>(mx, mw, a); break;
        default: router_tc_kernel<kRouterMaxK><<<grid, kRtThreads, smem, s>>>(mx, mw, a); break;
        }
    }
    {
        StageTimer timer(L, TFMOE_STAGE_TOPK, s);
        router_refine_kernel<<<(T + kRefTokens - 1) / kRefTokens, 256, 0, s>>>(
            x, L.w.router_w, bias, T, H, E, k, shared_slots(L), L.ws.logits, L.ws.cand_cnt, L.ws.cand, L.ws.ids,
            L.ws.topk_w,
            L.ws.err_word, (L.desc.flags & TFMOE_FLAG_DEBUG_CHECKS) ? 1 : 0, seg_cnt, L.ws.xexp, L.w.router_wexp);
    }
    *launches += 3;
    return cudaGetLastError();
}

}  // namespace tfmoe
