// route.cu -- router logits, top-k + softmax weights, and the expert
// permutation ("plan") of the MoE layer.
//
// Router and top-k are the first two launches of the MoE chain in
// TensorFold issue #627 (per-launch kernel table: router, topk); the pages'
// fused one-block router was slower because it serialised a row's expert dot
// products on one SM (issue #627, comment on tf_nemo_route_row), so the
// logits here keep a wide grid: one warp per (expert, token group) for
// decode-sized T, a 64x64 register-tiled kernel for large T.
//
// Logits are the fp64 sum of exact bf16*bf16 products rounded once to fp32,
// then plus the fp32 bias: this makes the top-k ids bit-reproducible against
// a float64 reference (issue #627, "Description": error stated against a
// 64-bit reference).
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace tfmoe {
namespace {

constexpr int kSmallTokens = 8;     // tokens per warp in the small-T router kernel

// One warp per (expert, group of <= 8 tokens). Lane l covers 8 consecutive
// columns per 256-column step.
__global__ void __launch_bounds__(128) router_small_kernel(
    const uint16_t *__restrict__ x, const uint16_t *__restrict__ wr, const float *__restrict__ bias,
    float *__restrict__ logits, int T, int H, int E, int32_t *err_word, int debug)
{
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int n_groups = (T + kSmallTokens - 1) / kSmallTokens;
    if (warp >= E * n_groups) return;
    const int e = warp % E;
    const int t0 = (warp / E) * kSmallTokens;
    const int nt = min(kSmallTokens, T - t0);
    double acc[kSmallTokens];
#pragma unroll
    for (int i = 0; i < kSmallTokens; ++i) acc[i] = 0.0;
    const uint16_t *wrow = wr + (size_t)e * H;
    for (int c = lane * 8; c < H; c += 256) {
        uint4 wv = *reinterpret_cast<const uint4 *>(wrow + c);
        double w[8];
        const uint32_t wu[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            w[2 * i] = (double)bf16_bits_to_float(wu[i] & 0xFFFFu);
            w[2 * i + 1] = (double)bf16_bits_to_float(wu[i] >> 16);
        }
#pragma unroll
        for (int t = 0; t < kSmallTokens; ++t) {
            if (t < nt) {
                uint4 xv = *reinterpret_cast<const uint4 *>(x + (size_t)(t0 + t) * H + c);
                const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[t] = fma((double)bf16_bits_to_float(xu[i] & 0xFFFFu), w[2 * i], acc[t]);
                    acc[t] = fma((double)bf16_bits_to_float(xu[i] >> 16), w[2 * i + 1], acc[t]);
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < kSmallTokens; ++t) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
    }
    if (lane < nt) {
        double v = acc[0];
#pragma unroll
        for (int t = 1; t < kSmallTokens; ++t)
            if (lane == t) v = acc[t];
        float l = (float)v;
        if (bias) l = l + bias[e];
        if (debug && !isfinite(l)) atomicOr(err_word, DEV_ERR_NONFINITE);
        logits[(size_t)(t0 + lane) * E + e] = l;
    }
}

// 64 tokens x 64 experts per CTA, 256 threads, 4x4 fp64 accumulators per
// thread, K staged through shared memory in steps of 32 (converted to fp64).
constexpr int RT_T = 64, RT_E = 64, RT_K = 32;
__global__ void __launch_bounds__(256) router_tiled_kernel(
    const uint16_t *__restrict__ x, const uint16_t *__restrict__ wr, const float *__restrict__ bias,
    float *__restrict__ logits, int T, int H, int E, int32_t *err_word, int debug)
{
    __shared__ double xs[RT_K][RT_T + 1];
    __shared__ double ws[RT_K][RT_E + 1];
    const int t_base = blockIdx.x * RT_T, e_base = blockIdx.y * RT_E;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    for (int k0 = 0; k0 < H; k0 += RT_K) {
        // 64 rows x 32 columns of x and of wr: 2048 elements each, 8 per thread.
        for (int i = threadIdx.x; i < RT_T * RT_K / 8; i += 256) {
            const int row = i / (RT_K / 8), col = (i % (RT_K / 8)) * 8;
            const int t = t_base + row, e = e_base + row;
            uint4 xv = make_uint4(0, 0, 0, 0), wv = make_uint4(0, 0, 0, 0);
            if (t < T) xv = *reinterpret_cast<const uint4 *>(x + (size_t)t * H + k0 + col);
            if (e < E) wv = *reinterpret_cast<const uint4 *>(wr + (size_t)e * H + k0 + col);
            const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w}, wu[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                xs[col + 2 * j][row] = (double)bf16_bits_to_float(xu[j] & 0xFFFFu);
                xs[col + 2 * j + 1][row] = (double)bf16_bits_to_float(xu[j] >> 16);
                ws[col + 2 * j][row] = (double)bf16_bits_to_float(wu[j] & 0xFFFFu);
                ws[col + 2 * j + 1][row] = (double)bf16_bits_to_float(wu[j] >> 16);
            }
        }
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < RT_K; ++kk) {
            double xv[4], wv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) xv[i] = xs[kk][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) wv[j] = ws[kk][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(xv[i], wv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t_base + ty + 16 * i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e_base + tx + 16 * j;
            if (e >= E) continue;
            float l = (float)acc[i][j];
            if (bias) l = l + bias[e];
            if (debug && !isfinite(l)) atomicOr(err_word, DEV_ERR_NONFINITE);
            logits[(size_t)t * E + e] = l;
        }
    }
}

// One warp per token: k rounds of a warp arg-max over (logit desc, index asc),
// then softmax over the selected logits (max-subtracted, fp32).
constexpr int kMaxEPerLane = 8;   // E <= 256

// Order-preserving key of a finite fp32 logit: a larger logit has a larger key, and -0
// counts as +0 (equal logits tie). No finite logit maps to key 0.
__device__ __forceinline__ uint32_t logit_key(float v) {
    uint32_t b = __float_as_uint(v);
    if ((b << 1) == 0u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One warp selects a token's top k experts: k rounds, each a lane-local best (largest key,
// lowest expert on ties) followed by a warp-wide max of the keys and a min of the expert ids
// that hold it (two redux.sync), so ties go to the lower expert index. With m shared slots the
// row continues with slots k..k+m-1 = experts E..E+m-1 at weight 1 (the shared expert).
__device__ __forceinline__ void topk_warp(const float *row, int E, int k, int32_t *ids_row, float *w_row,
                                          int32_t *ids_copy = nullptr, int m = 0)
{
    const int lane = threadIdx.x & 31;
    float v[kMaxEPerLane];
    uint32_t key[kMaxEPerLane];
    uint32_t taken = 0;                       // bit i: candidate lane + 32 i used or absent
#pragma unroll
    for (int i = 0; i < kMaxEPerLane; ++i) {
        const int e = lane + 32 * i;
        v[i] = (e < E) ? __ldcg(row + e) : 0.f;
        key[i] = logit_key(v[i]);
        if (e >= E) taken |= 1u << i;
    }
    float sel_first = 0.f, my_sel = 0.f;
    int my_id = -1;
    for (int s = 0; s < k; ++s) {
        uint32_t bk = 0u;
        float bv = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxEPerLane; ++i) {
            if (!(taken & (1u << i)) && key[i] > bk) {   // strict: the lower i (lower expert) keeps ties
                bk = key[i];
                bv = v[i];
            }
        }
        const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
        uint32_t mine = 0xffffffffu;
#pragma unroll
        for (int i = kMaxEPerLane - 1; i >= 0; --i)
            if (!(taken & (1u << i)) && key[i] == mk) mine = (uint32_t)(lane + 32 * i);
        const uint32_t win = __reduce_min_sync(0xffffffffu, mine);
        const float wv = __shfl_sync(0xffffffffu, bv, (int)(win & 31u));
        if ((int)(win & 31u) == lane) taken |= 1u << (win >> 5);
        if (s == 0) sel_first = wv;
        if (lane == s) { my_sel = wv; my_id = (int)win; }
    }
    const float ex = (lane < k) ? expf(my_sel - sel_first) : 0.f;
    float den = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane < k) {
        ids_row[lane] = my_id;
        w_row[lane] = ex / den;
        if (ids_copy) ids_copy[lane] = my_id;
    } else if (lane < k + m) {
        ids_row[lane] = E + lane - k;
        w_row[lane] = 1.f;
        if (ids_copy) ids_copy[lane] = E + lane - k;
    }
}

// x [T][H] -> xq (f16 times a power of two per 16 elements) and xq_inv, for the
// GEMV regime; blocks spread over all threads of the grid.
__device__ __forceinline__ void convert_x_blocks(const uint16_t *__restrict__ x, int T, int H, uint16_t *xq,
                                                 float *xq_inv) {
    const int per_row = H / 16, n = T * per_row;
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < n; b += gridDim.x * blockDim.x) {
        const size_t off = (size_t)(b / per_row) * H + (size_t)(b % per_row) * 16;
        xq_inv[b] = block16_bf16_to_f16(x + off, xq + off);
    }
}

// One warp per token of full logits: top k and softmax weights (the allocation-free routing).
__global__ void __launch_bounds__(256) topk_kernel(const float *__restrict__ logits, int32_t *__restrict__ ids,
                                                   float *__restrict__ wts, int T, int E, int k)
{
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t < T) topk_warp(logits + (size_t)t * E, E, k, ids + (size_t)t * k, wts + (size_t)t * k);
}

// The expert plan, computed by one CTA of W warps. Pairs p = t*k + s are split
// into W contiguous segments, one per warp. Pass 1 counts per (segment,
// expert); a scan turns the counts into per-expert offsets and per-segment
// bases; pass 2 places each pair at base + its rank among same-expert pairs of
// the segment, so rows are ordered by (expert, pair index): a stable counting
// sort. Then every routed expert gets its regime and joins its regime's list.
struct PlanArgs {
    int E, gemv_max_tokens, mma_tile;
    uint32_t flags;
    int32_t *counts, *offsets, *perm, *inv, *regime, *gemv_list, *mma_list, *list_sizes, *err_word;
    int32_t *mma_entries;   // [max][4]: expert, first permuted row, rows (<= mma_tile), 0
    int debug;
};

__host__ __device__ constexpr size_t plan_smem_ints(int warps, int E) { return (size_t)warps * E + 2 * E + 1; }

// Exclusive scan of tot[0..E) into off[0..E] by one warp (E <= 256: 8 experts per lane).
__device__ __forceinline__ void scan_experts_warp(const int32_t *tot, int32_t *off, int E) {
    const int lane = threadIdx.x & 31;
    int local[8], s = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane * 8 + i;
        local[i] = (e < E) ? tot[e] : 0;
        s += local[i];
    }
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int run = incl - s;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane * 8 + i;
        if (e < E) off[e] = run;
        run += local[i];
    }
    if (lane == 31) off[E] = incl;
}

// Regime of every expert, the per-regime expert lists and the tensor-core token tiles,
// from the per-expert totals and offsets; run by one warp.
__device__ void plan_tail_warp(const int32_t *tot, const int32_t *off, const PlanArgs &pa)
{
    const int E = pa.E, lane = threadIdx.x & 31;
    int n_gemv = 0, n_mma = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        const int m = (e < E) ? tot[e] : 0;
        int reg = 0;
        if (m > 0) {
            if (pa.flags & TFMOE_FLAG_FORCE_GEMV) reg = 1;
            else if (pa.flags & TFMOE_FLAG_FORCE_MMA) reg = 2;
            else reg = (m <= pa.gemv_max_tokens) ? 1 : 2;
        }
        if (e < E) { pa.regime[e] = reg; pa.counts[e] = m; }
        const uint32_t bg = __ballot_sync(0xffffffffu, reg == 1);
        const uint32_t bm = __ballot_sync(0xffffffffu, reg == 2);
        const uint32_t lt = (1u << lane) - 1u;
        if (reg == 1) pa.gemv_list[n_gemv + __popc(bg & lt)] = e;
        if (reg == 2) pa.mma_list[n_mma + __popc(bm & lt)] = e;
        n_gemv += __popc(bg);
        n_mma += __popc(bm);
    }
    if (lane == 0) { pa.list_sizes[0] = n_gemv; pa.list_sizes[1] = n_mma; }
    // token tiles of the MMA-regime experts: ceil(m_e / pa.mma_tile) entries per
    // expert, in expert order; lane l handles experts 8l .. 8l+7
    int ntl[8], mine = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane * 8 + i;
        int n = 0;
        if (e < E) {
            const int m = tot[e];
            const bool mma = m > 0 && !(pa.flags & TFMOE_FLAG_FORCE_GEMV) &&
                             ((pa.flags & TFMOE_FLAG_FORCE_MMA) || m > pa.gemv_max_tokens);
            n = mma ? (m + pa.mma_tile - 1) / pa.mma_tile : 0;
        }
        ntl[i] = n;
        mine += n;
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int idx = incl - mine;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane * 8 + i;
        for (int j = 0; j < ntl[i]; ++j, ++idx) {
            int32_t *ent = pa.mma_entries + 4 * (size_t)idx;
            ent[0] = e;
            ent[1] = off[e] + j * pa.mma_tile;
            ent[2] = min(pa.mma_tile, tot[e] - j * pa.mma_tile);
            ent[3] = 0;
        }
    }
    if (lane == 31) pa.list_sizes[2] = incl;
}

// ids: the pairs' expert ids, written by an earlier kernel (global) or by this CTA (shared).
__device__ void plan_block(const int32_t *__restrict__ ids, int P, const PlanArgs &pa, int32_t *sm)
{
    const int E = pa.E;
    const int W = blockDim.x >> 5;
    int32_t *cnt = sm;               // [W][E]
    int32_t *tot = sm + W * E;       // [E]
    int32_t *off = tot + E;          // [E+1]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (P <= (int)blockDim.x && P <= W * E) {
        // small batches: one thread per pair. Warp w holds pairs 32w .. 32w+31; its lanes
        // with the same expert find each other with match_any, the first of them records
        // the warp's count of that expert, and a pair's stable rank is its rank inside the
        // warp plus the counts of the earlier warps.
        for (int i = threadIdx.x; i < W * E; i += blockDim.x) cnt[i] = 0;
        for (int e = threadIdx.x; e < E; e += blockDim.x) tot[e] = 0;
        __syncthreads();
        const int p = threadIdx.x;
        int e = -1;
        if (p < P) {
            e = ids[p];
            if (e >= E || e < 0) {
                if (pa.debug) atomicOr(pa.err_word, DEV_ERR_BAD_EXPERT);
                e = -1;
            }
        }
        const uint32_t same = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(same) - 1) {
            cnt[warp * E + e] = __popc(same);
            atomicAdd(&tot[e], __popc(same));
        }
        __syncthreads();
        if (warp == 0) scan_experts_warp(tot, off, E);
        __syncthreads();
        for (int i = threadIdx.x; i <= E; i += blockDim.x) pa.offsets[i] = off[i];
        if (e >= 0) {
            int rank = __popc(same & ((1u << lane) - 1u));
            for (int w = 0; w < warp; ++w) rank += cnt[w * E + e];
            const int r = off[e] + rank;
            pa.perm[r] = p;
            pa.inv[p] = r;
        }
    } else {
        // P contiguous pairs split into W warp segments: count per (segment, expert), scan,
        // then place each pair at its segment's base + its rank among same-expert pairs
        for (int i = threadIdx.x; i < W * E; i += blockDim.x) cnt[i] = 0;
        __syncthreads();
        const int seg = (P + W - 1) / W;
        const int p_begin = min(P, warp * seg), p_end = min(P, p_begin + seg);
        int32_t *my_cnt = cnt + warp * E;
        for (int p0 = p_begin; p0 < p_end; p0 += 32) {
            const int p = p0 + lane;
            int e = (p < p_end) ? ids[p] : -1;
            if (e >= E || (e < 0 && p < p_end)) {
                if (pa.debug) atomicOr(pa.err_word, DEV_ERR_BAD_EXPERT);
                e = -1;
            }
            const uint32_t m = __match_any_sync(0xffffffffu, e);
            if (e >= 0 && lane == __ffs(m) - 1) my_cnt[e] += __popc(m);
            __syncwarp();
        }
        __syncthreads();
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            int run = 0;
            for (int w = 0; w < W; ++w) {
                const int c = cnt[w * E + e];
                cnt[w * E + e] = run;
                run += c;
            }
            tot[e] = run;
        }
        __syncthreads();
        if (warp == 0) scan_experts_warp(tot, off, E);
        __syncthreads();
        for (int i = threadIdx.x; i < W * E; i += blockDim.x) cnt[i] += off[i % E];
        for (int e = threadIdx.x; e <= E; e += blockDim.x) pa.offsets[e] = off[e];
        __syncthreads();
        for (int p0 = p_begin; p0 < p_end; p0 += 32) {
            const int p = p0 + lane;
            int e = (p < p_end) ? ids[p] : -1;
            if (e >= E) e = -1;
            const uint32_t m = __match_any_sync(0xffffffffu, e);
            if (e >= 0) {
                const int rank = __popc(m & ((1u << lane) - 1u));
                const int r = my_cnt[e] + rank;
                pa.perm[r] = p;
                pa.inv[p] = r;
            }
            __syncwarp();
            if (e >= 0 && lane == __ffs(m) - 1) my_cnt[e] += __popc(m);
            __syncwarp();
        }
    }
    if (warp == 0) plan_tail_warp(tot, off, pa);
}

__global__ void __launch_bounds__(1024) permute_kernel(const int32_t *__restrict__ ids, int P, PlanArgs pa)
{
    extern __shared__ int32_t sm[];
    plan_block(ids, P, pa, sm);
}

// Multi-CTA plan, step 1 (large batches): CTA e scans expert e's counts over the segments
// (exclusive prefix = the segment's first rank among the expert's rows) and stores the
// total; the last CTA to arrive turns the totals into offsets and runs the plan's tail.
__global__ void __launch_bounds__(256) plan_scan_kernel(const int32_t *__restrict__ seg_cnt, int nseg,
                                                        int32_t *seg_base, int32_t *tot_g, int32_t *counter,
                                                        PlanArgs pa)
{
    __shared__ int32_t wsum[8];
    __shared__ int32_t tot[256], off[257];
    __shared__ int is_last;
    const int E = pa.E, e = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int carry = 0;
    for (int s0 = 0; s0 < nseg; s0 += blockDim.x) {
        const int sidx = s0 + threadIdx.x;
        const int v = (sidx < nseg) ? seg_cnt[(size_t)sidx * E + e] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int before = 0, all = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            if (w < warp) before += wsum[w];
            all += wsum[w];
        }
        if (sidx < nseg) seg_base[(size_t)sidx * E + e] = carry + before + incl - v;
        carry += all;
        __syncthreads();
    }
    if (threadIdx.x == 0) tot_g[e] = carry;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = (atomicAdd(counter, 1) == (int)gridDim.x - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    for (int i = threadIdx.x; i < E; i += blockDim.x) tot[i] = __ldcg(tot_g + i);
    __syncthreads();
    if (warp == 0) scan_experts_warp(tot, off, E);
    __syncthreads();
    for (int i = threadIdx.x; i <= E; i += blockDim.x) pa.offsets[i] = off[i];
    if (warp == 0) plan_tail_warp(tot, off, pa);
    if (threadIdx.x == 0) *counter = 0;
}

// Multi-CTA plan, step 2: CTA s places the pairs of segment s at the expert's offset plus
// the segment's base plus the pair's rank among the segment's same-expert pairs, which
// keeps the rows ordered by (expert, pair index).
__global__ void __launch_bounds__(256) plan_place_kernel(const int32_t *__restrict__ ids, int P, int k,
                                                         const int32_t *__restrict__ seg_base,
                                                         const int32_t *__restrict__ offsets, int E,
                                                         int32_t *__restrict__ perm, int32_t *__restrict__ inv)
{
    __shared__ int32_t ids_s[kPlanSegTokens * 32];
    const int p0 = blockIdx.x * kPlanSegTokens * k;
    const int n = min(kPlanSegTokens * k, P - p0);
    for (int i = threadIdx.x; i < n; i += blockDim.x) ids_s[i] = ids[p0 + i];
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int e = ids_s[i];
        if (e < 0 || e >= E) continue;
        int rank = 0;
        for (int q = 0; q < i; ++q) rank += (ids_s[q] == e);
        const int r = offsets[e] + seg_base[(size_t)blockIdx.x * E + e] + rank;
        perm[r] = p0 + i;
        inv[p0 + i] = r;
    }
}

// Decode-sized batches (T <= 16): router, top-k and plan in one launch.
// CTA e computes the logits of expert e for every token (its 8 warps split
// the hidden dimension, partial sums are added in a fixed order), then the
// last CTA to finish -- found with an atomic counter, which it resets --
// takes the top-k of every token and builds the plan. The wide grid keeps
// the expert dot products parallel; folding top-k into the last-arriving
// block is the launch-saving shape proposed in TensorFold issue #627 (comment
// on the fused tf_nemo_route_row experiment).
constexpr int kFusedMaxT = 16;
constexpr int kFusedThreads = 256;
__global__ void __launch_bounds__(kFusedThreads) route_fused_kernel(
    const uint16_t *__restrict__ x, const uint16_t *__restrict__ wr, const float *__restrict__ bias,
    float *__restrict__ logits, int32_t *__restrict__ ids, float *__restrict__ wts, int T, int H, int k,
    PlanArgs pa, int32_t *counter, uint16_t *xq, float *xq_inv, int m)
{
    extern __shared__ int32_t sm[];
    __shared__ int is_last;
    // one CTA per routed expert; the plan (pa.E) also covers the m shared slots
    const int E = (int)gridDim.x, e = blockIdx.x, kx = k + m;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // logits of expert e: warp w takes tokens w, w + 8 (T <= 16); lane l covers 8 columns per
    // 256-column step, and the warp adds its lanes in a fixed shuffle order
    const uint16_t *wrow = wr + (size_t)e * H;
    for (int t = warp; t < T; t += kFusedThreads / 32) {
        const uint16_t *xrow = x + (size_t)t * H;
        double acc = 0.0;
        for (int c0 = lane * 8; c0 < H; c0 += 256 * 8) {
            uint4 wv[8], xv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int c = c0 + u * 256;
                wv[u] = (c < H) ? *reinterpret_cast<const uint4 *>(wrow + c) : make_uint4(0, 0, 0, 0);
                xv[u] = (c < H) ? *reinterpret_cast<const uint4 *>(xrow + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint32_t wu[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
                const uint32_t xu[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc = fma((double)bf16_bits_to_float(xu[i] & 0xFFFFu), (double)bf16_bits_to_float(wu[i] & 0xFFFFu), acc);
                    acc = fma((double)bf16_bits_to_float(xu[i] >> 16), (double)bf16_bits_to_float(wu[i] >> 16), acc);
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) {
            float l = (float)acc;
            if (bias) l = l + bias[e];
            if (pa.debug && !isfinite(l)) atomicOr(pa.err_word, DEV_ERR_NONFINITE);
            logits[(size_t)t * E + e] = l;
        }
    }
    if (xq) convert_x_blocks(x, T, H, xq, xq_inv);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = (atomicAdd(counter, 1) == (int)gridDim.x - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    // the ids stay in shared memory for the plan: no global round trip on the serial tail
    __shared__ int32_t ids_sm[kFusedMaxT * 32];
    for (int t = warp; t < T; t += kFusedThreads / 32)
        topk_warp(logits + (size_t)t * E, E, k, ids + (size_t)t * kx, wts + (size_t)t * kx, ids_sm + t * kx, m);
    __syncthreads();
    plan_block(ids_sm, T * kx, pa, sm);
    if (threadIdx.x == 0) *counter = 0;
}

}  // namespace

static PlanArgs plan_args(const Layer &L, int T) {
    PlanArgs pa{};
    pa.E = expert_slots(L);
    pa.gemv_max_tokens = gemv_threshold(L, T);
    pa.mma_tile = L.mma_small ? kMmaSmallTileTokens : kMmaTileTokens;
    pa.flags = L.desc.flags;
    pa.counts = L.ws.counts; pa.offsets = L.ws.offsets; pa.perm = L.ws.perm; pa.inv = L.ws.inv;
    pa.regime = L.ws.regime; pa.gemv_list = L.ws.gemv_list; pa.mma_list = L.ws.mma_list;
    pa.list_sizes = L.ws.list_sizes; pa.err_word = L.ws.err_word;
    pa.mma_entries = L.ws.mma_entries;
    pa.debug = (L.desc.flags & TFMOE_FLAG_DEBUG_CHECKS) ? 1 : 0;
    return pa;
}

bool route_fused_applies(const Layer &, int T) { return T <= kFusedMaxT; }

static bool large_plan(const Layer &L, int T) {
    return T > kFusedMaxT && (long long)T * token_slots(L) > kLargePlanPairs;
}

cudaError_t launch_router(Layer &L, const uint16_t *x, int T, cudaStream_t s, int *launches)
{
    const int H = L.desc.hidden, E = L.desc.num_experts, k = L.desc.top_k;
    const float *bias = L.desc.has_router_bias ? L.w.router_bias : nullptr;
    const bool gemv = !(L.desc.flags & TFMOE_FLAG_FORCE_MMA);   // the GEMV regime may run: write its x operand
    if (route_fused_applies(L, T)) {
        // router, top-k and plan in one launch (the permute launcher then does nothing)
        StageTimer timer(L, TFMOE_STAGE_ROUTER, s);
        const size_t smem = sizeof(int32_t) * plan_smem_ints(kFusedThreads / 32, expert_slots(L));
        route_fused_kernel<<<E, kFusedThreads, smem, s>>>(x, L.w.router_w, bias, L.ws.logits, L.ws.ids,
                                                          L.ws.topk_w, T, H, k, plan_args(L, T), L.ws.route_counter,
                                                          gemv ? L.ws.xq : nullptr, L.ws.xq_inv, shared_slots(L));
        *launches += 1;
        return cudaGetLastError();
    }
    // larger batches: tensor-core approximate logits, exact candidates, exact top k
    return launch_router_tc(L, x, T, gemv, large_plan(L, T) ? L.ws.seg_cnt : nullptr, s, launches);
}

cudaError_t launch_permute(Layer &L, int T, cudaStream_t s, int *launches)
{
    if (route_fused_applies(L, T)) return cudaSuccess;
    StageTimer timer(L, TFMOE_STAGE_PERMUTE, s);
    const int E = expert_slots(L), kx = token_slots(L), P = T * kx;
    if (large_plan(L, T)) {
        const int nseg = (T + kPlanSegTokens - 1) / kPlanSegTokens;
        plan_scan_kernel<<<E, 256, 0, s>>>(L.ws.seg_cnt, nseg, L.ws.seg_base, L.ws.plan_tot, L.ws.plan_counter,
                                           plan_args(L, T));
        plan_place_kernel<<<nseg, 256, 0, s>>>(L.ws.ids, P, kx, L.ws.seg_base, L.ws.offsets, E, L.ws.perm,
                                               L.ws.inv);
        *launches += 2;
        return cudaGetLastError();
    }
    const size_t smem = sizeof(int32_t) * plan_smem_ints(32, E);
    permute_kernel<<<1, 1024, smem, s>>>(L.ws.ids, P, plan_args(L, T));
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace tfmoe

// ---------------------------------------------------------------------------
// Allocation-free routing for callers that cannot allocate device memory
// (tfmoe_route_noalloc in tfmoe.h). The router logits go to a fixed array
// compiled into the library instead of a workspace: every GPU that loads the
// library holds TFMOE_ROUTE_NOALLOC_MAX_LOGITS floats of it until exit, and all
// calls on a device share it, so calls that overlap on the GPU race.
namespace tfmoe {
namespace {

static __device__ __align__(256) float g_noalloc_logits[TFMOE_ROUTE_NOALLOC_MAX_LOGITS];

// Host code cannot use g_noalloc_logits as a device address: the symbol is a host-side
// stand-in, and the array's device address belongs to one CUDA context (a device reset
// reloads the module and may move it; another context on the same device has its own
// copy). So every call made outside a stream capture looks the address up again with
// cudaGetSymbolAddress and records it under the current context's unique id; a call
// made during a capture (where that lookup is not allowed) uses the address recorded
// for the current context, and fails if there is none.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);
constexpr int kNoAllocSlots = 64;
std::mutex g_noalloc_mutex;
unsigned long long g_noalloc_ctx[kNoAllocSlots] = {};   // 0 = empty slot
float *g_noalloc_ptr[kNoAllocSlots] = {};
int g_noalloc_next = 0;

template <class Fn>
Fn driver_fn(const char *name) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(p);
}

// Unique id of the context current on this thread (0 if it cannot be found).
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id + 1;   // never 0
}

cudaError_t noalloc_scratch(cudaStream_t s, float **out) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
        cudaGetLastError();                       // e.g. the legacy stream while another captures
        cs = cudaStreamCaptureStatusActive;
    }
    if (cs == cudaStreamCaptureStatusNone) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_logits);   // also creates the context
        if (e != cudaSuccess) return e;
        const unsigned long long id = current_context_id();
        if (id) {
            int slot = -1;
            for (int i = 0; i < kNoAllocSlots; ++i)
                if (g_noalloc_ctx[i] == id) slot = i;
            if (slot < 0) {
                slot = g_noalloc_next;
                g_noalloc_next = (g_noalloc_next + 1) % kNoAllocSlots;
            }
            g_noalloc_ctx[slot] = id;
            g_noalloc_ptr[slot] = static_cast<float *>(p);
        }
        *out = static_cast<float *>(p);
        return cudaSuccess;
    }
    const unsigned long long id = current_context_id();
    for (int i = 0; id && i < kNoAllocSlots; ++i)
        if (g_noalloc_ctx[i] == id) {
            *out = g_noalloc_ptr[i];
            return cudaSuccess;
        }
    return cudaErrorStreamCaptureUnsupported;
}

}  // namespace
}  // namespace tfmoe

extern "C" tfmoe_status tfmoe_route_noalloc(const uint16_t *x, int32_t T, int32_t hidden,
                                            const uint16_t *router_w, const float *router_bias,
                                            int32_t num_experts, int32_t top_k,
                                            int32_t *ids_out, float *weights_out, void *cuda_stream)
{
    using namespace tfmoe;
    const int H = hidden, E = num_experts, k = top_k;
    if (T < 0) return record_error(TFMOE_ERR_INVALID_ARG, "tfmoe_route_noalloc: T=%d is negative", T);
    if (H <= 0 || H % 16)
        return record_error(TFMOE_ERR_INVALID_ARG, "tfmoe_route_noalloc: hidden=%d must be a positive multiple of 16", H);
    if (E <= 0 || k <= 0 || k > E)
        return record_error(TFMOE_ERR_INVALID_ARG, "tfmoe_route_noalloc: need 1 <= top_k (%d) <= num_experts (%d)", k, E);
    if (H % 32 || E > 256 || k > 32)
        return record_error(TFMOE_ERR_UNSUPPORTED,
                            "tfmoe_route_noalloc: needs hidden %% 32 == 0, num_experts <= 256, top_k <= 32");
    if ((long long)T * E > (long long)TFMOE_ROUTE_NOALLOC_MAX_LOGITS)
        return record_error(TFMOE_ERR_INVALID_ARG,
                            "tfmoe_route_noalloc: T * num_experts = %lld exceeds the fixed scratch of %d logits; "
                            "route the batch in parts of at most %d tokens",
                            (long long)T * E, TFMOE_ROUTE_NOALLOC_MAX_LOGITS, TFMOE_ROUTE_NOALLOC_MAX_LOGITS / E);
    if (T == 0) return record_ok();
    if (!x || !router_w || !ids_out || !weights_out)
        return record_error(TFMOE_ERR_INVALID_ARG, "tfmoe_route_noalloc: NULL buffer");
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(router_w)) & 15u)
        return record_error(TFMOE_ERR_INVALID_ARG, "tfmoe_route_noalloc: x and router_w must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    float *logits = nullptr;
    cudaError_t e = noalloc_scratch(s, &logits);
    if (e == cudaErrorStreamCaptureUnsupported)
        return record_error(TFMOE_ERR_CUDA, "tfmoe_route_noalloc: first call in this context made during a stream "
                            "capture; make one call outside capture first");
    if (e != cudaSuccess)
        return record_error(TFMOE_ERR_CUDA, "tfmoe_route_noalloc: scratch address: %s", cudaGetErrorString(e));
    if (T <= 2 * kSmallTokens) {
        const int warps = E * ((T + kSmallTokens - 1) / kSmallTokens);
        router_small_kernel<<<(warps + 3) / 4, 128, 0, s>>>(x, router_w, router_bias, logits, T, H, E, nullptr, 0);
    } else {
        dim3 grid((T + RT_T - 1) / RT_T, (E + RT_E - 1) / RT_E);
        router_tiled_kernel<<<grid, 256, 0, s>>>(x, router_w, router_bias, logits, T, H, E, nullptr, 0);
    }
    topk_kernel<<<(T + 7) / 8, 256, 0, s>>>(logits, ids_out, weights_out, T, E, k);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return record_error(TFMOE_ERR_CUDA, "tfmoe_route_noalloc: launch: %s", cudaGetErrorString(e));
    return record_ok();
}

