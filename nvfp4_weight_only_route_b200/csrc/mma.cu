// mma.cu -- the prefill regime of the NVFP4 grouped expert projections:
// dequantise into the tensor core's operand memory and run tcgen05 MMAs.
//
// Prefill pushes all prompt tokens through the active experts as one large
// matrix multiply, so it is limited by tensor throughput rather than memory
// (DGX Spark GB10 bandwidth-budget page, section "Mechanism: decode is
// bandwidth-bound, prefill is compute-bound"). The weights stay W4A16: they are
// decoded to 16-bit floats and multiplied against the 16-bit activations
// (TensorFold 1.0.12 GLM-5.3-Flash post, section "NVFP4 is neither uniform
// 4-bit nor all-FP4 compute"). The decode is exact: an E2M1 value times an E4M3
// scale has at most 6 significant bits and lies in [2^-10, 2688], so it is an
// f16 and a bf16 value; the per-tensor fp32 scale multiplies the accumulator.
//
//   gate/up: f16 x f16 -> fp32. The activation rows are stored as f16 times an
//            exact per-row power of two (every bf16 element within 2^28 of the
//            row's largest is then an exact f16), undone in the epilogue.
//            E2M1 -> f16 is one conversion, the scale one f16x2 multiply.
//   down   : bf16 x bf16 -> fp32; the SwiGLU output a is a bf16 tensor already.
//
// Tile: 128 weight rows (MMA M) x N <= 256 token rows of one expert (MMA N, the
// tile's tokens rounded up to 16), the reduction in stages of 64. One persistent CTA
// per SM (big shape), 24 warps:
//   warp 0       producer of the token tiles (TMA, 128-byte swizzle, box 64 x rows)
//                into a 4-stage ring that the MMA commit frees
//   warp 2       producer of the 4 KB code tiles + their 512 B scale slabs (bulk copies)
//                into a 12-stage ring that the decoders free once they have read it
//   warp 1       allocates tensor memory; lane 0 issues the MMAs and commits: one wait
//                and one commit per stage, four MMAs of K = 16 in between
//   warps 4-15   three dequant warpgroups taking every third stage (all 64 columns):
//                thread q of a warpgroup owns weight row q = tensor-memory lane q
//   warps 16-23  epilogue, two warpgroups taking alternate 16-column steps of the
//                accumulator: SwiGLU for interleaved gate/up rows (row 2j gate j,
//                2j+1 up j) staged through shared memory into 16-byte row pieces,
//                fp32 store for down; the accumulator is handed back once read
// Tensor memory: the accumulator at columns [0,256), four A stages of 32 columns
// from 256. The small shape (two CTAs per SM, N <= 64) double-buffers its
// accumulator instead. Every wait is bounded; on a timeout the CTA records
// the error and stops issuing work; before it exits its issued copies land and
// its issued MMAs complete (a final commit), and only then is tensor memory freed.
#include <cuda.h>

#include <new>

#include "common.cuh"
#include "internal.h"

namespace tfmoe {
namespace {

constexpr int kM = 128;
constexpr int kEpiCols = 16;               // accumulator columns per epilogue step

// Kernel shapes. Big: one CTA per SM, token tiles of up to 256 rows (prefill): an
// expert's few hundred tokens take one tile, so its weights are decoded once, and the
// MMAs are as wide as the instruction allows. The accumulator is single-buffered (256
// columns; the other 256 hold the decoded weight stages): the epilogue drains it
// before the next tile's first MMA. Small: two CTAs per SM, token tiles of up to 64
// rows (batched decode, tens of tokens per expert), double-buffered accumulators.
// MMAs issued from different CTAs of an SM overlap on the tensor core, so at small N
// two issuing CTAs per SM nearly double the weight rate.
//   warps 0, 2: token-tile and code producers; warp 1: TMEM owner and MMA issuer;
//   warps kDqWarp0..: DqGroups dequant warpgroups; then EpiGroups epilogue warpgroups.
template <int MaxN, int NumBoxes, int Stages, int CStages, int DqGroups, int EpiGroups, int CtasPerSm, int DBufs>
struct MmaCfg {
    static constexpr int kMaxN = MaxN, kNumBoxes = NumBoxes, kStages = Stages, kCStages = CStages;
    static constexpr int kDqGroups = DqGroups, kEpiGroups = EpiGroups, kCtasPerSm = CtasPerSm, kDBufs = DBufs;
    static constexpr int kDqWarp0 = 4, kEpiWarp0 = 4 + 4 * DqGroups;
    static constexpr int kThreads = 32 * (kEpiWarp0 + 4 * EpiGroups);
    static constexpr uint32_t kACol = DBufs * MaxN;  // accumulators at [b N, (b+1) N); A stages after them
    static constexpr uint32_t kTmemCols =
        (kACol + Stages * 32 <= 128) ? 128u : (kACol + Stages * 32 <= 256) ? 256u : 512u;
    static constexpr int kBStageBytes = MaxN * 128;  // N rows x 64 16-bit elements
    static_assert(kACol + Stages * 32 <= kTmemCols && kTmemCols * CtasPerSm <= 512, "tensor memory budget");
    static_assert(kBStageBytes % 1024 == 0, "token stages must stay 1 KB aligned");
};
using BigCfg = MmaCfg<kMmaTileTokens, 5, 4, 12, 3, 2, 1, 1>;       // 768 threads, 512 TMEM columns
using SmallCfg = MmaCfg<kMmaSmallTileTokens, 3, 4, 12, 2, 1, 2, 2>; // 512 threads, 256 TMEM columns

template <class C>
struct MmaSmem {
    uint8_t b[C::kStages][C::kBStageBytes];   // 1024-byte aligned
    uint8_t codes[C::kCStages][kTileCodeBytes];
    uint8_t scales[C::kCStages][kTileScaleBytes];
    uint16_t stage_out[4 * C::kEpiGroups][kEpiCols][16];   // per epilogue warp: 16 tokens x 16 outputs
    float xi_s[4 * C::kEpiGroups][C::kMaxN];              // per epilogue warp: the tile's token scales
    uint64_t full[C::kStages], empty[C::kStages], aready[C::kStages];
    uint64_t cfull[C::kCStages], cempty[C::kCStages];
    uint64_t dfull[C::kDBufs], dempty[C::kDBufs];
    uint64_t mma_done;                        // the issuer's last commit: every MMA of the CTA complete
    uint32_t tmem_base;
    int32_t abort_flag;
};

template <class C>
struct TokenMaps {
    CUtensorMap box[C::kNumBoxes];         // same tensor, box heights 16 << i, the last kMaxN
};

enum class Proj { GateUp, Down };

struct MmaArgs {
    const uint8_t *codes, *scales;
    const float *glob0, *glob1;
    int R, K;                              // projection rows, reduction length
    const int32_t *entries;                // [n][4] expert, first permuted row, rows, 0
    const int32_t *list_sizes;             // [2] = number of entries
    uint16_t *act_out;                     // gate/up output [P][I]
    float *y_out;                          // down output [P][H]
    const float *row_inv_scale;            // gate/up: 2^-sh of each f16 activation row [P]
    int I;
    int32_t *err_word;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, int32_t *abort_flag, int32_t *err) {
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

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    // K-major, 128-byte swizzle: start>>4, leading offset 1 (unused), stride 1024 B
    // between 8-row groups, descriptor version 1, layout type 2 (SWIZZLE_128B).
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// kind::f16, A and B K-major of one 16-bit type (0 = f16, 1 = bf16), D = F32, M = 128, N given.
__device__ __forceinline__ uint32_t instr_desc_16bit(int n, uint32_t type) {
    return (1u << 4) | (type << 7) | (type << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kM >> 4) << 24);
}

__device__ __forceinline__ void mma_16bit_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u));
}

// True in one lane of a converged warp (the lowest active lane, so the same lane at
// every call while the warp stays converged).
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile("{\n\t.reg .b32 rx;\n\t.reg .pred px;\n\telect.sync rx|px, %1;\n\t@px mov.s32 %0, 1;\n\t}"
                 : "+r"(pred) : "r"(0xffffffffu));
    return pred != 0;
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Two decoded E2M1 values (f16x2) times the block scale (f16 pair, both halves equal) -> f16x2.
__device__ __forceinline__ uint32_t scale_pair_f16(uint32_t h, __half2 scale2) {
    const __half2 v = __hmul2(*reinterpret_cast<const __half2 *>(&h), scale2);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// Two decoded E2M1 values (f16x2) times the block scale -> bf16x2. Products are exact
// in f16 (<= 6 significant bits, magnitudes 2^-10 .. 2688) and in bf16.
__device__ __forceinline__ uint32_t scale_pair_bf16(uint32_t h, __half2 scale2) {
    const __half2 v = __hmul2(*reinterpret_cast<const __half2 *>(&h), scale2);
    const float2 f = __half22float2(v);
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<const uint32_t *>(&b);
}

// Token-tile heights: 16, 32, 64, 128, ..., then kMaxN.
template <class C>
__host__ __device__ __forceinline__ int box_rows(int i) { return i < C::kNumBoxes - 1 ? (16 << i) : C::kMaxN; }
template <class C>
__device__ __forceinline__ int box_index(int rows) {
    int i = 0;
    while (box_rows<C>(i) < rows && i < C::kNumBoxes - 1) ++i;
    return i;
}
// MMA N of a token tile of `rows` tokens: the rows rounded up to 16 (the box loaded
// may be taller; its extra rows are not multiplied).
__device__ __forceinline__ int mma_n(int rows) { return (rows + 15) & ~15; }

template <class C, Proj P>
__global__ void __launch_bounds__(C::kThreads, C::kCtasPerSm) mma_kernel(const __grid_constant__ TokenMaps<C> maps,
                                                                         const MmaArgs a)
{
    constexpr int kMaxN = C::kMaxN, kStages = C::kStages, kCStages = C::kCStages;
    constexpr int kDqWarp0 = C::kDqWarp0, kEpiWarp0 = C::kEpiWarp0, kBStageBytes = C::kBStageBytes;
    constexpr uint32_t kTmemCols = C::kTmemCols, kACol = C::kACol;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    MmaSmem<C> &sm = *reinterpret_cast<MmaSmem<C> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = a.K / kTileK, RT = a.R / kM;
    const int n_tiles = __ldg(a.list_sizes + 2) * RT;
    if ((int)blockIdx.x >= n_tiles) return;
    constexpr uint32_t kType = (P == Proj::GateUp) ? 0u : 1u;   // f16 : bf16

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
            mbar_init(&sm.aready[s], 4);               // one arrival per decoder warp
        }
        for (int c = 0; c < kCStages; ++c) {
            mbar_init(&sm.cfull[c], 1);
            mbar_init(&sm.cempty[c], 4);
        }
        for (int b = 0; b < C::kDBufs; ++b) {
            mbar_init(&sm.dfull[b], 1);
            mbar_init(&sm.dempty[b], 4 * C::kEpiGroups);   // one arrival per epilogue warp
        }
        mbar_init(&sm.mma_done, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&sm.tmem_base)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0 || warp == 2) {
        // warp 0: token tiles into the 8-stage ring (freed by the MMA commit);
        // warp 2: code/scale tiles into the 16-stage ring (freed once decoded)
        if (lane == 0) {
            const bool tokens = (warp == 0);
            const int nst = tokens ? kStages : kCStages;
            uint32_t g = 0, issued = 0;
            for (int t = blockIdx.x; t < n_tiles && !sm.abort_flag; t += gridDim.x) {
                const int32_t *ent = a.entries + 4 * (t / RT);
                const int e = __ldg(ent), row0 = __ldg(ent + 1), rows = __ldg(ent + 2);
                const int rt = t % RT, bi = box_index<C>(rows);
                const uint32_t b_bytes = (uint32_t)box_rows<C>(bi) * 128u;
                const size_t rti = (size_t)e * RT + rt;
                for (int kt = 0; kt < KT; ++kt, ++g) {
                    const int s = g % nst;
                    const uint32_t ph = (g / nst) & 1u;
                    if (tokens) {
                        if (!wait_or_abort(&sm.empty[s], ph ^ 1u, &sm.abort_flag, a.err_word)) break;
                        mbar_arrive_expect_tx(&sm.full[s], b_bytes);
                        tma_load_2d(sm.b[s], &maps.box[bi], kt * kTileK, row0, &sm.full[s]);
                    } else {
                        if (!wait_or_abort(&sm.cempty[s], ph ^ 1u, &sm.abort_flag, a.err_word)) break;
                        mbar_arrive_expect_tx(&sm.cfull[s], kTileCodeBytes + kTileScaleBytes);
                        bulk_g2s(sm.codes[s], a.codes + (rti * KT + kt) * kTileCodeBytes, kTileCodeBytes, &sm.cfull[s]);
                        bulk_g2s(sm.scales[s], a.scales + scale_offset(rti, KT, kt), kTileScaleBytes, &sm.cfull[s]);
                    }
                    issued = g + 1;
                }
            }
            if (sm.abort_flag) {
                // aborted: let the copies already issued land before the CTA exits (bounded)
                for (uint32_t j = (issued > (uint32_t)nst ? issued - nst : 0); j < issued; ++j) {
                    uint64_t *bar = tokens ? &sm.full[j % nst] : &sm.cfull[j % nst];
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait_sleep(bar, (j / nst) & 1u) && global_timer_ns() - t0 < kWaitLimitNs / 4) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // The MMA issue is the kernel's critical path (each tcgen05.mma keeps the issuing
        // thread busy for tens of cycles). The whole warp runs the loop and waits, and one
        // elected lane (the same one throughout: the warp is converged at every election)
        // issues each stage's four MMAs and its commit, so a commit covers every MMA before
        // it. Per stage: one wait (the decoders also wait for the token tile), four MMAs with
        // descriptors advanced by adds, one commit; the stage slot and phase advance by
        // increments.
        const uint64_t bdesc0 = smem_desc_sw128(smem_u32(sm.b[0]));
        const uint32_t acol0 = tmem + kACol;
        int s = 0;
        uint32_t ph = 0, tile_i = 0;
        for (int t = blockIdx.x; t < n_tiles && !sm.abort_flag; t += gridDim.x, ++tile_i) {
            const int rows = __ldg(a.entries + 4 * (t / RT) + 2);
            const uint32_t idesc = instr_desc_16bit(mma_n(rows), kType);
            const int buf = (int)(tile_i % C::kDBufs);
            const uint32_t use = tile_i / C::kDBufs;
            if (!__all_sync(0xffffffffu, wait_or_abort(&sm.dempty[buf], (use & 1u) ^ 1u, &sm.abort_flag, a.err_word)))
                break;
            tc_fence_after();
            const uint32_t dt = tmem + (uint32_t)buf * kMaxN;
            bool ok = true;
            for (int kt = 0; kt < KT; ++kt) {
                if (!__all_sync(0xffffffffu, wait_or_abort(&sm.aready[s], ph, &sm.abort_flag, a.err_word))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one()) {
                    const uint64_t bd = bdesc0 + (uint64_t)(s * (kBStageBytes >> 4));
                    const uint32_t ad = acol0 + (uint32_t)s * 32u;
                    mma_16bit_ts(dt, ad, bd, idesc, kt != 0);
                    mma_16bit_ts(dt, ad + 8u, bd + 2u, idesc, 1u);
                    mma_16bit_ts(dt, ad + 16u, bd + 4u, idesc, 1u);
                    mma_16bit_ts(dt, ad + 24u, bd + 6u, idesc, 1u);
                    mma_commit(&sm.empty[s]);
                }
                __syncwarp();
                if (++s == kStages) { s = 0; ph ^= 1u; }
            }
            if (!ok) break;
            if (elect_one()) mma_commit(&sm.dfull[buf]);
            __syncwarp();
        }
        // on every path, including an abort: tensor memory and the operand stages stay
        // in use until the MMAs already issued complete, which this commit reports
        if (elect_one()) mma_commit(&sm.mma_done);
        __syncwarp();
    } else if (warp >= kDqWarp0 && warp < kEpiWarp0) {
        // decode: warpgroup gq takes the stages g with g % kDqGroups == gq (all 64 columns), so
        // stages are decoded concurrently; thread q owns weight row q = TMEM lane q
        const int gq = (warp - kDqWarp0) >> 2;
        const int q = (warp & 3) * 32 + lane;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        uint32_t g = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
            for (int kt = 0; kt < KT; ++kt, ++g) {
                if ((int)(g % C::kDqGroups) != gq) continue;
                const int s = g % kStages, cs = g % kCStages;
                const uint32_t ph = (g / kStages) & 1u, pc = (g / kCStages) & 1u;
                ok = wait_or_abort(&sm.cfull[cs], pc, &sm.abort_flag, a.err_word);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                const uint4 c0 = *reinterpret_cast<const uint4 *>(sm.codes[cs] + q * 16);
                const uint4 c1 = *reinterpret_cast<const uint4 *>(sm.codes[cs] + 2048 + q * 16);
                const uint32_t sc4 = *reinterpret_cast<const uint32_t *>(sm.scales[cs] + q * 4);
                __syncwarp();                                              // every lane has read its codes
                if (lane == 0) mbar_arrive(&sm.cempty[cs]);                // code stage consumed
                // decode the whole stage into registers first; then wait for the A stage to be
                // free and for the token tile (so that the MMA issuer needs one wait per stage)
                const uint32_t s01 = e4m3x2_to_f16x2(sc4 & 0xFFFFu), s23 = e4m3x2_to_f16x2(sc4 >> 16);
                const __half2 h01 = *reinterpret_cast<const __half2 *>(&s01);
                const __half2 h23 = *reinterpret_cast<const __half2 *>(&s23);
                const __half2 sb[4] = {__low2half2(h01), __high2half2(h01), __low2half2(h23), __high2half2(h23)};
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint32_t r[2][16];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {      // columns 0..31, then 32..63
#pragma unroll
                    for (int w4 = 0; w4 < 4; ++w4) {  // word holds elements 8*w4 .. 8*w4 + 7 of the half
                        uint32_t h4[4];
                        e2m1x8_to_f16x2x4(words[4 * hh + w4], h4);
                        const __half2 sc = sb[2 * hh + (w4 >> 1)];
#pragma unroll
                        for (int b = 0; b < 4; ++b)
                            r[hh][4 * w4 + b] = (kType == 0u) ? scale_pair_f16(h4[b], sc) : scale_pair_bf16(h4[b], sc);
                    }
                }
                ok = wait_or_abort(&sm.empty[s], ph ^ 1u, &sm.abort_flag, a.err_word);   // A stage free
                if (ok) ok = wait_or_abort(&sm.full[s], ph, &sm.abort_flag, a.err_word); // token tile landed
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tmem_st16(tmem + lane_base + kACol + (uint32_t)s * 32u, r[0]);
                tmem_st16(tmem + lane_base + kACol + (uint32_t)s * 32u + 16u, r[1]);
                tc_wait_st();
                tc_fence_before();
                __syncwarp();                        // the warp's stores precede its one arrival
                if (lane == 0) mbar_arrive(&sm.aready[s]);
            }
        }
    } else if (warp >= kEpiWarp0) {
        // epilogue warpgroups take alternate 16-column steps of the accumulator. Each warp
        // has the next step's tensor-memory load in flight while it processes the current
        // one, and stages the tile's per-token activation scales in shared memory once.
        const int eg = (warp - kEpiWarp0) >> 2;
        const int ew = warp - kEpiWarp0;                           // staging slot
        const int q = (warp & 3) * 32 + lane;                      // weight row = TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        uint32_t tile_i = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tile_i) {
            const int32_t *ent = a.entries + 4 * (t / RT);
            const int e = __ldg(ent), row0 = __ldg(ent + 1), rows = __ldg(ent + 2);
            const int rt = t % RT;
            const int n = mma_n(rows);
            const int buf = (int)(tile_i % C::kDBufs);
            const float gs = __ldg(a.glob0 + e);                               // gate (or down) scale
            const float gs_up = (P == Proj::GateUp) ? __ldg(a.glob1 + e) : 0.f;
            if (P == Proj::GateUp) {
                __syncwarp();
                for (int c = lane; c < n; c += 32)
                    sm.xi_s[ew][c] = (c < rows) ? __ldg(a.row_inv_scale + row0 + c) : 0.f;
                __syncwarp();
            }
            if (!__all_sync(0xffffffffu, wait_or_abort(&sm.dfull[buf], (tile_i / C::kDBufs) & 1u, &sm.abort_flag,
                                                       a.err_word)))
                break;                           // warp-uniform: the loads below are warp-collective
            tc_fence_after();
            const int grow = rt * kM + q;
            const uint32_t dcol = tmem + lane_base + (uint32_t)buf * kMaxN;
            // this group's steps: eg, eg + kEpiGroups, ...
            const int steps = n / kEpiCols;
            auto hand_back = [&]() {             // the warp's reads precede its one arrival
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.dempty[buf]);
            };
            auto process = [&](const uint32_t (&d)[16], int st) {
                const int c = st * kEpiCols;
                if (P == Proj::GateUp) {
                    // even lane 2i holds gate row j of the step's 16 tokens, lane 2i+1 the up row of
                    // the same j. The pair splits the work: the even lane takes tokens 0..7 of the
                    // step, the odd lane tokens 8..15, each receiving its partner's values of those
                    // tokens (one shuffle per token), so no lane idles through the SwiGLU. The a
                    // values [16 tokens][16 j] are staged in shared memory, then written as 16-byte
                    // row pieces.
                    const bool odd = (lane & 1) != 0;
                    const int half = odd ? 8 : 0;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float keep = __uint_as_float(odd ? d[i + 8] : d[i]);
                        const float give = __uint_as_float(odd ? d[i] : d[i + 8]);
                        const float got = __shfl_xor_sync(0xffffffffu, give, 1);
                        const float xi = sm.xi_s[ew][c + half + i];            // an exact power of two
                        const float gv = (odd ? got : keep) * (gs * xi);
                        const float uv = (odd ? keep : got) * (gs_up * xi);
                        sm.stage_out[ew][half + i][lane >> 1] = float_to_bf16_bits_rn(silu_f32(gv) * uv);
                    }
                    __syncwarp();
                    // 16 tokens x 32 bytes: lane l writes token l/2, bytes 16*(l&1) .. +16
                    const int tok = c + (lane >> 1);
                    if (tok < rows) {
                        const uint4 v4 = *reinterpret_cast<const uint4 *>(&sm.stage_out[ew][lane >> 1][8 * (lane & 1)]);
                        const int j0 = (rt * kM + (warp & 3) * 32) / 2 + 8 * (lane & 1);
                        *reinterpret_cast<uint4 *>(a.act_out + (size_t)(row0 + tok) * a.I + j0) = v4;
                    }
                    __syncwarp();
                } else {
#pragma unroll
                    for (int i = 0; i < kEpiCols; ++i) {
                        const int tok = c + i;
                        if (tok < rows) a.y_out[(size_t)(row0 + tok) * a.R + grow] = __uint_as_float(d[i]) * gs;
                    }
                }
            };
            uint32_t d0[16], d1[16];
            int st = eg;
            if (st < steps) tmem_ld16(dcol + (uint32_t)(st * kEpiCols), d0);
            // two steps per iteration, alternating the register buffers: load step st+G while
            // processing step st. After the last load lands the accumulator is handed back.
            while (st < steps) {
                tc_wait_ld();
                int nst = st + C::kEpiGroups;
                if (nst < steps) tmem_ld16(dcol + (uint32_t)(nst * kEpiCols), d1);
                else hand_back();
                process(d0, st);
                st = nst;
                if (st >= steps) break;
                tc_wait_ld();
                nst = st + C::kEpiGroups;
                if (nst < steps) tmem_ld16(dcol + (uint32_t)(nst * kEpiCols), d0);
                else hand_back();
                process(d1, st);
                st = nst;
            }
            if (eg >= steps) hand_back();        // no step for this group in this tile
        }
    }
    __syncthreads();
    if (warp == 1) {
        if (lane == 0) mbar_wait_bounded(&sm.mma_done, 0, a.err_word);
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

// x_perm[r] = f16(x[token of pair perm[r]] * 2^sh_r) for the rows of every MMA token
// tile, sh_r the power of two that puts the row's largest magnitude just below
// 2^15 (exact for every element within 2^28 of the largest); row_inv[r] = 2^-sh_r.
__global__ void __launch_bounds__(256) gather_kernel(const uint16_t *__restrict__ x, const int32_t *__restrict__ perm,
                                                     const int32_t *__restrict__ entries,
                                                     const int32_t *__restrict__ list_sizes, int H, int k,
                                                     uint16_t *__restrict__ x_perm, float *__restrict__ row_inv)
{
    __shared__ uint32_t wmax[8];
    const int ent = blockIdx.x;
    if (ent >= __ldg(list_sizes + 2)) return;
    const int row0 = __ldg(entries + 4 * ent + 1), rows = __ldg(entries + 4 * ent + 2);
    const int chunks = H / 8;
    for (int rr = blockIdx.y; rr < rows; rr += gridDim.y) {
        const int r = row0 + rr;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)(__ldg(perm + r) / k) * H);
        uint4 *dst = reinterpret_cast<uint4 *>(x_perm + (size_t)r * H);
        uint32_t emax = 0;
        for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
            const uint4 v = __ldg(src + c);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) emax = max(emax, max((u[j] >> 7) & 0xFFu, (u[j] >> 23) & 0xFFu));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
        if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = emax;
        __syncthreads();
        emax = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) emax = max(emax, wmax[w]);
        __syncthreads();
        int sh = 14 - ((int)emax - 127);
        sh = max(-120, min(120, sh));
        const float up = __int_as_float((127 + sh) << 23);
        if (threadIdx.x == 0) row_inv[r] = __int_as_float((127 - sh) << 23);
        for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
            const uint4 v = __ldg(src + c);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const __half lo = __float2half_rn(bf16_bits_to_float(u[j] & 0xFFFFu) * up);
                const __half hi = __float2half_rn(bf16_bits_to_float(u[j] >> 16) * up);
                o[j] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
            }
            dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

template <class C>
size_t mma_smem_bytes() { return sizeof(MmaSmem<C>) + 1024; }

template <class C>
CUresult make_token_maps(TokenMaps<C> &m, void *base, int cols, int rows, CUtensorMapDataType type) {
    for (int i = 0; i < C::kNumBoxes; ++i) {
        CUresult r = encode_tensor_map_2d(&m.box[i], type, base, (uint64_t)cols, (uint64_t)rows, (uint64_t)cols * 2,
                                          (uint32_t)kTileK, (uint32_t)box_rows<C>(i), CU_TENSOR_MAP_SWIZZLE_128B);
        if (r != CUDA_SUCCESS) return r;
    }
    return CUDA_SUCCESS;
}

template <class C>
cudaError_t set_smem_attrs() {
    cudaError_t e = cudaFuncSetAttribute(mma_kernel<C, Proj::GateUp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)mma_smem_bytes<C>());
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(mma_kernel<C, Proj::Down>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)mma_smem_bytes<C>());
    return e;
}

}  // namespace

struct MmaMaps {
    TokenMaps<BigCfg> x_perm, act;
    TokenMaps<SmallCfg> x_perm_small, act_small;
};

bool mma_use_small_tiles(const Layer &L, int T) {
    return (long long)T * token_slots(L) <= (long long)kMmaSmallMaxAvgTokens * expert_slots(L);
}

cudaError_t mma_setup(Layer &L)
{
    const int maxP = L.desc.max_tokens * token_slots(L);
    const int H = L.desc.hidden, I = L.desc.intermediate;
    MmaMaps *mm = new (std::nothrow) MmaMaps();
    if (!mm) return cudaErrorMemoryAllocation;
    if (make_token_maps(mm->x_perm, L.ws.x_perm, H, maxP, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) != CUDA_SUCCESS ||
        make_token_maps(mm->act, L.ws.act, I, maxP, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) != CUDA_SUCCESS ||
        make_token_maps(mm->x_perm_small, L.ws.x_perm, H, maxP, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) != CUDA_SUCCESS ||
        make_token_maps(mm->act_small, L.ws.act, I, maxP, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) != CUDA_SUCCESS) {
        delete mm;
        return cudaErrorInvalidValue;
    }
    L.mma_maps = mm;
    cudaError_t e = set_smem_attrs<BigCfg>();
    if (e == cudaSuccess) e = set_smem_attrs<SmallCfg>();
    return e;
}

void mma_teardown(Layer &L)
{
    delete static_cast<MmaMaps *>(L.mma_maps);
    L.mma_maps = nullptr;
}

cudaError_t launch_gather(Layer &L, const uint16_t *x, int T, cudaStream_t s, int *launches)
{
    StageTimer timer(L, TFMOE_STAGE_GATHER, s);
    const int P = T * token_slots(L);
    dim3 grid((unsigned)max_mma_entries(P, expert_slots(L)), 16);
    gather_kernel<<<grid, 256, 0, s>>>(x, L.ws.perm, L.ws.mma_entries, L.ws.list_sizes, L.desc.hidden,
                                       token_slots(L), L.ws.x_perm, L.ws.row_inv);
    *launches += 1;
    return cudaGetLastError();
}

static MmaArgs base_args(const Layer &L) {
    MmaArgs a{};
    a.entries = L.ws.mma_entries;
    a.list_sizes = L.ws.list_sizes;
    a.I = L.desc.intermediate;
    a.err_word = L.ws.err_word;
    return a;
}

cudaError_t launch_mma_gate_up(Layer &L, cudaStream_t s, int *launches)
{
    StageTimer timer(L, TFMOE_STAGE_MMA_GATE_UP, s);
    MmaArgs a = base_args(L);
    a.codes = L.w.gu_codes; a.scales = L.w.gu_scales;
    a.glob0 = L.w.gate_global; a.glob1 = L.w.up_global;
    a.R = 2 * L.desc.intermediate; a.K = L.desc.hidden;
    a.act_out = L.ws.act;
    a.row_inv_scale = L.ws.row_inv;
    const MmaMaps *mm = static_cast<const MmaMaps *>(L.mma_maps);
    if (L.mma_small)
        mma_kernel<SmallCfg, Proj::GateUp><<<L.num_sms * SmallCfg::kCtasPerSm, SmallCfg::kThreads,
                                             mma_smem_bytes<SmallCfg>(), s>>>(mm->x_perm_small, a);
    else
        mma_kernel<BigCfg, Proj::GateUp><<<L.num_sms, BigCfg::kThreads, mma_smem_bytes<BigCfg>(), s>>>(mm->x_perm, a);
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_mma_down(Layer &L, cudaStream_t s, int *launches)
{
    StageTimer timer(L, TFMOE_STAGE_MMA_DOWN, s);
    MmaArgs a = base_args(L);
    a.codes = L.w.d_codes; a.scales = L.w.d_scales;
    a.glob0 = L.w.down_global; a.glob1 = nullptr;
    a.R = L.desc.hidden; a.K = L.desc.intermediate;
    a.y_out = L.ws.y;
    const MmaMaps *mm = static_cast<const MmaMaps *>(L.mma_maps);
    if (L.mma_small)
        mma_kernel<SmallCfg, Proj::Down><<<L.num_sms * SmallCfg::kCtasPerSm, SmallCfg::kThreads,
                                           mma_smem_bytes<SmallCfg>(), s>>>(mm->act_small, a);
    else
        mma_kernel<BigCfg, Proj::Down><<<L.num_sms, BigCfg::kThreads, mma_smem_bytes<BigCfg>(), s>>>(mm->act, a);
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace tfmoe
