// mma.cu -- the prefill regime of the NVFP4 grouped expert projections:
// dequantise into the tensor core's operand memory and run BF16 tcgen05 MMAs.
//
// Prefill pushes all prompt tokens through the active experts as one large
// matrix multiply, so it is limited by tensor throughput rather than memory
// (DGX Spark GB10 bandwidth-budget page, section "Mechanism: decode is
// bandwidth-bound, prefill is compute-bound"). The weights stay W4A16: they are
// decoded to BF16 and multiplied against BF16 activations (TensorFold 1.0.12
// GLM-5.3-Flash post, section "NVFP4 is neither uniform 4-bit nor all-FP4
// compute"); the decode is exact (an E2M1 value times an E4M3 scale has at most
// 6 significant bits) and the per-tensor fp32 scale multiplies the fp32
// accumulator in the epilogue.
//
// Tile: 128 weight rows (MMA M) x N <= 256 token rows of one expert (MMA N), the
// reduction in stages of 64. One CTA per SM, persistent over tiles; roles:
//   warp 0     producer: per stage, the token tile (TMA, 128-byte swizzle, box
//              64 x N) and the 4 KB code tile + 2 x 256 B scales (bulk copies)
//   warp 1     allocates tensor memory; lane 0 issues tcgen05.mma (A from tensor
//              memory, B from shared memory, D fp32 in tensor memory) and commits
//   warps 4-7  thread q owns weight row q = tensor-memory lane q: decodes its 64
//              codes per stage to BF16 and stores them into the A stage; after
//              the last stage reads its row of D and runs the epilogue (SwiGLU for
//              interleaved gate/up rows, fp32 store for down).
// Tensor memory: D at columns [0, 256), A stages of 32 columns from 256 on.
// Every wait is bounded; on a timeout the CTA records the error, stops issuing
// work, and still frees its tensor memory.
#include <cuda.h>

#include <new>

#include "common.cuh"
#include "internal.h"

namespace tfmoe {
namespace {

constexpr int kM = 128;
constexpr int kMaxN = kMmaTileTokens;      // 256
constexpr int kStages = 4;
constexpr int kThreads = 256;
constexpr int kDequantWarp0 = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;
constexpr uint32_t kACol = 256;
constexpr int kBStageBytes = kMaxN * 128;  // N rows x 64 bf16
constexpr int kNumBoxes = 5;               // token-tile heights 16, 32, 64, 128, 256

struct MmaSmem {
    uint8_t b[kStages][kBStageBytes];      // 1024-byte aligned (each stage is 32 KB)
    uint8_t codes[kStages][kTileCodeBytes];
    uint8_t scales[kStages][kTileScaleBytes];
    uint64_t full[kStages], empty[kStages], aready[kStages];
    uint64_t dfull, dempty;
    uint32_t tmem_base;
    int32_t abort_flag;
};

struct TokenMaps {
    CUtensorMap box[kNumBoxes];            // same tensor, box heights 16 << i
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
    int I;
    int32_t *err_word;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, MmaSmem &sm, int32_t *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        for (int i = 0; i < 128; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*reinterpret_cast<volatile int32_t *>(&sm.abort_flag)) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, DEV_ERR_WAIT_TIMEOUT);
            *reinterpret_cast<volatile int32_t *>(&sm.abort_flag) = 1;
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

// kind::f16, A = B = BF16 (K-major), D = F32, M = 128, N given.
__device__ __forceinline__ uint32_t instr_desc_bf16(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u));
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]));
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Two E2M1 codes (one byte) times the block scale (f16 pair, both halves equal) -> bf16x2.
// Products are exact in f16 (<= 6 significant bits, magnitudes 2^-10 .. 2688) and in bf16.
__device__ __forceinline__ uint32_t dequant_pair_bf16(uint32_t byte, __half2 scale2) {
    const uint32_t h = e2m1x2_to_f16x2(byte);
    const __half2 v = __hmul2(*reinterpret_cast<const __half2 *>(&h), scale2);
    const float2 f = __half22float2(v);
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<const uint32_t *>(&b);
}

__device__ __forceinline__ int box_index(int rows) {
    int i = 0;
    while ((16 << i) < rows && i < kNumBoxes - 1) ++i;
    return i;
}

template <Proj P>
__global__ void __launch_bounds__(kThreads, 1) mma_kernel(const __grid_constant__ TokenMaps maps, const MmaArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    MmaSmem &sm = *reinterpret_cast<MmaSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = a.K / kTileK, RT = a.R / kM;
    const int n_tiles = __ldg(a.list_sizes + 2) * RT;
    if ((int)blockIdx.x >= n_tiles) return;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
            mbar_init(&sm.aready[s], 128);
        }
        mbar_init(&sm.dfull, 1);
        mbar_init(&sm.dempty, 128);
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

    if (warp == 0) {
        if (lane == 0) {
            uint32_t g = 0;
            uint32_t issued = 0;
            for (int t = blockIdx.x; t < n_tiles && !sm.abort_flag; t += gridDim.x) {
                const int32_t *ent = a.entries + 4 * (t / RT);
                const int e = __ldg(ent), row0 = __ldg(ent + 1), rows = __ldg(ent + 2);
                const int rt = t % RT, bi = box_index(rows);
                const uint32_t b_bytes = (uint32_t)(16 << bi) * 128u;
                const size_t rti = (size_t)e * RT + rt;
                for (int kt = 0; kt < KT; ++kt, ++g) {
                    const int s = g % kStages;
                    const uint32_t ph = (g / kStages) & 1u;
                    if (!wait_or_abort(&sm.empty[s], ph ^ 1u, sm, a.err_word)) break;
                    mbar_arrive_expect_tx(&sm.full[s], b_bytes + kTileCodeBytes + kTileScaleBytes);
                    tma_load_2d(sm.b[s], &maps.box[bi], kt * kTileK, row0, &sm.full[s]);
                    bulk_g2s(sm.codes[s], a.codes + (rti * KT + kt) * kTileCodeBytes, kTileCodeBytes, &sm.full[s]);
                    bulk_g2s(sm.scales[s], a.scales + scale_offset(rti, KT, 0, kt), kTileScaleBytes / 2, &sm.full[s]);
                    bulk_g2s(sm.scales[s] + kTileScaleBytes / 2, a.scales + scale_offset(rti, KT, 1, kt),
                             kTileScaleBytes / 2, &sm.full[s]);
                    issued = g + 1;
                }
            }
            if (sm.abort_flag) {
                // aborted: let the copies already issued land before the CTA exits (bounded)
                for (uint32_t j = (issued > kStages ? issued - kStages : 0); j < issued; ++j) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(&sm.full[j % kStages], (j / kStages) & 1u) &&
                           global_timer_ns() - t0 < kWaitLimitNs / 4) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            uint32_t g = 0, tile_i = 0;
            for (int t = blockIdx.x; t < n_tiles && !sm.abort_flag; t += gridDim.x, ++tile_i) {
                const int rows = __ldg(a.entries + 4 * (t / RT) + 2);
                const int n = 16 << box_index(rows);
                const uint32_t idesc = instr_desc_bf16(n);
                if (!wait_or_abort(&sm.dempty, (tile_i & 1u) ^ 1u, sm, a.err_word)) break;
                tc_fence_after();
                bool ok = true;
                for (int kt = 0; kt < KT; ++kt, ++g) {
                    const int s = g % kStages;
                    const uint32_t ph = (g / kStages) & 1u;
                    if (!wait_or_abort(&sm.full[s], ph, sm, a.err_word) ||
                        !wait_or_abort(&sm.aready[s], ph, sm, a.err_word)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t b0 = smem_u32(sm.b[s]);
#pragma unroll
                    for (int k4 = 0; k4 < kTileK / 16; ++k4)
                        mma_bf16_ts(tmem + kAccCol, tmem + kACol + (uint32_t)s * 32u + (uint32_t)k4 * 8u,
                                    smem_desc_sw128(b0 + (uint32_t)k4 * 32u), idesc, (kt | k4) != 0);
                    mma_commit(&sm.empty[s]);
                }
                if (!ok) break;
                mma_commit(&sm.dfull);
            }
        }
    } else if (warp >= kDequantWarp0) {
        const int q = threadIdx.x - kDequantWarp0 * 32;          // weight row of the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)((warp - kDequantWarp0) * 32) << 16;
        uint32_t g = 0, tile_i = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tile_i) {
            const int32_t *ent = a.entries + 4 * (t / RT);
            const int e = __ldg(ent), row0 = __ldg(ent + 1), rows = __ldg(ent + 2);
            const int rt = t % RT;
            const int n = 16 << box_index(rows);
            bool ok = !sm.abort_flag;
            for (int kt = 0; kt < KT && ok; ++kt, ++g) {
                const int s = g % kStages;
                const uint32_t ph = (g / kStages) & 1u;
                ok = wait_or_abort(&sm.full[s], ph, sm, a.err_word);
                if (ok) ok = wait_or_abort(&sm.empty[s], ph ^ 1u, sm, a.err_word);   // A stage free
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                const uint4 c0 = *reinterpret_cast<const uint4 *>(sm.codes[s] + q * 16);
                const uint4 c1 = *reinterpret_cast<const uint4 *>(sm.codes[s] + 2048 + q * 16);
                const uint32_t sc4 = *reinterpret_cast<const uint32_t *>(sm.scales[s] + q * 4);
                const uint32_t s01 = e4m3x2_to_f16x2(sc4 & 0xFFFFu), s23 = e4m3x2_to_f16x2(sc4 >> 16);
                const __half2 h01 = *reinterpret_cast<const __half2 *>(&s01);
                const __half2 h23 = *reinterpret_cast<const __half2 *>(&s23);
                const __half2 sb[4] = {__low2half2(h01), __high2half2(h01), __low2half2(h23), __high2half2(h23)};
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint32_t r[32];
#pragma unroll
                for (int w8 = 0; w8 < 8; ++w8)       // word w8 holds elements 8*w8 .. 8*w8 + 7
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        r[4 * w8 + b] = dequant_pair_bf16((words[w8] >> (8 * b)) & 0xFFu, sb[w8 >> 1]);
                tmem_st32(tmem + lane_base + kACol + (uint32_t)s * 32u, r);
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(&sm.aready[s]);
            }
            if (!ok) break;
            // epilogue: this thread's row of D, N token columns
            if (!wait_or_abort(&sm.dfull, tile_i & 1u, sm, a.err_word)) break;
            tc_fence_after();
            const int grow = rt * kM + q;
            const float gs = (P == Proj::GateUp) ? ((grow & 1) ? __ldg(a.glob1 + e) : __ldg(a.glob0 + e))
                                                 : __ldg(a.glob0 + e);
            for (int c = 0; c < n; c += 32) {
                uint32_t d[32];
                tmem_ld32(tmem + lane_base + kAccCol + (uint32_t)c, d);
                tc_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float v = __uint_as_float(d[i]) * gs;
                    const int tok = c + i;
                    if (P == Proj::GateUp) {
                        const float other = __shfl_xor_sync(0xffffffffu, v, 1);
                        if (!(grow & 1) && tok < rows)
                            a.act_out[(size_t)(row0 + tok) * a.I + (grow >> 1)] = float_to_bf16_bits_rn(silu_f32(v) * other);
                    } else {
                        if (tok < rows) a.y_out[(size_t)(row0 + tok) * a.R + grow] = v;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&sm.dempty);
        }
    }
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

// x_perm[r] = x[token of pair perm[r]] for the rows of every MMA token tile.
__global__ void __launch_bounds__(256) gather_kernel(const uint16_t *__restrict__ x, const int32_t *__restrict__ perm,
                                                     const int32_t *__restrict__ entries,
                                                     const int32_t *__restrict__ list_sizes, int H, int k,
                                                     uint16_t *__restrict__ x_perm)
{
    const int ent = blockIdx.x;
    if (ent >= __ldg(list_sizes + 2)) return;
    const int row0 = __ldg(entries + 4 * ent + 1), rows = __ldg(entries + 4 * ent + 2);
    const int chunks = H / 8;
    for (int rr = blockIdx.y; rr < rows; rr += gridDim.y) {
        const int r = row0 + rr;
        const uint16_t *src = x + (size_t)(__ldg(perm + r) / k) * H;
        uint16_t *dst = x_perm + (size_t)r * H;
        for (int c = threadIdx.x; c < chunks; c += blockDim.x)
            reinterpret_cast<uint4 *>(dst)[c] = __ldg(reinterpret_cast<const uint4 *>(src) + c);
    }
}

size_t mma_smem_bytes() { return sizeof(MmaSmem) + 1024; }

// cuTensorMapEncodeTiled, looked up through the runtime so the library does not
// link the driver library directly (it loads on machines without a GPU driver).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

CUresult make_token_maps(TokenMaps &m, void *base, int cols, int rows) {
    EncodeTiledFn encode = encode_tiled_fn();
    if (!encode) return CUDA_ERROR_NOT_FOUND;
    for (int i = 0; i < kNumBoxes; ++i) {
        const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
        const cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kTileK, (cuuint32_t)(16 << i)};
        const cuuint32_t estride[2] = {1, 1};
        CUresult r = encode(&m.box[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, gdim, gstride, box,
                                            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return r;
    }
    return CUDA_SUCCESS;
}

}  // namespace

struct MmaMaps {
    TokenMaps x_perm, act;
};

cudaError_t mma_setup(Layer &L)
{
    const int maxP = L.desc.max_tokens * L.desc.top_k;
    MmaMaps *mm = new (std::nothrow) MmaMaps();
    if (!mm) return cudaErrorMemoryAllocation;
    if (make_token_maps(mm->x_perm, L.ws.x_perm, L.desc.hidden, maxP) != CUDA_SUCCESS ||
        make_token_maps(mm->act, L.ws.act, L.desc.intermediate, maxP) != CUDA_SUCCESS) {
        delete mm;
        return cudaErrorInvalidValue;
    }
    L.mma_maps = mm;
    cudaError_t e = cudaFuncSetAttribute(mma_kernel<Proj::GateUp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)mma_smem_bytes());
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(mma_kernel<Proj::Down>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)mma_smem_bytes());
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
    const int P = T * L.desc.top_k;
    dim3 grid((unsigned)max_mma_entries(P, L.desc.num_experts), 16);
    gather_kernel<<<grid, 256, 0, s>>>(x, L.ws.perm, L.ws.mma_entries, L.ws.list_sizes, L.desc.hidden,
                                       L.desc.top_k, L.ws.x_perm);
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
    const MmaMaps *mm = static_cast<const MmaMaps *>(L.mma_maps);
    mma_kernel<Proj::GateUp><<<L.num_sms, kThreads, mma_smem_bytes(), s>>>(mm->x_perm, a);
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
    mma_kernel<Proj::Down><<<L.num_sms, kThreads, mma_smem_bytes(), s>>>(mm->act, a);
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace tfmoe
