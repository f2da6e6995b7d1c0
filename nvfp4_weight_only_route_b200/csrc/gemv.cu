// gemv.cu -- the decode regime of the NVFP4 grouped expert projections:
// bandwidth-bound GEMV on CUDA cores, no tensor cores.
//
// Decode reads each routed expert's 4-bit weights once per step, so its time
// is the weight bytes over HBM bandwidth (DGX Spark GB10 bandwidth-budget
// page, section "Mechanism: decode is bandwidth-bound, prefill is
// compute-bound"); the expert up/down kernels are the largest share of decode
// GPU time in TensorFold issue #627 (comment with the RTX 4090 per-launch
// table). So the kernel is built around the memory stream: the packed codes
// arrive with 128-bit coalesced loads (16-byte cp.async per lane) into a
// per-warp shared-memory ring that runs two 4-tile chunks ahead, across passes
// and tasks; each task's E4M3 block scales arrive in shared memory with one
// 2-D tensor copy (TMA), and each pass's activation rows with bulk copies,
// both issued two passes ahead by a control warp. Per weight and token the
// inner loop spends one mixed-precision FMA and half an E2M1 conversion; the
// addresses are 32-bit shared-memory bases with immediate offsets, so little
// else is issued.
//
// Task = (expert of the GEMV list, 16*RG consecutive weight rows). The 8 warps
// of a CTA split it as RG row groups x KS column slices (RG * KS = 8): lane l
// of a warp owns row (l % 16) of its group and half (l / 16) of every 64-column
// tile of its slice (16 code bytes = 32 weights, 2 scale bytes). Partial sums
// leave the warp through a shuffle (the two halves) and shared memory (the
// slices), added in a fixed order; then the epilogue threads (one per row and
// token) apply the per-tensor scale and either SwiGLU (gate/up) or the fp32
// store (down). Tasks are small so that the few waves of a decode step stay
// balanced across the CTAs; when a batch gives every CTA several tasks, the
// down projection switches to longer ones (fewer column slices, more tiles per
// warp and pass).
//
// Arithmetic: the activation operand is an f16 tensor with one power of two
// per 16 elements (exact for every bf16 element within 2^28 of its block's
// largest; the routing kernels write it for x, the gate/up epilogue for the
// SwiGLU output a). E2M1 -> f16 is exact and each product w*x is exact inside
// one mixed-precision fma.rn.f32.f16, so a 16-element partial sum is an fp32
// sum of exact products; it is scaled by (E4M3 block scale * inverse power of
// two of the activation block, an exact product) into the fp32 row accumulator.
#include <algorithm>
#include <new>

#include "common.cuh"
#include "internal.h"

namespace tfmoe {
namespace {

constexpr int kWarps = 8;                       // compute warps (column slices x row groups)
constexpr int kComputeWarps = kWarps;
constexpr int kThreads = (kComputeWarps + 1) * 32;   // + the control warp
constexpr int kCtasPerSm = 2;
constexpr int kChunk = 4;   // column tiles per ring slot of a compute warp
constexpr int kRing = 3;    // ring slots per compute warp (kRing - 1 chunks in flight)
static_assert(kRing >= 2, "ring depth");
constexpr int kMaxNT = 2;
constexpr uint32_t kTestWaitNs = 1000000;   // the forced-timeout test's wait: 1 ms   // tokens per pass (the partial sums of a pass are one f32 pair per lane)

enum class Proj { GateUp, Down };

// A GEMV task: id = li * tpe + sub (entry li of the GEMV list, row group sub).
struct Cursor {
    int id, li, sub;
};

struct GemvArgs {
    const uint8_t *codes;       // tiled codes of all experts
    const float *glob0;         // gate (GateUp) or down (Down) per-tensor scale [E]
    const float *glob1;         // up (GateUp)
    int R, K;                   // rows (2I or H) and reduction length (H or I)
    int KS, RG;                 // column slices and 16-row groups of a task
    const int32_t *expert_list; // GEMV-regime experts
    const int32_t *list_size;   // [0] = number of GEMV experts
    const int32_t *offsets;     // [E+1]
    const int32_t *perm;        // [P] pair index of permuted row
    int top_k;
    const uint16_t *src;        // GateUp: xq [T][H] (token rows); Down: aq [P][I] (permuted rows)
    const float *src_inv;       // [rows][K/16] inverse powers of two of src
    uint16_t *act_out;          // GateUp: act [P][I] bf16
    uint16_t *aq_out;           // GateUp: aq [P][I]
    float *aq_inv_out;          // GateUp: [P][I/16]
    float *y_out;               // Down output [P][H]
    int I;
    int32_t *err_word;
    uint32_t test_wait_ns;      // > 0: CTA 0 first waits this long on a barrier nothing completes
};

struct Geometry {
    int KS, RG;
};

// Gate/up tasks hold at least two 16-row groups (32 interleaved rows = 16 SwiGLU
// outputs = one 16-element block of a). KT = K / 64 is even there (H % 128 == 0).
// Each projection has two task shapes: the default one (more, shorter tasks) and a
// long one (each warp streams more column tiles per pass, so the per-pass costs are
// spread over more weights), used when the batch gives every CTA enough tasks.
constexpr int kGateUpLongKS = 4;     // column slices of the long gate/up task shape
constexpr int kDownLongKS = 2;       // column slices of the long down task shape
constexpr int kLongTasksPerCta = 4;   // the long shape needs this many tasks per CTA (estimated)
Geometry geometry_from(int ks_start, int K) {
    const int KT = K / kTileK;
    int KS = ks_start;
    while (KT % KS) KS >>= 1;
    return {KS, kWarps / KS};
}
Geometry geometry(bool gate_up, int K) {
    const int KT = K / kTileK;
    int KS = gate_up ? 4 : 8;
    while (KT % KS) KS >>= 1;
    return {KS, kWarps / KS};
}

// Shared memory of a CTA, in bytes from a 128-byte aligned base: two buffers each of
// the task's scales [KT][16*RG] u32, the partial sums [KS][16*RG][kMaxNT] f32, the
// pass's activation rows [kMaxNT][K] f16 and their inverse scales [kMaxNT][K/16] f32;
// the GEMV list table [5][<= 256] (expert, first row, rows, per-tensor scales); per compute warp a ring of kRing code chunks
// (kChunk tiles x 32 lanes x 16 bytes); 8 mbarriers, an abort flag and a barrier that
// nothing completes (the forced-timeout test).
constexpr int kMaxList = 256;
struct SmemLayout {
    size_t sc_sz, red_sz, x_sz, xi_sz;
    size_t sc, red, x, xi, tab, ring, bar, total;
    __host__ __device__ __forceinline__ SmemLayout(int K, int KS, int RG) {
        sc_sz = ((size_t)(K / kTileK) * 16 * RG * 4 + 127) & ~static_cast<size_t>(127);
        red_sz = (size_t)KS * 16 * RG * kMaxNT * 4;
        x_sz = (size_t)kMaxNT * K * 2;
        xi_sz = ((size_t)kMaxNT * (K / 16) * 4 + 127) & ~static_cast<size_t>(127);
        sc = 0;
        red = sc + 2 * sc_sz;
        x = red + 2 * red_sz;
        xi = x + 2 * x_sz;
        tab = xi + 2 * xi_sz;
        ring = tab + 5 * kMaxList * 4;
        bar = ring + (size_t)kComputeWarps * kRing * kChunk * 32 * 16;
        total = bar + 10 * sizeof(uint64_t);
    }
};
size_t gemv_smem_bytes(int K, Geometry g) { return 128 + SmemLayout(K, g.KS, g.RG).total; }

// 16-byte asynchronous copy global -> shared (cp.async, bypassing L1): the code stream
// stays 128-bit coalesced loads while the data waits in shared memory, not registers.
// The offsets are immediates of the instruction: a chunk's copies share two base registers.
template <int DOFF, int SOFF>
__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void *gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0+%2], [%1+%3], 16;" ::"r"(smem_dst), "l"(gmem_src), "n"(DOFF),
                 "n"(SOFF) : "memory");
}
// Shared-memory loads by 32-bit address: the inner loop's addresses are a few
// per-pass bases plus constant offsets, with no generic-pointer arithmetic.
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
template <int OFF>
__device__ __forceinline__ float2 lds64f(uint32_t a) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2+%3];" : "=f"(v.x), "=f"(v.y) : "r"(a), "n"(OFF));
    return v;
}
__device__ __forceinline__ void sts_f32x2(uint32_t a, float v0, float v1) {
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(v0), "f"(v1) : "memory");
}
template <int OFF>
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4+%5];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a), "n"(OFF));
    return v;
}
// The E4M3 pair in bits [sh, sh + 16) of w -> two floats (exact).
__device__ __forceinline__ float2 e4m3_pair_at(uint32_t w, uint32_t sh) {
    uint32_t h2;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}" : "=r"(h2) : "r"(w >> sh));
    return f16x2_to_float2(h2);
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// acc += w * x over two f16 pairs, each product exact, one fp32 rounding per step.
__device__ __forceinline__ float fma2_f16_f32(uint32_t w2, uint32_t x2, float acc) {
    asm("{\n\t.reg .f16 wl, wh, xl, xh;\n\t"
        "mov.b32 {wl, wh}, %1;\n\tmov.b32 {xl, xh}, %2;\n\t"
        "fma.rn.f32.f16 %0, wl, xl, %0;\n\tfma.rn.f32.f16 %0, wh, xh, %0;\n\t}"
        : "+f"(acc) : "r"(w2), "r"(x2));
    return acc;
}

// Eight weights (one code word) against the matching 8 activations of each token:
// XOFF is the byte offset of those activations from the chunk's bases xa0 / xa1.
template <int NT, int XOFF>
__device__ __forceinline__ void word8(uint32_t w, uint32_t xa0, uint32_t xa1, float (&pp)[NT]) {
    uint32_t wp[4];
    e2m1x8_to_f16x2x4(w, wp);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const uint4 xv = lds128<XOFF>(t == 0 ? xa0 : xa1);
        pp[t] = fma2_f16_f32(wp[0], xv.x, pp[t]);
        pp[t] = fma2_f16_f32(wp[1], xv.y, pp[t]);
        pp[t] = fma2_f16_f32(wp[2], xv.z, pp[t]);
        pp[t] = fma2_f16_f32(wp[3], xv.w, pp[t]);
    }
}

// Tile J of a chunk: the lane's 32 weights (16 code bytes at cs + 512 J) against NT
// tokens. Activations of token t start at xa_t + 128 J (32 f16 values, 4 per word
// pair) with their two inverse block scales at xi_t + 16 J; the lane's two E4M3
// scales are bits [hsh, hsh + 16) of the word at sc.
template <int NT, int J>
__device__ __forceinline__ void tile_compute(uint32_t cs, uint32_t sc, uint32_t hsh, uint32_t xa0, uint32_t xa1,
                                             uint32_t xi0, uint32_t xi1, float (&acc)[kMaxNT])
{
    const float2 s = e4m3_pair_at(lds32(sc), hsh);
    const uint4 cw = lds128<J * 512>(cs);
    float p0[NT], p1[NT];   // 16-column blocks 0 and 1 of the lane's 32 columns
#pragma unroll
    for (int t = 0; t < NT; ++t) p0[t] = p1[t] = 0.f;
    word8<NT, J * 128 + 0>(cw.x, xa0, xa1, p0);
    word8<NT, J * 128 + 16>(cw.y, xa0, xa1, p0);
    word8<NT, J * 128 + 32>(cw.z, xa0, xa1, p1);
    word8<NT, J * 128 + 48>(cw.w, xa0, xa1, p1);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const float2 inv = lds64f<J * 16>(t == 0 ? xi0 : xi1);
        acc[t] = fmaf(p0[t], s.x * inv.x, acc[t]);
        acc[t] = fmaf(p1[t], s.y * inv.y, acc[t]);
    }
}

// The n <= kChunk tiles of one chunk (n is a constant for full chunks).
static_assert(kChunk == 4, "tile_compute is unrolled for 4-tile chunks");
template <int NT>
__device__ __forceinline__ void chunk_compute(uint32_t cs, int n, uint32_t sc, uint32_t sc_step, uint32_t hsh,
                                              uint32_t xa0, uint32_t xa1, uint32_t xi0, uint32_t xi1,
                                              float (&acc)[kMaxNT])
{
    tile_compute<NT, 0>(cs, sc, hsh, xa0, xa1, xi0, xi1, acc);
    if (n > 1) tile_compute<NT, 1>(cs, sc + sc_step, hsh, xa0, xa1, xi0, xi1, acc);
    if (n > 2) tile_compute<NT, 2>(cs, sc + 2 * sc_step, hsh, xa0, xa1, xi0, xi1, acc);
    if (n > 3) tile_compute<NT, 3>(cs, sc + 3 * sc_step, hsh, xa0, xa1, xi0, xi1, acc);
}

// A lane's position in its code stream. The ring holds kRing chunk slots of
// kChunk * 512 bytes; `use` and `fill` are byte offsets of the slot read next and
// the slot filled next (kRing - 1 slots apart).
constexpr uint32_t kSlotBytes = kChunk * 512;
__device__ __forceinline__ uint32_t next_slot(uint32_t off) {
    return off == (kRing - 1) * kSlotBytes ? 0u : off + kSlotBytes;
}

// All column chunks of one pass: wait for the lane's oldest copies, compute, and let
// `refill` put the next chunk of the stream into the slot freed by the previous one.
template <int NT, class Refill>
__device__ __forceinline__ void pass_run(uint32_t ring, uint32_t &use, int nch, int n_last, uint32_t sc,
                                         uint32_t sc_step, uint32_t hsh, uint32_t xa0, uint32_t xa1, uint32_t xi0,
                                         uint32_t xi1, float (&acc)[kMaxNT], Refill &refill)
{
    for (int ch = 0; ch < nch; ++ch) {
        cp_async_wait<kRing - 2>();
        if (ch + 1 < nch || n_last == kChunk)
            chunk_compute<NT>(ring + use, kChunk, sc, sc_step, hsh, xa0, xa1, xi0, xi1, acc);
        else
            chunk_compute<NT>(ring + use, n_last, sc, sc_step, hsh, xa0, xa1, xi0, xi1, acc);
        refill();
        use = next_slot(use);
        sc += kChunk * sc_step;
        xa0 += kChunk * 128;
        xa1 += kChunk * 128;
        xi0 += kChunk * 16;
        xi1 += kChunk * 16;
    }
}

// Bounded mbarrier wait shared by every role of the CTA: gives up (returning false)
// once another thread has flagged an abort or after kWaitLimitNs, flagging it itself.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int32_t *abort_flag,
                                              int32_t *err_word) {
    if (mbar_try_wait_at(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        for (int i = 0; i < 4; ++i)
            if (mbar_try_wait_sleep_at(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            atomicOr(err_word, DEV_ERR_WAIT_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

// CTA = 8 compute warps + 1 control warp. The compute warps only stream codes and
// do arithmetic: they never wait for one another. The control warp issues the
// tensor/bulk copies of scales and activation rows two passes ahead (pass p+2's as
// soon as pass p's partial sums are in) and runs one pass behind adding the compute
// warps' partial sums (in slice order) and storing the outputs, so no warp holds a
// CTA-wide barrier per pass.
//
// Barriers (parity = use count / 2 mod 2, every barrier alternating between 2 buffers):
//   sfull[b]  scales of task #i landed (b = i & 1; expect-tx by the control warp)
//   xfull[b]  activation rows of pass #p landed (b = p & 1)
//   full[b]   the 8 compute warps wrote their partial sums of pass #p (count 8)
//   rfree[b]  the control warp consumed the partial sums of pass #p (count 1)
// A buffer of scales / activations is refilled only after the control warp saw
// full[] of the last pass that read it, which the compute warps signal after reading.
template <Proj P>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) gemv_kernel(const __grid_constant__ CUtensorMap smap,
                                                                    const GemvArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    // everything gate/up reads comes from the kernels before it: were it launched as their
    // programmatic dependent, it would wait here (a no-op for the plain launch it gets), before
    // it lets the down projection launch
    if (P == Proj::GateUp) grid_dep_wait();
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int K = a.K, KT = K / kTileK, KS = a.KS, RG = a.RG;
    const int rows_task = 16 * RG, KTW = KT / KS;
    const int rt_log2 = 31 - __clz(rows_task);            // rows_task is a power of two
    const int RT = a.R / kTileRows, tpe = a.R / rows_task;
    const int n_list = __ldg(a.list_size);
    const int n_tasks = n_list * tpe;
    // The next launch (down after gate/up, the combine after down) depends on this grid
    // programmatically: its CTAs may start while this grid runs and wait for it there.
    grid_dep_launch_dependents();
    if ((int)blockIdx.x >= n_tasks) return;

    const SmemLayout lay(K, KS, RG);
    auto sbuf = [&](int b) { return reinterpret_cast<uint32_t *>(base + lay.sc + b * lay.sc_sz); };
    auto red = [&](int b) { return reinterpret_cast<float *>(base + lay.red + b * lay.red_sz); };
    auto xbuf = [&](int b) { return reinterpret_cast<uint16_t *>(base + lay.x + b * lay.x_sz); };
    auto xibuf = [&](int b) { return reinterpret_cast<float *>(base + lay.xi + b * lay.xi_sz); };
    int32_t *tab = reinterpret_cast<int32_t *>(base + lay.tab);     // [5][n_list]: expert, first row, rows, g0, g1
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + lay.bar);
    uint64_t *sfull = bars, *xfull = bars + 2, *full = bars + 4, *rfree = bars + 6;
    volatile int32_t *abort_flag = reinterpret_cast<volatile int32_t *>(bars + 8);
    uint64_t *never = bars + 9;                           // no thread ever arrives on it

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sfull[i], 1);
            mbar_init(&xfull[i], 1);
            mbar_init(&full[i], kComputeWarps);
            mbar_init(&rfree[i], 1);
        }
        mbar_init(never, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // the GEMV list with each expert's rows, read once (one dependent load per thread)
    for (int i = threadIdx.x; i < n_list; i += kThreads) {
        const int e = __ldg(a.expert_list + i);
        const int rb = __ldg(a.offsets + e);
        tab[i] = e;
        tab[n_list + i] = rb;
        tab[2 * n_list + i] = __ldg(a.offsets + e + 1) - rb;
        tab[3 * n_list + i] = __float_as_int(__ldg(a.glob0 + e));
        tab[4 * n_list + i] = P == Proj::GateUp ? __float_as_int(__ldg(a.glob1 + e)) : 0;
    }
    __syncthreads();

    // The CTA's tasks are blockIdx.x + i * gridDim.x. A cursor carries a task's list
    // entry (li = task / tpe) and row group (sub = task % tpe) and steps without dividing.
    const int g_li = (int)gridDim.x / tpe, g_sub = (int)gridDim.x % tpe;
    const Cursor c0{(int)blockIdx.x, (int)blockIdx.x / tpe, (int)blockIdx.x % tpe};
    auto advance = [&](Cursor &c) {
        c.id += gridDim.x;
        c.li += g_li;
        c.sub += g_sub;
        if (c.sub >= tpe) { c.sub -= tpe; ++c.li; }
    };
    auto task_rows = [&](const Cursor &c, int &r_begin) {
        r_begin = tab[n_list + c.li];
        return tab[2 * n_list + c.li];
    };
    // the pass after (task c, t0) in this CTA's sequence; tasks without rows have no pass
    auto next_pass = [&](const Cursor &c, int t0, int m, Cursor &nc, int &nt0) {
        if (t0 + kMaxNT < m) { nc = c; nt0 = t0 + kMaxNT; return true; }
        Cursor k = c;
        for (advance(k); k.id < n_tasks; advance(k)) {
            int rb;
            if (task_rows(k, rb) > 0) { nc = k; nt0 = 0; return true; }
        }
        return false;
    };
    auto first_pass = [&](Cursor &fc) {
        int rb, t0;
        if (task_rows(c0, rb) > 0) { fc = c0; return true; }
        return next_pass(c0, 0, 0, fc, t0);
    };

    if (warp == kComputeWarps) {
        // ------------------------------------------------------------ control warp
        const uint32_t scale_tx = (uint32_t)(KT * rows_task * 4);
        // per buffer: whether a copy was issued into it and the phase parity of the latest
        // one. A buffer is refilled only after every compute warp waited for (or, aborting,
        // gave up on) its previous copy, and after an abort nothing is issued, so each of
        // the four barriers has at most one phase in flight: its latest.
        bool s_used[2] = {false, false}, x_used[2] = {false, false};
        uint32_t s_par[2] = {0u, 0u}, x_par[2] = {0u, 0u};
        auto issue = [&](const Cursor &c, int t0, int tn, int p, bool first) {
            int r_begin;
            const int m = task_rows(c, r_begin);
            const int nt = min(kMaxNT, m - t0);
            int row = 0;
            if (lane < nt) {
                const int r = r_begin + t0 + lane;
                row = (P == Proj::GateUp) ? __ldg(a.perm + r) / a.top_k : r;
            }
            const int xb = p & 1;
            if (lane == 0) {
                if (t0 == 0) {
                    const int sb = tn & 1, row0 = c.sub * rows_task;
                    mbar_arrive_expect_tx(&sfull[sb], scale_tx);
                    tma_load_2d(sbuf(sb), &smap, row0 % kTileRows, (tab[c.li] * RT + row0 / kTileRows) * KT,
                                &sfull[sb]);
                    s_used[sb] = true;
                    s_par[sb] = (tn >> 1) & 1;
                }
            }
            // the down pass reads aq, which the gate/up grid writes: wait for that grid here,
            // after the first scale copy and before the first activation copy
            if (P == Proj::Down && first) {
                __syncwarp();
                grid_dep_wait();
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&xfull[xb], (uint32_t)nt * (uint32_t)(K * 2 + K / 4));
                x_used[xb] = true;
                x_par[xb] = (p >> 1) & 1;
            }
            for (int t = 0; t < nt; ++t) {
                const int rr = __shfl_sync(0xffffffffu, row, t);
                if (lane == 0) {
                    bulk_g2s(xbuf(xb) + (size_t)t * K, a.src + (size_t)rr * K, (uint32_t)K * 2, &xfull[xb]);
                    bulk_g2s(xibuf(xb) + (size_t)t * (K / 16), a.src_inv + (size_t)rr * (K / 16), (uint32_t)K / 4,
                             &xfull[xb]);
                }
            }
        };
        // The issue cursor runs two passes ahead of the pass being consumed: pass p+2's
        // copies go out as soon as pass p's partial sums are in (its buffers were last
        // read by pass p), before pass p's epilogue.
        Cursor ic;
        bool ivalid = first_pass(ic);
        int it0 = 0, itn = 0, ip = 0;
        auto issue_next = [&](bool first) {
            // after an abort no copy is issued: a compute warp may have stopped waiting for
            // the copy that last filled the buffer (its arrive on full[] publishes the flag)
            if (!ivalid || *abort_flag) return;
            int rb;
            const int m = task_rows(ic, rb);
            issue(ic, it0, itn, ip, first);
            Cursor nc;
            int nt0;
            if (next_pass(ic, it0, m, nc, nt0)) {
                if (nc.id != ic.id) ++itn;
                ic = nc;
                it0 = nt0;
            } else {
                ivalid = false;
            }
            ++ip;
        };
        Cursor fc;
        if (first_pass(fc)) {
            issue_next(true);
            issue_next(false);
            int p = 0;
            for (Cursor c = fc; c.id < n_tasks; advance(c)) {
                int r_begin;
                const int m = task_rows(c, r_begin);
                if (m <= 0) continue;
                const int row0 = c.sub * rows_task;
                for (int t0 = 0; t0 < m; t0 += kMaxNT, ++p) {
                    const int nt = min(kMaxNT, m - t0);
                    wait_or_abort(smem_u32(&full[p & 1]), (p >> 1) & 1, abort_flag, a.err_word);
                    issue_next(false);
                    const float *rb = red(p & 1);
                    if (P == Proj::GateUp) {
                        // rows_task is a multiple of 32: a round covers 32 rows (16 gate/up pairs) of one token
                        const float g0 = __int_as_float(tab[3 * n_list + c.li]), g1 = __int_as_float(tab[4 * n_list + c.li]);
                        for (int i0 = 0; i0 < rows_task * nt; i0 += 32) {
                            const int i = i0 + lane, t = i >> rt_log2, rl = i & (rows_task - 1);
                            float v = 0.f;
                            for (int s = 0; s < KS; ++s) v += rb[((size_t)s * rows_task + rl) * kMaxNT + t];
                            const int grow = row0 + rl;
                            const bool up = (grow & 1) != 0;
                            v *= up ? g1 : g0;
                            const float other = __shfl_xor_sync(0xffffffffu, v, 1);
                            const size_t r = (size_t)(r_begin + t0 + t);
                            const int j = grow >> 1;
                            uint32_t ab = 0;
                            if (!up) {
                                ab = float_to_bf16_bits_rn(silu_f32(v) * other);
                                a.act_out[r * a.I + j] = (uint16_t)ab;
                            }
                            // the round's 16 outputs form one block of aq and share its power of two
                            const uint32_t emax = __reduce_max_sync(0xffffffffu, up ? 0u : ((ab >> 7) & 0xFFu));
                            int sh = 14 - ((int)emax - 127);
                            sh = max(-120, min(120, sh));
                            if (!up)
                                a.aq_out[r * a.I + j] = __half_as_ushort(
                                    __float2half_rn(bf16_bits_to_float(ab) * __int_as_float((127 + sh) << 23)));
                            if (lane == 0) a.aq_inv_out[r * (a.I / 16) + (j >> 4)] = __int_as_float((127 - sh) << 23);
                        }
                    } else {
                        const float gs = __int_as_float(tab[3 * n_list + c.li]);
                        for (int i = lane; i < rows_task * nt; i += 32) {
                            const int t = i >> rt_log2, rl = i & (rows_task - 1);
                            float v = 0.f;
                            for (int s = 0; s < KS; ++s) v += rb[((size_t)s * rows_task + rl) * kMaxNT + t];
                            a.y_out[(size_t)(r_begin + t0 + t) * a.R + row0 + rl] = v * gs;
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&rfree[p & 1]);
                }
            }
        }
        // after an abort, let every copy still in flight land before the CTA exits (bounded)
        if (lane == 0 && *abort_flag) {
            for (int b = 0; b < 2; ++b) {
                if (s_used[b]) mbar_wait_bounded(&sfull[b], s_par[b], a.err_word);
                if (x_used[b]) mbar_wait_bounded(&xfull[b], x_par[b], a.err_word);
            }
        }
        return;
    }

    // ---------------------------------------------------------------- compute warps
    const int ks = warp % KS, rgl = warp / KS;
    const int h = lane >> 4;
    const int lrow = rgl * 16 + (lane & 15);              // row of the lane inside the task
    const int col0 = ks * KTW * kTileK + h * 32;          // first column of the lane's slice and half
    const int nch = (KTW + kChunk - 1) / kChunk, n_last = KTW - (nch - 1) * kChunk;
    // the lane's bytes of a task's first code tile: tile (e, rt, ks * KTW), half h, row lrow
    const uint32_t lane_off = (uint32_t)(ks * KTW) * kTileCodeBytes + (uint32_t)h * 2048u + (uint32_t)lrow * 16u;
    auto task_codes = [&](const Cursor &c) -> const uint8_t * {
        const int row0 = c.sub << rt_log2;
        return a.codes + (size_t)((tab[c.li] * RT + (row0 >> 7)) * KT) * kTileCodeBytes + lane_off +
               (uint32_t)(row0 & (kTileRows - 1)) * 16u;
    };
    // The warp's code stream: the (task, pass, chunk) sequence it consumes, kRing - 1
    // chunks ahead. Each lane copies and later reads only its own 16-byte pieces, so a
    // lane's cp.async.wait_group is all the synchronisation the ring needs.
    const uint32_t ring = smem_u32(base + lay.ring) + (uint32_t)(warp * kRing * kChunk * 32 + lane) * 16u;
    Cursor pc{};                                          // task of the next chunk of the stream
    bool pvalid = false;
    int pt0 = 0, pm = 0, pleft = nch;                     // its first token, rows, chunks left in the pass
    uint32_t fill = 0;
    const uint8_t *pg = nullptr;                          // next chunk of the stream (this lane's bytes)
    {
        Cursor ft;
        if (first_pass(ft)) {
            int rb;
            pc = ft;
            pvalid = true;
            pm = task_rows(ft, rb);
            pg = task_codes(ft);
        }
    }
    auto refill = [&]() {
        if (pvalid) {
            const uint32_t d = ring + fill;
            if (pleft > 1 || n_last == kChunk) {
                cp_async16<0, 0>(d, pg);
                cp_async16<512, kTileCodeBytes>(d, pg);
                cp_async16<1024, 2 * kTileCodeBytes>(d, pg);
                cp_async16<1536, 3 * kTileCodeBytes>(d, pg);
            } else {
                cp_async16<0, 0>(d, pg);
                if (n_last > 1) cp_async16<512, kTileCodeBytes>(d, pg);
                if (n_last > 2) cp_async16<1024, 2 * kTileCodeBytes>(d, pg);
            }
            pg += kChunk * kTileCodeBytes;
            if (--pleft == 0) {
                pleft = nch;
                if (pt0 + kMaxNT < pm) {                  // same task, next tokens
                    pt0 += kMaxNT;
                    pg -= (size_t)nch * kChunk * kTileCodeBytes;
                } else {
                    Cursor nc;
                    int nt0;
                    if (next_pass(pc, pt0, pm, nc, nt0)) {
                        int rb;
                        pc = nc;
                        pt0 = 0;
                        pm = task_rows(nc, rb);
                        pg = task_codes(nc);
                    } else {
                        pvalid = false;
                    }
                }
            }
        }
        cp_async_commit();
        fill = next_slot(fill);
    };
    const bool has_work = pvalid;
    for (int i = 0; i < kRing - 1; ++i) refill();
    // weights only so far; the bounded waits below start after the gate/up grid is done
    if (P == Proj::Down && has_work) grid_dep_wait();
    // forced-timeout test: one thread of CTA 0 waits a short time on a barrier that nothing
    // completes, then takes the timeout path (error word, abort flag) like any other wait
    if (a.test_wait_ns && blockIdx.x == 0 && warp == 0) {
        if (lane == 0) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait_sleep(never, 0u)) {
                if (global_timer_ns() - t0 > a.test_wait_ns) {
                    atomicOr(a.err_word, DEV_ERR_WAIT_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
            }
        }
        __syncwarp();
    }

    uint32_t use = 0;
    int p = 0, tn = 0;
    const uint32_t sc_step = (uint32_t)rows_task * 4u, hsh = (uint32_t)h * 16u;
    const uint32_t x_tok = (uint32_t)K * 2u, xi_tok = (uint32_t)(K / 16) * 4u;
    // this lane's addresses in buffer 0 of each double buffer; buffer 1 is one size further
    const uint32_t sm0 = smem_u32(base);
    const uint32_t sc0 = sm0 + (uint32_t)lay.sc + (uint32_t)((ks * KTW) * rows_task + lrow) * 4u;
    const uint32_t x0 = sm0 + (uint32_t)lay.x + (uint32_t)col0 * 2u;
    const uint32_t xi0 = sm0 + (uint32_t)lay.xi + (uint32_t)(col0 / 16) * 4u;
    const uint32_t red0 = sm0 + (uint32_t)lay.red + (uint32_t)(ks * rows_task + lrow) * (kMaxNT * 4u);
    const uint32_t bar0 = smem_u32(bars);                 // sfull, xfull, full, rfree: 2 each, 8 bytes apart
    for (Cursor c = c0; c.id < n_tasks; advance(c)) {
        int r_begin;
        const int m = task_rows(c, r_begin);
        if (m <= 0) continue;
        const int sb = tn & 1;
        const uint32_t sc = sc0 + (uint32_t)sb * (uint32_t)lay.sc_sz;
        wait_or_abort(bar0 + 8u * sb, (tn >> 1) & 1, abort_flag, a.err_word);
        for (int t0 = 0; t0 < m; t0 += kMaxNT, ++p) {
            const int xb = p & 1;
            wait_or_abort(bar0 + 16u + 8u * xb, (p >> 1) & 1, abort_flag, a.err_word);
            const uint32_t xa = x0 + (uint32_t)xb * (uint32_t)lay.x_sz;
            const uint32_t xia = xi0 + (uint32_t)xb * (uint32_t)lay.xi_sz;
            float acc[kMaxNT] = {};
            if (m - t0 == 1)
                pass_run<1>(ring, use, nch, n_last, sc, sc_step, hsh, xa, xa + x_tok, xia, xia + xi_tok, acc, refill);
            else
                pass_run<2>(ring, use, nch, n_last, sc, sc_step, hsh, xa, xa + x_tok, xia, xia + xi_tok, acc, refill);
#pragma unroll
            for (int t = 0; t < kMaxNT; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 16);
            // the control warp has consumed what pass p-2 left in this buffer
            if (p >= 2) wait_or_abort(bar0 + 48u + 8u * xb, ((p - 2) >> 1) & 1, abort_flag, a.err_word);
            if (h == 0) sts_f32x2(red0 + (uint32_t)xb * (uint32_t)lay.red_sz, acc[0], acc[1]);
            __syncwarp();
            if (lane == 0) mbar_arrive_at(bar0 + 32u + 8u * xb);
        }
        ++tn;
    }
    cp_async_wait<0>();   // copies of the empty tail groups: nothing may be in flight at exit
}

template <Proj P>
int gemv_grid(int K, Geometry g, int num_sms) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_kernel<P>, kThreads, gemv_smem_bytes(K, g)) !=
            cudaSuccess || per_sm < 1)
        per_sm = 1;
    return per_sm * num_sms;
}

struct GemvShape {
    CUtensorMap map;   // the scales, box = one task's rows x all column tiles
    Geometry g;
    int grid;
    size_t smem;
};
struct GemvMaps {
    GemvShape gu[2], down[2];   // [0] default, [1] long
};

// The shape for a batch of T tokens: long when the GEMV list (at most min(E, T k)
// experts) gives each CTA kLongTasksPerCta long tasks.
const GemvShape &pick_shape(const Layer &L, const GemvShape (&sh)[2], int R, int T) {
    const int experts = min(expert_slots(L), T * token_slots(L));
    const long long tasks = (long long)experts * (R / (16 * sh[1].g.RG));
    return (sh[1].g.KS != sh[0].g.KS && tasks >= (long long)kLongTasksPerCta * sh[1].grid) ? sh[1] : sh[0];
}

}  // namespace

cudaError_t gemv_setup(Layer &L)
{
    const int H = L.desc.hidden, I = L.desc.intermediate, E = expert_slots(L);
    GemvMaps *gm = new (std::nothrow) GemvMaps();
    if (!gm) return cudaErrorMemoryAllocation;
    gm->gu[0].g = geometry(true, H);
    gm->gu[1].g = geometry_from(kGateUpLongKS, H);
    gm->down[0].g = geometry(false, I);
    gm->down[1].g = geometry_from(kDownLongKS, I);
    // scale slabs viewed as [E * RT * KT][128 rows] of u32; a task's box is 16*RG rows x all KT slabs
    const uint64_t slabs_gu = (uint64_t)E * (2 * I / kTileRows) * (H / kTileK);
    const uint64_t slabs_d = (uint64_t)E * (H / kTileRows) * (I / kTileK);
    for (int v = 0; v < 2; ++v) {
        if (encode_tensor_map_2d(&gm->gu[v].map, CU_TENSOR_MAP_DATA_TYPE_UINT32, L.w.gu_scales, kTileRows, slabs_gu,
                                 kTileScaleBytes, 16 * gm->gu[v].g.RG, H / kTileK,
                                 CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS ||
            encode_tensor_map_2d(&gm->down[v].map, CU_TENSOR_MAP_DATA_TYPE_UINT32, L.w.d_scales, kTileRows, slabs_d,
                                 kTileScaleBytes, 16 * gm->down[v].g.RG, I / kTileK,
                                 CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS) {
            delete gm;
            return cudaErrorInvalidValue;
        }
        gm->gu[v].smem = gemv_smem_bytes(H, gm->gu[v].g);
        gm->down[v].smem = gemv_smem_bytes(I, gm->down[v].g);
    }
    L.gemv_maps = gm;
    // The attribute belongs to the kernel, not to this handle: every handle of the process
    // launches the same two kernels with its own shared-memory size. So it is raised to the
    // device's limit once and never lowered (a handle with a smaller layer created later
    // must not shrink it under an earlier, larger one).
    int optin = 0;
    cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, L.device);
    if (e != cudaSuccess) return e;
    if (std::max(gm->gu[0].smem, gm->gu[1].smem) > (size_t)optin ||
        std::max(gm->down[0].smem, gm->down[1].smem) > (size_t)optin)
        return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(gemv_kernel<Proj::GateUp>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gemv_kernel<Proj::Down>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e != cudaSuccess) return e;
    for (int v = 0; v < 2; ++v) {
        gm->gu[v].grid = gemv_grid<Proj::GateUp>(H, gm->gu[v].g, L.num_sms);
        gm->down[v].grid = gemv_grid<Proj::Down>(I, gm->down[v].g, L.num_sms);
    }
    return cudaSuccess;
}

void gemv_teardown(Layer &L)
{
    delete static_cast<GemvMaps *>(L.gemv_maps);
    L.gemv_maps = nullptr;
}

static GemvArgs common_args(const Layer &L) {
    GemvArgs g{};
    g.expert_list = L.ws.gemv_list; g.list_size = L.ws.list_sizes;
    g.offsets = L.ws.offsets; g.perm = L.ws.perm; g.top_k = token_slots(L);
    g.I = L.desc.intermediate; g.err_word = L.ws.err_word;
    g.test_wait_ns = 0;
    return g;
}

cudaError_t launch_gemv_gate_up(Layer &L, const uint16_t *x, int T, cudaStream_t s, int *launches)
{
    (void)x;   // the routing kernels left x in block-scaled f16 form in ws.xq
    StageTimer timer(L, TFMOE_STAGE_GEMV_GATE_UP, s);
    const GemvMaps *gm = static_cast<const GemvMaps *>(L.gemv_maps);
    GemvArgs g = common_args(L);
    g.codes = L.w.gu_codes;
    g.glob0 = L.w.gate_global; g.glob1 = L.w.up_global;
    g.R = 2 * L.desc.intermediate; g.K = L.desc.hidden;
    const GemvShape &sh = pick_shape(L, gm->gu, g.R, T);
    g.KS = sh.g.KS; g.RG = sh.g.RG;
    g.src = L.ws.xq; g.src_inv = L.ws.xq_inv;
    g.act_out = L.ws.act; g.aq_out = L.ws.aq; g.aq_inv_out = L.ws.aq_inv;
    if (L.desc.flags & TFMOE_FLAG_TEST_TIMEOUT) g.test_wait_ns = kTestWaitNs;
    // a plain launch: as a programmatic dependent of the routing kernel it measured slower
    // (decode T=8 61.3 -> 62.9 us, T=1 24.6 -> 24.9 us)
    gemv_kernel<Proj::GateUp><<<sh.grid, kThreads, sh.smem, s>>>(sh.map, g);
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_gemv_down(Layer &L, int T, cudaStream_t s, int *launches)
{
    StageTimer timer(L, TFMOE_STAGE_GEMV_DOWN, s);
    const GemvMaps *gm = static_cast<const GemvMaps *>(L.gemv_maps);
    GemvArgs d = common_args(L);
    d.codes = L.w.d_codes;
    d.glob0 = L.w.down_global; d.glob1 = nullptr;
    d.R = L.desc.hidden; d.K = L.desc.intermediate;
    const GemvShape &sh = pick_shape(L, gm->down, d.R, T);
    d.KS = sh.g.KS; d.RG = sh.g.RG;
    d.src = L.ws.aq; d.src_inv = L.ws.aq_inv;
    d.y_out = L.ws.y;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(sh.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = sh.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = L.plain_order ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_kernel<Proj::Down>, sh.map, d);
    *launches += 1;
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_gemv(Layer &L, const uint16_t *x, int T, cudaStream_t s, int *launches)
{
    cudaError_t e = launch_gemv_gate_up(L, x, T, s, launches);
    if (e == cudaSuccess) e = launch_gemv_down(L, T, s, launches);
    return e;
}

}  // namespace tfmoe
