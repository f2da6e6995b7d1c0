// common.cuh -- small device helpers shared by the libtfmoe kernels (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace tfmoe {

// Device error word bits (workspace int32, read by tfmoe_sync_status).
enum : int32_t {
    DEV_ERR_BAD_EXPERT = 1,     // an expert id outside [0, E)
    DEV_ERR_BAD_ROW = 2,        // a permuted row outside [0, P)
    DEV_ERR_WAIT_TIMEOUT = 4,   // a bounded mbarrier wait gave up
    DEV_ERR_NONFINITE = 8,      // a non-finite router logit
};

// Upper bound on one mbarrier wait, in nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte streaming load that bypasses L1 (weights are read once per task).
__device__ __forceinline__ uint4 ldg_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// The barrier operations by 32-bit shared address (the *_at forms) and by pointer.
__device__ __forceinline__ void mbar_arrive_at(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) { mbar_arrive_at(smem_u32(bar)); }
__device__ __forceinline__ bool mbar_try_wait_at(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    return mbar_try_wait_at(smem_u32(bar), parity);
}
// As mbar_try_wait, but a thread whose phase is not complete is suspended (up to
// kSuspendHintNs) instead of returning at once, so waiting warps do not take issue
// slots from the warps doing the work.
constexpr uint32_t kSuspendHintNs = 20000;
__device__ __forceinline__ bool mbar_try_wait_sleep_at(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity), "r"(kSuspendHintNs) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity) {
    return mbar_try_wait_sleep_at(smem_u32(bar), parity);
}
// Programmatic dependent launch. A grid launched with programmatic stream
// serialisation may start once every CTA of the grid before it has called
// launch_dependents (or exited); grid_dep_wait returns when that grid has completed
// and its memory is visible. Both are no-ops for a grid launched normally.
__device__ __forceinline__ void grid_dep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bounded wait: returns false (and sets the error word) when the limit passes.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, int32_t *err_word) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        for (int i = 0; i < 4; ++i)
            if (mbar_try_wait_sleep(bar, parity)) return true;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            if (err_word) atomicOr(err_word, DEV_ERR_WAIT_TIMEOUT);
            return false;
        }
    }
}

// 1-D bulk copy global -> shared, completing on an mbarrier (tx bytes).
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(smem_dst)), "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// 2-D tensor copy global -> shared (box given by the tensor map), completing on an
// mbarrier. The innermost coordinate times the element size must be a multiple of 16.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------- formats
// Two E2M1 codes (one byte: element 2i low nibble, 2i+1 high nibble) -> f16x2.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    uint32_t out;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(out) : "r"(byte));
    return out;
}
// Eight E2M1 codes (one 32-bit word; byte i holds elements 2i (low nibble) and 2i+1)
// -> four f16x2. Unpacking the word into byte registers lets each conversion read its
// byte directly (about one instruction per pair instead of shift, mask and convert).
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t (&o)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]) : "r"(w));
}
// Two E4M3 bytes (low byte first) -> f16x2 (exact: every E4M3 value is an f16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
    uint32_t out;
    uint16_t in = static_cast<uint16_t>(two_bytes);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(out) : "h"(in));
    return out;
}
__device__ __forceinline__ float2 f16x2_to_float2(uint32_t h2) {
    __half2 h = *reinterpret_cast<__half2 *>(&h2);
    return __half22float2(h);
}
__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}
__device__ __forceinline__ uint16_t float_to_bf16_bits_rn(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t *>(&b);
}

// Sixteen bf16 values -> f16 values times 2^sh, sh chosen from the block's largest
// exponent so that the largest magnitude lands in [2^14, 2^15). Every bf16 element
// within 2^28 of the block's largest is then an exact f16 (its 8-bit significand stays
// above the f16 normal range); returns 2^-sh. src and dst 16-byte aligned.
__device__ __forceinline__ float block16_bf16_to_f16(const uint16_t *src, uint16_t *dst) {
    const uint4 v0 = *reinterpret_cast<const uint4 *>(src);
    const uint4 v1 = *reinterpret_cast<const uint4 *>(src + 8);
    const uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t emax = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) emax = max(emax, max((u[j] >> 7) & 0xFFu, (u[j] >> 23) & 0xFFu));
    int sh = 14 - ((int)emax - 127);
    sh = max(-120, min(120, sh));
    const float up = __int_as_float((127 + sh) << 23);
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const __half lo = __float2half_rn(bf16_bits_to_float(u[j] & 0xFFFFu) * up);
        const __half hi = __float2half_rn(bf16_bits_to_float(u[j] >> 16) * up);
        o[j] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
    }
    *reinterpret_cast<uint4 *>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4 *>(dst + 8) = make_uint4(o[4], o[5], o[6], o[7]);
    return __int_as_float((127 - sh) << 23);
}

// z * sigmoid(z); exp and reciprocal each one special-function-unit instruction
// (relative errors of a few ulp of fp32, far below the bf16 rounding that follows).
// Large -z gives 1 / inf = 0.
__device__ __forceinline__ float rcp_approx(float v) {
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}
__device__ __forceinline__ float silu_f32(float z) { return z * rcp_approx(1.0f + __expf(-z)); }

}  // namespace tfmoe
