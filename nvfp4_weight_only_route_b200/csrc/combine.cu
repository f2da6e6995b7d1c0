// combine.cu -- weighted un-permute and accumulate of the expert outputs:
// out[t,h] = bf16_rn( sum over slots s = 0..k+m-1, in slot order, of
//                     g[t,s] * y[row of pair (t,s)][h]  (+ residual[t,h]) ),
// the shared expert's m slots last with g = 1; and, for tfmoe_forward_add_norm, the RMS
// norm of out. This is the add_moe_norm step that closes the MoE chain in TensorFold
// issue #627 (per-launch kernel table).
#include "common.cuh"
#include "internal.h"


namespace tfmoe {
namespace {

// The fp32 sum of 8 consecutive outputs h..h+7 of token t over its k slots (slot order),
// plus the residual's values when given.
__device__ __forceinline__ void combine8(const float *__restrict__ y, const float *__restrict__ g,
                                         const int32_t *__restrict__ inv, const uint16_t *residual, int t, int h,
                                         int H, int k, int P, int32_t *err_word, int debug, float (&acc)[8])
{
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    for (int s = 0; s < k; ++s) {
        const int r = inv[(size_t)t * k + s];
        if (debug && (r < 0 || r >= P)) { atomicOr(err_word, DEV_ERR_BAD_ROW); continue; }
        const float gw = g[(size_t)t * k + s];
        const float4 a = *reinterpret_cast<const float4 *>(y + (size_t)r * H + h);
        const float4 b = *reinterpret_cast<const float4 *>(y + (size_t)r * H + h + 4);
        acc[0] = fmaf(gw, a.x, acc[0]); acc[1] = fmaf(gw, a.y, acc[1]);
        acc[2] = fmaf(gw, a.z, acc[2]); acc[3] = fmaf(gw, a.w, acc[3]);
        acc[4] = fmaf(gw, b.x, acc[4]); acc[5] = fmaf(gw, b.y, acc[5]);
        acc[6] = fmaf(gw, b.z, acc[6]); acc[7] = fmaf(gw, b.w, acc[7]);
    }
    if (residual) {
        const uint4 rv = *reinterpret_cast<const uint4 *>(residual + (size_t)t * H + h);
        const uint32_t ru[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            acc[2 * q] += bf16_bits_to_float(ru[q] & 0xFFFFu);
            acc[2 * q + 1] += bf16_bits_to_float(ru[q] >> 16);
        }
    }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float (&acc)[8]) {
    uint4 o;
    o.x = (uint32_t)float_to_bf16_bits_rn(acc[0]) | ((uint32_t)float_to_bf16_bits_rn(acc[1]) << 16);
    o.y = (uint32_t)float_to_bf16_bits_rn(acc[2]) | ((uint32_t)float_to_bf16_bits_rn(acc[3]) << 16);
    o.z = (uint32_t)float_to_bf16_bits_rn(acc[4]) | ((uint32_t)float_to_bf16_bits_rn(acc[5]) << 16);
    o.w = (uint32_t)float_to_bf16_bits_rn(acc[6]) | ((uint32_t)float_to_bf16_bits_rn(acc[7]) << 16);
    return o;
}

// One thread per 8 consecutive outputs of one token: 2 x 16-byte loads of y
// per slot, one 16-byte store of bf16.
__global__ void __launch_bounds__(256) combine_kernel(
    const float *__restrict__ y, const float *__restrict__ g, const int32_t *__restrict__ inv,
    const uint16_t *residual, uint16_t *out, int T, int H, int k, int P, int32_t *err_word, int debug)
{
    // launched as a programmatic dependent of the down projection: y is final past this wait
    grid_dep_wait();
    const int per_token = H / 8;
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (size_t)T * per_token) return;
    const int t = (int)(i / per_token), h = (int)(i % per_token) * 8;
    float acc[8];
    combine8(y, g, inv, residual, t, h, H, k, P, err_word, debug, acc);
    *reinterpret_cast<uint4 *>(out + (size_t)t * H + h) = pack_bf16x8(acc);
}

// Correctly rounded fp64 -> bf16 (nearest, ties to even): round to fp32 toward zero and
// make the result odd when that step was inexact ("round to odd"), then round that fp32
// to bf16. fp32 keeps 16 more significand bits than bf16, so the second rounding sees the
// true position of the value between its two bf16 neighbours (Boldo and Melquiond's
// round-to-odd method).
__device__ __forceinline__ uint16_t double_to_bf16_bits_rn(double d) {
    float f = __double2float_rz(d);
    if ((double)f != d && f == f) f = __uint_as_float(__float_as_uint(f) | 1u);
    return float_to_bf16_bits_rn(f);
}

// One CTA per token: the combine (as combine_kernel) into out, kept in shared memory; the
// fp64 sum of squares of the rounded row; then out_norm = bf16(out * gamma * r) with
// r = 1 / sqrt(sum / H + eps), the products in fp64.
constexpr int kNormThreads = 256;
__global__ void __launch_bounds__(kNormThreads) combine_norm_kernel(
    const float *__restrict__ y, const float *__restrict__ g, const int32_t *__restrict__ inv,
    const uint16_t *residual, const uint16_t *__restrict__ gamma, uint16_t *out, uint16_t *__restrict__ out_norm,
    int H, int k, int P, double eps, int32_t *err_word, int debug)
{
    __shared__ uint4 row_s[kMaxReduction / 8];
    __shared__ double part[kNormThreads / 32];
    grid_dep_wait();
    const int t = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    double ss = 0.0;
    for (int c = threadIdx.x; c < H / 8; c += kNormThreads) {
        float acc[8];
        combine8(y, g, inv, residual, t, c * 8, H, k, P, err_word, debug, acc);
        const uint4 o = pack_bf16x8(acc);
        *reinterpret_cast<uint4 *>(out + (size_t)t * H + c * 8) = o;
        row_s[c] = o;
        const uint32_t u[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const double lo = bf16_bits_to_float(u[q] & 0xFFFFu), hi = bf16_bits_to_float(u[q] >> 16);
            ss = fma(lo, lo, ss);
            ss = fma(hi, hi, ss);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) part[warp] = ss;
    __syncthreads();
    double tot = 0.0;
#pragma unroll
    for (int w = 0; w < kNormThreads / 32; ++w) tot += part[w];
    const double r = 1.0 / sqrt(tot / (double)H + eps);
    for (int c = threadIdx.x; c < H / 8; c += kNormThreads) {
        const uint4 o = row_s[c];
        const uint4 gv = *reinterpret_cast<const uint4 *>(gamma + c * 8);
        const uint32_t u[4] = {o.x, o.y, o.z, o.w}, gu[4] = {gv.x, gv.y, gv.z, gv.w};
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const double lo = (double)bf16_bits_to_float(u[q] & 0xFFFFu) * r * (double)bf16_bits_to_float(gu[q] & 0xFFFFu);
            const double hi = (double)bf16_bits_to_float(u[q] >> 16) * r * (double)bf16_bits_to_float(gu[q] >> 16);
            w[q] = (uint32_t)double_to_bf16_bits_rn(lo) | ((uint32_t)double_to_bf16_bits_rn(hi) << 16);
        }
        *reinterpret_cast<uint4 *>(out_norm + (size_t)t * H + c * 8) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace

cudaError_t launch_combine(Layer &L, int T, uint16_t *out, cudaStream_t s, int *launches, const uint16_t *residual,
                           const uint16_t *norm_w, uint16_t *out_norm)
{
    StageTimer timer(L, TFMOE_STAGE_COMBINE, s);
    const int H = L.desc.hidden, k = token_slots(L);
    const size_t n = (size_t)T * (H / 8);
    const int debug = (L.desc.flags & TFMOE_FLAG_DEBUG_CHECKS) ? 1 : 0;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((n + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = L.plain_order ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (norm_w) {
        cfg.gridDim = dim3((unsigned)T);
        cfg.blockDim = dim3(kNormThreads);
        e = cudaLaunchKernelEx(&cfg, combine_norm_kernel, (const float *)L.ws.y, (const float *)L.ws.topk_w,
                               (const int32_t *)L.ws.inv, residual, norm_w, out, out_norm, H, k, T * k,
                               (double)L.desc.norm_eps, L.ws.err_word, debug);
    } else {
        e = cudaLaunchKernelEx(&cfg, combine_kernel, (const float *)L.ws.y, (const float *)L.ws.topk_w,
                               (const int32_t *)L.ws.inv, residual, out, T, H, k, T * k, L.ws.err_word, debug);
    }
    *launches += 1;
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace tfmoe
