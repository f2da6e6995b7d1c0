// combine.cu -- weighted un-permute and accumulate of the expert outputs:
// out[t,h] = bf16_rn( sum over slots s = 0..k-1, in slot order, of
//                     g[t,s] * y[row of pair (t,s)][h] ).
// This is the weighted-combine half of the add_moe_norm step that closes the
// MoE chain in TensorFold issue #627 (per-launch kernel table); the residual
// add and the norm are not part of this layer.
#include "common.cuh"
#include "internal.h"


namespace tfmoe {
namespace {

// One thread per 8 consecutive outputs of one token: 2 x 16-byte loads of y
// per slot, one 16-byte store of bf16.
__global__ void __launch_bounds__(256) combine_kernel(
    const float *__restrict__ y, const float *__restrict__ g, const int32_t *__restrict__ inv,
    uint16_t *__restrict__ out, int T, int H, int k, int P, int32_t *err_word, int debug)
{
    // launched as a programmatic dependent of the down projection: y is final past this wait
    grid_dep_wait();
    const int per_token = H / 8;
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (size_t)T * per_token) return;
    const int t = (int)(i / per_token), h = (int)(i % per_token) * 8;
    float acc[8];
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
    uint4 o;
    o.x = (uint32_t)float_to_bf16_bits_rn(acc[0]) | ((uint32_t)float_to_bf16_bits_rn(acc[1]) << 16);
    o.y = (uint32_t)float_to_bf16_bits_rn(acc[2]) | ((uint32_t)float_to_bf16_bits_rn(acc[3]) << 16);
    o.z = (uint32_t)float_to_bf16_bits_rn(acc[4]) | ((uint32_t)float_to_bf16_bits_rn(acc[5]) << 16);
    o.w = (uint32_t)float_to_bf16_bits_rn(acc[6]) | ((uint32_t)float_to_bf16_bits_rn(acc[7]) << 16);
    *reinterpret_cast<uint4 *>(out + (size_t)t * H + h) = o;
}

}  // namespace

cudaError_t launch_combine(Layer &L, int T, uint16_t *out, cudaStream_t s, int *launches)
{
    StageTimer timer(L, TFMOE_STAGE_COMBINE, s);
    const int H = L.desc.hidden, k = L.desc.top_k;
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
    const cudaError_t e = cudaLaunchKernelEx(&cfg, combine_kernel, (const float *)L.ws.y, (const float *)L.ws.topk_w,
                                             (const int32_t *)L.ws.inv, out, T, H, k, T * k, L.ws.err_word, debug);
    *launches += 1;
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace tfmoe
