// api.cu -- the C ABI of libtfmoe (declared in include/tfmoe.h): argument
// validation, device memory ownership, and the stream-ordered launch chain
// router -> top-k -> permute -> expert projections -> combine.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>

#include "common.cuh"
#include "internal.h"

using namespace tfmoe;

struct tfmoe_layer {
    Layer impl;
};

namespace {

thread_local std::string g_last_error;

tfmoe_status fail(tfmoe_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
tfmoe_status fail(tfmoe_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

tfmoe_status ok() { g_last_error.clear(); return TFMOE_OK; }

tfmoe_status cuda_fail(cudaError_t e, const char *where) {
    return fail(e == cudaErrorMemoryAllocation ? TFMOE_ERR_OOM : TFMOE_ERR_CUDA, "%s: %s (%s)", where,
                cudaGetErrorName(e), cudaGetErrorString(e));
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Lays out `n` sub-buffers in one block; returns the total size.
struct Carver {
    size_t off = 0;
    template <class T>
    size_t take(T **slot, size_t count, uint8_t *base) {
        off = align_up(off, 256);
        if (base) *slot = reinterpret_cast<T *>(base + off);
        const size_t at = off;
        off += sizeof(T) * count;
        return at;
    }
};

void carve_workspace(Layer &L, uint8_t *base, size_t *total) {
    // E: expert slots (routed + shared), k: slots per token; the logits cover the routed experts
    const size_t T = L.desc.max_tokens, E = expert_slots(L), k = token_slots(L);
    const size_t H = L.desc.hidden, I = L.desc.intermediate, P = T * k;
    Workspace &w = L.ws;
    Carver c;
    c.take(&w.logits, T * L.desc.num_experts, base);
    c.take(&w.xnorm, T, base);
    c.take(&w.xexp, T, base);
    c.take(&w.cand_cnt, T, base);
    c.take(&w.cand, T * kRouterMaxCand, base);
    c.take(&w.ids, P, base);
    c.take(&w.topk_w, P, base);
    c.take(&w.counts, E, base);
    c.take(&w.offsets, E + 1, base);
    c.take(&w.perm, P, base);
    c.take(&w.inv, P, base);
    c.take(&w.regime, E, base);
    c.take(&w.gemv_list, E, base);
    c.take(&w.mma_list, E, base);
    c.take(&w.list_sizes, 4, base);
    c.take(&w.err_word, 1, base);
    c.take(&w.route_counter, 1, base);
    c.take(&w.seg_cnt, ((T + 7) / 8) * E, base);
    c.take(&w.seg_base, ((T + 7) / 8) * E, base);
    c.take(&w.plan_tot, E, base);
    c.take(&w.plan_counter, 1, base);
    c.take(&w.mma_entries, 4 * max_mma_entries(P, E), base);
    c.take(&w.x_perm, P * H, base);
    c.take(&w.row_inv, P, base);
    c.take(&w.act, P * I, base);
    c.take(&w.xq, T * H, base);
    c.take(&w.xq_inv, T * H / 16, base);
    c.take(&w.aq, P * I, base);
    c.take(&w.aq_inv, P * I / 16, base);
    c.take(&w.y, P * H, base);
    c.take(&w.x_stage, T * H, base);
    c.take(&w.out_stage, T * H, base);
    *total = align_up(c.off, 256);
}

void carve_weights(Layer &L, uint8_t *base, size_t *total) {
    const size_t E = expert_slots(L), ER = L.desc.num_experts, H = L.desc.hidden, I = L.desc.intermediate;
    Weights &w = L.w;
    Carver c;
    c.take(&w.router_w, ER * H, base);
    c.take(&w.router_cst, ER, base);
    c.take(&w.router_wexp, 2, base);
    c.take(&w.router_bias, ER, base);
    c.take(&w.gu_codes, E * 2 * I * H / 2, base);
    c.take(&w.gu_scales, E * 2 * I * H / 16, base);
    c.take(&w.d_codes, E * H * I / 2, base);
    c.take(&w.d_scales, E * H * I / 16, base);
    c.take(&w.gate_global, E, base);
    c.take(&w.up_global, E, base);
    c.take(&w.down_global, E, base);
    *total = align_up(c.off, 256);
}

struct DeviceGuard {
    int prev = -1;
    bool changed = false;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) changed = (cudaSetDevice(dev) == cudaSuccess);
    }
    ~DeviceGuard() { if (changed) cudaSetDevice(prev); }
};

}  // namespace

namespace tfmoe {
tfmoe_status record_error(tfmoe_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}
tfmoe_status record_ok() { return ok(); }
}  // namespace tfmoe

extern "C" {

const char *tfmoe_last_error(void) { return g_last_error.c_str(); }

tfmoe_status tfmoe_create(const tfmoe_layer_desc *desc, tfmoe_layer **out)
{
    if (!out) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_create: out is NULL");
    *out = nullptr;
    if (!desc) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_create: desc is NULL");
    const tfmoe_layer_desc d = *desc;
    if (d.hidden <= 0 || d.intermediate <= 0 || d.hidden % 16 || d.intermediate % 16)
        return fail(TFMOE_ERR_INVALID_ARG, "hidden (%d) and intermediate (%d) must be positive multiples of 16",
                    d.hidden, d.intermediate);
    if (d.num_experts <= 0 || d.top_k <= 0 || d.top_k > d.num_experts)
        return fail(TFMOE_ERR_INVALID_ARG, "need 1 <= top_k (%d) <= num_experts (%d)", d.top_k, d.num_experts);
    if (d.max_tokens <= 0) return fail(TFMOE_ERR_INVALID_ARG, "max_tokens (%d) must be >= 1", d.max_tokens);
    if ((d.flags & TFMOE_FLAG_FORCE_GEMV) && (d.flags & TFMOE_FLAG_FORCE_MMA))
        return fail(TFMOE_ERR_INVALID_ARG, "FORCE_GEMV and FORCE_MMA are exclusive");
    if (d.flags & ~(TFMOE_FLAG_FORCE_GEMV | TFMOE_FLAG_FORCE_MMA | TFMOE_FLAG_DEBUG_CHECKS | TFMOE_FLAG_TEST_TIMEOUT))
        return fail(TFMOE_ERR_INVALID_ARG, "unknown flag bits 0x%x", d.flags);
    if (d.hidden % 128 || d.intermediate % 64)
        return fail(TFMOE_ERR_UNSUPPORTED, "libtfmoe needs hidden %% 128 == 0 and intermediate %% 64 == 0 (got %d, %d)",
                    d.hidden, d.intermediate);
    if (d.hidden > kMaxReduction || d.intermediate > kMaxReduction)
        return fail(TFMOE_ERR_UNSUPPORTED, "libtfmoe supports hidden and intermediate up to %d (got %d, %d)",
                    kMaxReduction, d.hidden, d.intermediate);
    if (d.shared_intermediate < 0 || d.shared_intermediate % d.intermediate)
        return fail(TFMOE_ERR_INVALID_ARG, "shared_intermediate (%d) must be 0 or a multiple of intermediate (%d)",
                    d.shared_intermediate, d.intermediate);
    if (!(d.norm_eps >= 0.f) || d.norm_eps == __builtin_inff())
        return fail(TFMOE_ERR_INVALID_ARG, "norm_eps must be finite and >= 0");
    const long long m = d.shared_intermediate / d.intermediate;
    if (d.num_experts + m > 256 || d.top_k + m > 32)
        return fail(TFMOE_ERR_UNSUPPORTED, "libtfmoe supports num_experts + m <= 256 and top_k + m <= 32 "
                    "(m = shared_intermediate / intermediate = %lld)", m);
    const long long kx = d.top_k + m;
    if ((long long)d.max_tokens * kx > (1LL << 30))
        return fail(TFMOE_ERR_UNSUPPORTED, "max_tokens * (top_k + m) too large");
    if ((long long)d.max_tokens * kx * (d.hidden > d.intermediate ? d.hidden : d.intermediate) >= (1LL << 32))
        return fail(TFMOE_ERR_UNSUPPORTED, "max_tokens * (top_k + m) * max(hidden, intermediate) must stay below 2^32");

    const char *fail_env = getenv("TFMOE_FAIL_ALLOC");
    if (fail_env && atoi(fail_env) != 0)
        return fail(TFMOE_ERR_OOM, "tfmoe_create: allocation failure injected by TFMOE_FAIL_ALLOC");

    tfmoe_layer *h = new (std::nothrow) tfmoe_layer();
    if (!h) return fail(TFMOE_ERR_OOM, "tfmoe_create: host allocation failed");
    Layer &L = h->impl;
    L.desc = d;
    L.gemv_max_tokens = d.gemv_max_tokens;
    cudaError_t e = cudaGetDevice(&L.device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&L.num_sms, cudaDevAttrMultiProcessorCount, L.device);
    if (e != cudaSuccess) { delete h; return cuda_fail(e, "tfmoe_create: device query"); }

    carve_workspace(L, nullptr, &L.ws_bytes);
    carve_weights(L, nullptr, &L.w_bytes);
    e = cudaMalloc(&L.ws_block, L.ws_bytes);
    if (e == cudaSuccess) e = cudaMalloc(&L.w_block, L.w_bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        if (L.ws_block) cudaFree(L.ws_block);
        delete h;
        return cuda_fail(e, "tfmoe_create: cudaMalloc");
    }
    carve_workspace(L, static_cast<uint8_t *>(L.ws_block), &L.ws_bytes);
    carve_weights(L, static_cast<uint8_t *>(L.w_block), &L.w_bytes);
    e = cudaMemset(L.ws.err_word, 0, sizeof(int32_t));
    if (e == cudaSuccess) e = cudaMemset(L.ws.route_counter, 0, sizeof(int32_t));
    if (e == cudaSuccess) e = cudaMemset(L.ws.plan_counter, 0, sizeof(int32_t));
    if (e == cudaSuccess) e = gemv_setup(L);
    if (e == cudaSuccess) e = mma_setup(L);
    if (e == cudaSuccess) e = router_setup(L);
    if (e != cudaSuccess) {
        router_teardown(L);
        mma_teardown(L);
        gemv_teardown(L);
        cudaFree(L.ws_block);
        cudaFree(L.w_block);
        delete h;
        return cuda_fail(e, "tfmoe_create: setup");
    }
    *out = h;
    return ok();
}

tfmoe_status tfmoe_load_weights(tfmoe_layer *layer, const tfmoe_weights *w)
{
    if (!layer || !w) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_load_weights: NULL argument");
    Layer &L = layer->impl;
    const void *req[] = {w->router_w, w->gate_codes, w->up_codes, w->gate_scales, w->up_scales, w->gate_global,
                         w->up_global, w->down_codes, w->down_scales, w->down_global};
    for (const void *p : req)
        if (!p) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_load_weights: a required weight pointer is NULL");
    if (L.desc.has_router_bias && !w->router_bias)
        return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_load_weights: has_router_bias but router_bias is NULL");
    const void *vec[] = {w->router_w, w->gate_codes, w->up_codes, w->down_codes};
    for (const void *p : vec)
        if (!aligned16(p)) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_load_weights: codes/router must be 16-byte aligned");
    const void *sc[] = {w->gate_scales, w->up_scales, w->down_scales};
    for (const void *p : sc)
        if (reinterpret_cast<uintptr_t>(p) & 3u)
            return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_load_weights: scales must be 4-byte aligned");
    const int m = shared_slots(L);
    if (m > 0) {
        const void *sh[] = {w->shared_gate_codes, w->shared_up_codes, w->shared_gate_scales, w->shared_up_scales,
                            w->shared_gate_global, w->shared_up_global, w->shared_down_codes,
                            w->shared_down_scales, w->shared_down_global};
        for (const void *p : sh)
            if (!p) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_load_weights: a shared-expert weight pointer is NULL");
        const void *shv[] = {w->shared_gate_codes, w->shared_up_codes, w->shared_down_codes};
        for (const void *p : shv)
            if (!aligned16(p))
                return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_load_weights: shared codes must be 16-byte aligned");
        const void *shs[] = {w->shared_gate_scales, w->shared_up_scales, w->shared_down_scales};
        for (const void *p : shs)
            if (reinterpret_cast<uintptr_t>(p) & 3u)
                return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_load_weights: shared scales must be 4-byte aligned");
    }

    DeviceGuard dg(L.device);
    const size_t E = L.desc.num_experts, H = L.desc.hidden;
    cudaStream_t s;
    cudaError_t e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_fail(e, "tfmoe_load_weights: stream");
    e = cudaMemcpyAsync(L.w.router_w, w->router_w, E * H * 2, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess && L.desc.has_router_bias)
        e = cudaMemcpyAsync(L.w.router_bias, w->router_bias, E * 4, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(L.w.gate_global, w->gate_global, E * 4, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(L.w.up_global, w->up_global, E * 4, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(L.w.down_global, w->down_global, E * 4, cudaMemcpyDeviceToDevice, s);
    // every shared slot carries the shared expert's per-tensor multipliers
    for (int j = 0; j < m && e == cudaSuccess; ++j) {
        e = cudaMemcpyAsync(L.w.gate_global + E + j, w->shared_gate_global, 4, cudaMemcpyDeviceToDevice, s);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(L.w.up_global + E + j, w->shared_up_global, 4, cudaMemcpyDeviceToDevice, s);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(L.w.down_global + E + j, w->shared_down_global, 4, cudaMemcpyDeviceToDevice, s);
    }
    if (e == cudaSuccess) e = launch_repack(L, *w, s);
    if (e == cudaSuccess) e = launch_router_norms(L, s);
    cudaError_t e2 = cudaStreamSynchronize(s);
    cudaStreamDestroy(s);
    if (e == cudaSuccess) e = e2;
    if (e != cudaSuccess) { L.loaded = false; return cuda_fail(e, "tfmoe_load_weights"); }
    L.loaded = true;
    return ok();
}

}  // extern "C"

namespace {

bool overlap(const void *a, const void *b, size_t bytes) {
    if (!a || !b) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + bytes && y < x + bytes;
}

// The forward chain; residual, norm_w and out_norm are the optional epilogue (see
// tfmoe_forward_add_norm), all NULL for tfmoe_forward.
tfmoe_status forward_impl(tfmoe_layer *layer, const char *who, const uint16_t *x, int32_t T,
                          const uint16_t *residual, const uint16_t *norm_w, uint16_t *out, uint16_t *out_norm,
                          void *cuda_stream)
{
    if (!layer) return fail(TFMOE_ERR_INVALID_ARG, "%s: layer is NULL", who);
    Layer &L = layer->impl;
    L.last_launches = 0;
    if (!L.loaded) return fail(TFMOE_ERR_NOT_LOADED, "%s: weights not loaded", who);
    if (T < 0 || T > L.desc.max_tokens)
        return fail(TFMOE_ERR_INVALID_ARG, "%s: T=%d outside [0, max_tokens=%d]", who, T, L.desc.max_tokens);
    if (T == 0) return ok();
    if (!x || !out) return fail(TFMOE_ERR_INVALID_ARG, "%s: x or out is NULL", who);
    if (norm_w && !out_norm) return fail(TFMOE_ERR_INVALID_ARG, "%s: norm_w given but out_norm is NULL", who);
    if (!norm_w) out_norm = nullptr;
    if (!aligned16(x) || !aligned16(out) || !aligned16(residual) || !aligned16(norm_w) || !aligned16(out_norm))
        return fail(TFMOE_ERR_INVALID_ARG, "%s: x, out, residual, norm_w and out_norm must be 16-byte aligned", who);
    const size_t bytes = (size_t)T * L.desc.hidden * 2;
    if (overlap(x, out, bytes) || overlap(x, out_norm, bytes) || overlap(out, out_norm, bytes) ||
        overlap(residual, out_norm, bytes) || overlap(residual, x, bytes) ||
        (residual != out && overlap(residual, out, bytes)))
        return fail(TFMOE_ERR_INVALID_ARG, "%s: overlapping x / residual / out / out_norm (only residual == out "
                    "is allowed)", who);

    DeviceGuard dg(L.device);
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    int n = 0;
    // An expert holds at most T tokens, so with T <= the GEMV threshold no expert can be
    // in the MMA regime and its launches are skipped (likewise under the FORCE flags).
    const bool use_mma = !(L.desc.flags & TFMOE_FLAG_FORCE_GEMV) &&
                         ((L.desc.flags & TFMOE_FLAG_FORCE_MMA) || T > gemv_threshold(L, T));
    const bool use_gemv = !(L.desc.flags & TFMOE_FLAG_FORCE_MMA);
    L.mma_small = mma_use_small_tiles(L, T);
    cudaError_t e = launch_router(L, x, T, s, &n);
    if (e == cudaSuccess) e = launch_permute(L, T, s, &n);
    if (e == cudaSuccess && use_mma) e = launch_gather(L, x, T, s, &n);
    if (e == cudaSuccess && use_mma) e = launch_mma_gate_up(L, s, &n);
    if (e == cudaSuccess && use_gemv) e = launch_gemv_gate_up(L, x, T, s, &n);
    if (e == cudaSuccess && use_mma) e = launch_mma_down(L, s, &n);
    if (e == cudaSuccess && use_gemv) e = launch_gemv_down(L, T, s, &n);
    if (e == cudaSuccess) e = launch_combine(L, T, out, s, &n, residual, norm_w, out_norm);
    L.last_use_mma = use_mma;
    L.last_use_gemv = use_gemv;
    L.last_launches = n;
    if (e != cudaSuccess) return cuda_fail(e, who);
    L.last_T = T;
    if (L.profiling) {
        e = cudaStreamSynchronize(s);
        for (int st = 0; st < TFMOE_STAGE_COUNT && e == cudaSuccess; ++st) {
            if (!L.prof_used[st]) continue;
            float ms = 0.f;
            e = cudaEventElapsedTime(&ms, L.prof_ev[st][0], L.prof_ev[st][1]);
            L.prof_ms[st] += ms;
            L.prof_calls[st] += 1;
            L.prof_used[st] = false;
        }
        if (e != cudaSuccess) return cuda_fail(e, "profiling events");
    }
    return ok();
}

}  // namespace

extern "C" {

tfmoe_status tfmoe_forward(tfmoe_layer *layer, const uint16_t *x, int32_t T, uint16_t *out, void *cuda_stream)
{
    return forward_impl(layer, "tfmoe_forward", x, T, nullptr, nullptr, out, nullptr, cuda_stream);
}

tfmoe_status tfmoe_forward_add_norm(tfmoe_layer *layer, const uint16_t *x, int32_t T, const uint16_t *residual,
                                    const uint16_t *norm_w, uint16_t *out, uint16_t *out_norm, void *cuda_stream)
{
    return forward_impl(layer, "tfmoe_forward_add_norm", x, T, residual, norm_w, out, out_norm, cuda_stream);
}

tfmoe_status tfmoe_forward_host(tfmoe_layer *layer, const uint16_t *x_host, int32_t T, uint16_t *out_host,
                                void *cuda_stream)
{
    if (!layer) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_forward_host: layer is NULL");
    Layer &L = layer->impl;
    if (!L.loaded) return fail(TFMOE_ERR_NOT_LOADED, "tfmoe_forward_host: weights not loaded");
    if (T < 0 || T > L.desc.max_tokens)
        return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_forward_host: T=%d outside [0, max_tokens=%d]", T, L.desc.max_tokens);
    if (T == 0) { L.last_launches = 0; return ok(); }
    if (!x_host || !out_host) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_forward_host: NULL buffer");
    DeviceGuard dg(L.device);
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    const size_t bytes = (size_t)T * L.desc.hidden * 2;
    cudaError_t e = cudaMemcpyAsync(L.ws.x_stage, x_host, bytes, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "tfmoe_forward_host: copy in");
    tfmoe_status st = tfmoe_forward(layer, L.ws.x_stage, T, L.ws.out_stage, cuda_stream);
    if (st != TFMOE_OK) return st;
    e = cudaMemcpyAsync(out_host, L.ws.out_stage, bytes, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "tfmoe_forward_host: copy out");
    return ok();
}

tfmoe_status tfmoe_sync_status(tfmoe_layer *layer, void *cuda_stream)
{
    if (!layer) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_sync_status: layer is NULL");
    Layer &L = layer->impl;
    DeviceGuard dg(L.device);
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream));
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "tfmoe_sync_status");
    int32_t word = 0;
    e = cudaMemcpy(&word, L.ws.err_word, sizeof word, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && word != 0) e = cudaMemset(L.ws.err_word, 0, sizeof(int32_t));
    if (e != cudaSuccess) return cuda_fail(e, "tfmoe_sync_status: error word");
    if (word & DEV_ERR_WAIT_TIMEOUT) return fail(TFMOE_ERR_TIMEOUT, "a device-side wait timed out (word 0x%x)", word);
    if (word) return fail(TFMOE_ERR_DEVICE, "device error word 0x%x (1 bad expert id, 2 bad row, 8 non-finite logit)", word);
    return ok();
}

void tfmoe_destroy(tfmoe_layer *layer)
{
    if (!layer) return;
    Layer &L = layer->impl;
    {
        DeviceGuard dg(L.device);
        for (auto &pair : L.prof_ev)
            for (auto &ev : pair)
                if (ev) cudaEventDestroy(ev);
        if (L.ws_block) cudaFree(L.ws_block);
        if (L.w_block) cudaFree(L.w_block);
        router_teardown(L);
        mma_teardown(L);
        gemv_teardown(L);
    }
    delete layer;
}

tfmoe_status tfmoe_get_buffer(tfmoe_layer *layer, tfmoe_buffer which, void **dev_ptr, size_t *bytes)
{
    if (!layer || !dev_ptr || !bytes) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_get_buffer: NULL argument");
    Layer &L = layer->impl;
    const size_t T = L.desc.max_tokens, E = expert_slots(L), k = token_slots(L);
    const size_t H = L.desc.hidden, I = L.desc.intermediate, P = T * k;
    switch (which) {
    case TFMOE_BUF_LOGITS: *dev_ptr = L.ws.logits; *bytes = T * L.desc.num_experts * 4; break;
    case TFMOE_BUF_TOPK_IDS: *dev_ptr = L.ws.ids; *bytes = P * 4; break;
    case TFMOE_BUF_TOPK_WEIGHTS: *dev_ptr = L.ws.topk_w; *bytes = P * 4; break;
    case TFMOE_BUF_EXPERT_COUNTS: *dev_ptr = L.ws.counts; *bytes = E * 4; break;
    case TFMOE_BUF_EXPERT_OFFSETS: *dev_ptr = L.ws.offsets; *bytes = (E + 1) * 4; break;
    case TFMOE_BUF_PERM: *dev_ptr = L.ws.perm; *bytes = P * 4; break;
    case TFMOE_BUF_INV: *dev_ptr = L.ws.inv; *bytes = P * 4; break;
    case TFMOE_BUF_ACT: *dev_ptr = L.ws.act; *bytes = P * I * 2; break;
    case TFMOE_BUF_EXPERT_OUT: *dev_ptr = L.ws.y; *bytes = P * H * 4; break;
    case TFMOE_BUF_REGIME: *dev_ptr = L.ws.regime; *bytes = E * 4; break;
    default: return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_get_buffer: unknown buffer %d", (int)which);
    }
    return ok();
}

int32_t tfmoe_last_launch_count(tfmoe_layer *layer) { return layer ? layer->impl.last_launches : 0; }

tfmoe_status tfmoe_forward_stage(tfmoe_layer *layer, int32_t stage, const uint16_t *x, int32_t T, uint16_t *out,
                                 void *cuda_stream)
{
    if (!layer) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_forward_stage: layer is NULL");
    Layer &L = layer->impl;
    if (!L.loaded) return fail(TFMOE_ERR_NOT_LOADED, "tfmoe_forward_stage: weights not loaded");
    if (T <= 0 || T != L.last_T)
        return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_forward_stage: T=%d must equal the last forward's T=%d", T, L.last_T);
    DeviceGuard dg(L.device);
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    int n = 0;
    cudaError_t e = cudaSuccess;
    struct PlainOrder {   // for this call only, whatever path it returns by
        Layer &L;
        explicit PlainOrder(Layer &l) : L(l) { L.plain_order = true; }
        ~PlainOrder() { L.plain_order = false; }
    } plain(L);
    switch (stage) {
    case TFMOE_STAGE_GEMV_GATE_UP:
        if (!x) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_forward_stage: x is NULL");
        if (L.last_use_gemv) e = launch_gemv_gate_up(L, x, T, s, &n);
        break;
    case TFMOE_STAGE_GEMV_DOWN:
        if (L.last_use_gemv) e = launch_gemv_down(L, T, s, &n);
        break;
    case TFMOE_STAGE_GATHER:
        if (!x) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_forward_stage: x is NULL");
        if (L.last_use_mma) e = launch_gather(L, x, T, s, &n);
        break;
    case TFMOE_STAGE_MMA_GATE_UP:
        if (L.last_use_mma) e = launch_mma_gate_up(L, s, &n);
        break;
    case TFMOE_STAGE_MMA_DOWN:
        if (L.last_use_mma) e = launch_mma_down(L, s, &n);
        break;
    case TFMOE_STAGE_COMBINE:
        if (!out) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_forward_stage: out is NULL");
        e = launch_combine(L, T, out, s, &n);
        break;
    default:
        return fail(TFMOE_ERR_UNSUPPORTED, "tfmoe_forward_stage: stage %d cannot be replayed", stage);
    }
    L.last_launches = n;
    if (e != cudaSuccess) return cuda_fail(e, "tfmoe_forward_stage: launch");
    return ok();
}

tfmoe_status tfmoe_profile_enable(tfmoe_layer *layer, int32_t enable)
{
    if (!layer) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_profile_enable: layer is NULL");
    Layer &L = layer->impl;
    DeviceGuard dg(L.device);
    if (enable && !L.prof_ev[0][0]) {
        for (auto &pair : L.prof_ev)
            for (auto &ev : pair) {
                cudaError_t e = cudaEventCreate(&ev);
                if (e != cudaSuccess) return cuda_fail(e, "tfmoe_profile_enable");
            }
    }
    L.profiling = enable != 0;
    return ok();
}

tfmoe_status tfmoe_profile_read(tfmoe_layer *layer, float *ms_total, int32_t *calls, int32_t reset)
{
    if (!layer || !ms_total || !calls) return fail(TFMOE_ERR_INVALID_ARG, "tfmoe_profile_read: NULL argument");
    Layer &L = layer->impl;
    for (int st = 0; st < TFMOE_STAGE_COUNT; ++st) {
        ms_total[st] = L.prof_ms[st];
        calls[st] = L.prof_calls[st];
        if (reset) { L.prof_ms[st] = 0.f; L.prof_calls[st] = 0; }
    }
    return ok();
}

}  // extern "C"
