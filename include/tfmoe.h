/*
 * tfmoe.h -- C ABI of libtfmoe: the forward pass of one mixture-of-experts FFN
 * layer with NVFP4 weights and BF16 activations (W4A16) on one NVIDIA B200
 * (sm_100a).
 *
 * What the layer computes (the operation every entry point below serves):
 *
 *   logits[t,e] = fp32( sum_h x[t,h] * Wr[e,h] ) (+ bias[e])        router
 *   ids[t,0..k) = the k largest logits, ties to the lower expert index
 *   g[t,s]      = softmax over the k selected logits                 weights
 *   G = fp32(x . deq(Wgate_e)), U = fp32(x . deq(Wup_e))              per routed pair
 *   a = bf16( silu(G) * U )                                           SwiGLU
 *   y = a . deq(Wdown_e)^T                                            down projection
 *   out[t,h] = bf16( sum_s g[t,s] * y_s[h] )                          weighted combine
 *
 * Optional steps on either side of the routed path (tfmoe_forward_add_norm):
 *   y_sh = the shared expert, an FFN of the same form and formats with width Is,
 *          that every token passes through with weight 1, added into the combine;
 *   out  = bf16( sum_s g[t,s] * y_s + y_sh + residual )               residual add
 *   out_norm = bf16( out * gamma / sqrt(mean_h(out^2) + eps) )         RMS norm
 *
 *   deq(W)[r,c] = E2M1(code[r,c]) * E4M3(scale[r, c/16]) * global
 *
 * Passages this follows:
 *  - W4A16, i.e. 4-bit-float weights with attached scales computed against
 *    BF16 inputs rather than as all-FP4 arithmetic: TensorFold 1.0.12
 *    GLM-5.3-Flash post, section "NVFP4 is neither uniform 4-bit nor all-FP4
 *    compute".
 *  - Only the routed experts' weights are read per token; decode streams
 *    those weights, prefill is one large matrix multiply: DGX Spark GB10
 *    bandwidth-budget page, section "Mechanism: decode is bandwidth-bound,
 *    prefill is compute-bound".
 *  - The chain router -> top-k -> plan -> routed experts -> weighted combine:
 *    TensorFold issue #627, comment "Where the 0.35 ms per step goes" and
 *    the per-launch kernel table (router, topk, add_moe_norm).
 *  - The shared expert beside the routed ones, and the combine fused with the
 *    residual add and the norm (add_moe_norm): the same comment and table.
 *    The pages do not spell out their arithmetic; this library takes the
 *    readings stated at tfmoe_forward_add_norm.
 *  - E2M1 and E4M3 bit layouts: OCP Microscaling (MX) format definitions.
 *
 * Threading: handles are not thread-safe; use one handle per host thread or
 * serialise. tfmoe_last_error() is thread-local.
 */
#ifndef TFMOE_H
#define TFMOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TFMOE_API __attribute__((visibility("default")))
#else
#define TFMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TFMOE_OK = 0,
    TFMOE_ERR_INVALID_ARG = 1,   /* a null pointer, a size out of range, T > max_tokens ... */
    TFMOE_ERR_OOM = 2,           /* device allocation failed in create / load_weights */
    TFMOE_ERR_CUDA = 3,          /* a CUDA call or kernel launch failed; see tfmoe_last_error() */
    TFMOE_ERR_NOT_LOADED = 4,    /* forward before load_weights */
    TFMOE_ERR_UNSUPPORTED = 5,   /* valid arguments the library does not handle (e.g. H % 128 != 0) */
    TFMOE_ERR_TIMEOUT = 6,       /* a bounded device-side wait gave up (reported by tfmoe_sync_status) */
    TFMOE_ERR_DEVICE = 7         /* a kernel's own check set the device error word */
} tfmoe_status;

typedef struct tfmoe_layer tfmoe_layer;   /* opaque */

/* Descriptor flags. */
#define TFMOE_FLAG_FORCE_GEMV    0x1u  /* every expert uses the CUDA-core GEMV regime */
#define TFMOE_FLAG_FORCE_MMA     0x2u  /* every expert uses the tcgen05 tensor-core regime */
#define TFMOE_FLAG_DEBUG_CHECKS  0x4u  /* kernels bounds-check ids/rows and set the error word */
/* Test aid for the failure path: in every forward that runs the GEMV gate/up kernel,
 * one thread of its first CTA waits 1 ms on a barrier that nothing completes and then
 * takes the timeout path (error word, abort). That forward's output is undefined;
 * tfmoe_sync_status reports TFMOE_ERR_TIMEOUT. Not for production use. */
#define TFMOE_FLAG_TEST_TIMEOUT  0x8u

/*
 * Layer shape. Requirements (else TFMOE_ERR_INVALID_ARG):
 *   hidden H and intermediate I positive multiples of 16; 1 <= top_k <= num_experts;
 *   max_tokens >= 1.
 * The library additionally needs H % 128 == 0, I % 64 == 0 and num_experts <= 256
 * (else TFMOE_ERR_UNSUPPORTED).
 * shared_intermediate: 0, or the shared expert's width Is, a multiple of I; the
 * library runs it as m = Is / I extra expert slots that every token takes with
 * weight 1 (needs num_experts + m <= 256 and top_k + m <= 32).
 * norm_eps: the RMS norm's epsilon (>= 0), used by tfmoe_forward_add_norm.
 */
typedef struct {
    int32_t hidden;            /* H */
    int32_t intermediate;      /* I: expert FFN width */
    int32_t num_experts;       /* E */
    int32_t top_k;             /* k */
    int32_t max_tokens;        /* the largest T tfmoe_forward will accept; sizes the workspace */
    int32_t has_router_bias;   /* 1: router_bias is read and added to the logits */
    uint32_t flags;            /* TFMOE_FLAG_* */
    int32_t gemv_max_tokens;   /* experts routed to <= this many tokens use the CUDA-core GEMV
                                  regime, the others the tcgen05 tensor-core regime;
                                  <= 0 selects the built-in crossover: every expert in the
                                  GEMV regime while T <= 16, else 2 tokens */
    int32_t shared_intermediate; /* Is: width of the shared expert, 0 = none */
    float norm_eps;            /* epsilon of the RMS norm */
} tfmoe_layer_desc;

/*
 * Weights in the canonical layout: DEVICE pointers, row-major, caller-owned,
 * read only during tfmoe_load_weights (which copies and repacks them).
 * NVFP4 element c of a row sits in byte c/2 of that row, in the low nibble
 * when c is even; one E4M3 scale byte per 16 consecutive elements of a row
 * (the reduction dimension); one fp32 multiplier per expert and projection.
 */
typedef struct {
    const uint16_t *router_w;       /* bf16 [E][H] */
    const float    *router_bias;    /* fp32 [E]; read only when has_router_bias */
    const uint8_t  *gate_codes;     /* [E][I][H/2] */
    const uint8_t  *up_codes;       /* [E][I][H/2] */
    const uint8_t  *gate_scales;    /* e4m3 [E][I][H/16] */
    const uint8_t  *up_scales;      /* e4m3 [E][I][H/16] */
    const float    *gate_global;    /* [E] */
    const float    *up_global;      /* [E] */
    const uint8_t  *down_codes;     /* [E][H][I/2] */
    const uint8_t  *down_scales;    /* e4m3 [E][H][I/16] */
    const float    *down_global;    /* [E] */
    /* The shared expert, read only when shared_intermediate > 0 (same formats): */
    const uint8_t  *shared_gate_codes;   /* [Is][H/2] */
    const uint8_t  *shared_up_codes;     /* [Is][H/2] */
    const uint8_t  *shared_gate_scales;  /* e4m3 [Is][H/16] */
    const uint8_t  *shared_up_scales;    /* e4m3 [Is][H/16] */
    const float    *shared_gate_global;  /* [1] */
    const float    *shared_up_global;    /* [1] */
    const uint8_t  *shared_down_codes;   /* [H][Is/2] */
    const uint8_t  *shared_down_scales;  /* e4m3 [H][Is/16] */
    const float    *shared_down_global;  /* [1] */
} tfmoe_weights;

/* Create a layer handle on the current CUDA device and allocate its
 * workspace (sized by max_tokens) and weight storage. On error *out is NULL
 * and nothing stays allocated. */
TFMOE_API tfmoe_status tfmoe_create(const tfmoe_layer_desc *desc, tfmoe_layer **out);

/* Copy the caller's canonical weights into library-owned device memory,
 * repacked into the tiled kernel layout (row tiles of 128, K tiles of 64,
 * gate and up rows interleaved). Synchronous: returns after the copy is
 * complete; the caller may free its tensors afterwards. May be called again
 * to replace the weights. */
TFMOE_API tfmoe_status tfmoe_load_weights(tfmoe_layer *layer, const tfmoe_weights *w);

/*
 * out[T][H] = layer(x[T][H]); x and out are DEVICE pointers to bf16, rows of
 * H contiguous elements, caller-owned; out must not overlap x.
 * Stream-ordered on `cuda_stream` (a cudaStream_t; NULL = legacy default
 * stream): returns after enqueueing, never synchronises the host, never
 * allocates, and reads no device value on the host, so it may be captured
 * in a CUDA graph. 0 <= T <= max_tokens; T == 0 launches nothing. One handle
 * has one workspace: do not run two forwards of the same handle
 * concurrently on different streams.
 * Argument errors return before anything is enqueued. Launch errors return
 * TFMOE_ERR_CUDA; faults inside kernels surface at the next synchronisation
 * (for example tfmoe_sync_status).
 */
TFMOE_API tfmoe_status tfmoe_forward(tfmoe_layer *layer, const uint16_t *x, int32_t T,
                           uint16_t *out, void *cuda_stream);

/*
 * The layer followed by the residual add and the RMS norm, fused into the
 * combine (the add_moe_norm step of TensorFold issue #627's per-launch table):
 *   out[t,h]      = bf16( sum_s g[t,s] y_s[t,h] + y_sh[t,h] + residual[t,h] )
 *   out_norm[t,h] = bf16( out[t,h] * norm_w[h] / sqrt(mean_h out[t,h]^2 + eps) )
 * with y_sh the shared expert (when the descriptor has one) and eps the
 * descriptor's norm_eps. Readings of the pages: the shared expert rounds its
 * SwiGLU output to bf16 like a routed expert; the residual joins the same sum,
 * rounded once; the norm reads the rounded out (the new residual stream).
 * DEVICE pointers, bf16 bits, 16-byte aligned, caller-owned: residual [T][H] or
 * NULL (no add); norm_w [H] or NULL (no norm: out_norm is not written and may
 * be NULL); out [T][H]; out_norm [T][H]. residual may be the same array as out
 * (the residual stream updated in place); otherwise none of x, residual, out
 * and out_norm may overlap. Everything else as tfmoe_forward.
 */
TFMOE_API tfmoe_status tfmoe_forward_add_norm(tfmoe_layer *layer, const uint16_t *x, int32_t T,
                                              const uint16_t *residual, const uint16_t *norm_w,
                                              uint16_t *out, uint16_t *out_norm, void *cuda_stream);

/*
 * Same computation with HOST buffers: x_host[T][H] is copied to the
 * device, the layer runs, and the result is copied into out_host[T][H];
 * all on `cuda_stream`, and the call returns after the result has arrived
 * in out_host. Page-locked host buffers make the copies asynchronous to other
 * host work; pageable buffers work too.
 */
TFMOE_API tfmoe_status tfmoe_forward_host(tfmoe_layer *layer, const uint16_t *x_host, int32_t T,
                                uint16_t *out_host, void *cuda_stream);

/* Synchronise `cuda_stream`, then report a pending CUDA error or the device
 * error word that kernels with TFMOE_FLAG_DEBUG_CHECKS set (and clear it). */
TFMOE_API tfmoe_status tfmoe_sync_status(tfmoe_layer *layer, void *cuda_stream);

/* Free everything the handle owns. NULL is accepted. Synchronises the device. */
TFMOE_API void tfmoe_destroy(tfmoe_layer *layer);

/* Message of the last failing call on this host thread ("" if none). */
TFMOE_API const char *tfmoe_last_error(void);

/*
 * Intermediate buffers of the last forward, for inspection (tests, tools).
 * Returns a DEVICE pointer into the handle's workspace and its size in
 * bytes; contents are valid after the forward has completed on its stream.
 * Layouts (P = T*(k+m) pairs, m the shared expert's slots (0 without one), rows
 * of the permuted order r = 0..P-1, grouped by expert slot in ascending
 * (slot, token, token's slot) order):
 */
typedef enum {
    TFMOE_BUF_LOGITS = 0,     /* fp32 [T][E] router logits (bias included). For T <= 16 every
                                 entry is the exact logit. For T > 16 the entries of every
                                 expert that could be in the token's top k -- the k selected
                                 ones included -- are exact; the others hold the tensor-core
                                 approximation, within (H + 34) 2^-22 ||x_t|| ||w_e|| +
                                 2^-21 |bias_e| of the exact value. */
    TFMOE_BUF_TOPK_IDS = 1,   /* int32 [T][k+m] selected experts, slot 0 = largest logit; with a
                                 shared expert of m = Is/I slots, slots k..k+m-1 hold the
                                 shared slots E..E+m-1 */
    TFMOE_BUF_TOPK_WEIGHTS = 2, /* fp32 [T][k+m] softmax weights over the selected logits
                                   (1 in the shared slots) */
    TFMOE_BUF_EXPERT_COUNTS = 3, /* int32 [E+m] tokens routed to each expert slot */
    TFMOE_BUF_EXPERT_OFFSETS = 4, /* int32 [E+m+1] exclusive prefix sum of the counts */
    TFMOE_BUF_PERM = 5,       /* int32 [P] pair index t*k+s held by permuted row r */
    TFMOE_BUF_INV = 6,        /* int32 [P] permuted row of pair t*k+s */
    TFMOE_BUF_ACT = 7,        /* bf16 [P][I] SwiGLU output a, permuted rows */
    TFMOE_BUF_EXPERT_OUT = 8, /* fp32 [P][H] down-projection output y, permuted rows */
    TFMOE_BUF_REGIME = 9      /* int32 [E+m] 0 = not routed, 1 = GEMV regime, 2 = MMA regime */
} tfmoe_buffer;

TFMOE_API tfmoe_status tfmoe_get_buffer(tfmoe_layer *layer, tfmoe_buffer which, void **dev_ptr, size_t *bytes);

/* Number of kernel launches the last tfmoe_forward enqueued. */
TFMOE_API int32_t tfmoe_last_launch_count(tfmoe_layer *layer);

/*
 * Per-stage timing. While enabled, tfmoe_forward records a CUDA event pair on
 * its stream around each stage below and, before returning, waits for the
 * last one and adds the elapsed times to per-stage totals (so a profiled
 * forward blocks the host and must not be graph-captured). tfmoe_profile_read
 * copies the totals (milliseconds) and per-stage call counts into arrays of
 * TFMOE_STAGE_COUNT entries and, if reset != 0, zeroes them.
 */
typedef enum {
    TFMOE_STAGE_ROUTER = 0,       /* router logits */
    TFMOE_STAGE_TOPK = 1,         /* top-k + softmax weights */
    TFMOE_STAGE_PERMUTE = 2,      /* per-expert counts, offsets, permutation, regimes */
    TFMOE_STAGE_GEMV_GATE_UP = 3, /* GEMV regime: gate/up projections + SwiGLU */
    TFMOE_STAGE_GEMV_DOWN = 4,    /* GEMV regime: down projection */
    TFMOE_STAGE_MMA_GATE_UP = 5,  /* tensor-core regime: gate/up projections + SwiGLU */
    TFMOE_STAGE_MMA_DOWN = 6,     /* tensor-core regime: down projection */
    TFMOE_STAGE_COMBINE = 7,      /* weighted combine (+ residual add and norm in tfmoe_forward_add_norm) */
    TFMOE_STAGE_GATHER = 8,       /* tensor-core regime: activation row gather */
    TFMOE_STAGE_COUNT = 9
} tfmoe_stage;

/*
 * Re-enqueue the kernels of one stage of the last tfmoe_forward on this
 * handle, reading the workspace that forward left (routing, plan,
 * intermediates) and rewriting that stage's outputs; a measurement aid for
 * timing one kernel in isolation. T must equal the last forward's T and x
 * must be its input (read by the gate/up stages); out receives the combine
 * stage's result (the plain weighted combine, also after a
 * tfmoe_forward_add_norm: no residual, no norm). Supported stages: GEMV_GATE_UP, GEMV_DOWN, MMA_GATE_UP,
 * MMA_DOWN, GATHER, COMBINE (others return TFMOE_ERR_UNSUPPORTED); a stage
 * whose kernels the forward did not use enqueues nothing. Stage kernels are
 * launched in plain stream order (tfmoe_forward lets the down projection and
 * the combine start early, as programmatic dependents of the kernel before
 * them), so back-to-back replays of one stage do not overlap.
 */
TFMOE_API tfmoe_status tfmoe_forward_stage(tfmoe_layer *layer, int32_t stage, const uint16_t *x, int32_t T,
                                           uint16_t *out, void *cuda_stream);

TFMOE_API tfmoe_status tfmoe_profile_enable(tfmoe_layer *layer, int32_t enable);
TFMOE_API tfmoe_status tfmoe_profile_read(tfmoe_layer *layer, float *ms_total, int32_t *calls, int32_t reset);

/*
 * Routing without any allocation (the pages describe no such entry point;
 * it exists for callers of this library that cannot allocate device memory:
 * code running while another component owns the whole memory budget through a
 * fixed pool, real-time loops that must not pay cudaMalloc's latency or its
 * implicit device synchronisation, and hosts whose rules forbid allocating
 * after start-up). It computes what tfmoe_forward computes for routing -- the
 * router logits (fp64-accumulated, rounded to fp32, plus the optional bias),
 * the top_k expert ids (ties to the lower index) and the softmax weights over
 * the selected logits -- without a tfmoe_layer handle and without calling
 * cudaMalloc, cudaFree or any allocating routine.
 *
 * The fp32 logits live in a fixed scratch array compiled into the library:
 * TFMOE_ROUTE_NOALLOC_MAX_LOGITS floats (4 MiB) on every GPU that loads it,
 * held until the process exits. T * num_experts above that limit returns
 * TFMOE_ERR_INVALID_ARG and launches nothing; split the batch instead.
 * Every call on a device shares that one array and leaves its logits in it:
 * calls whose work overlaps on the GPU (two streams, or two host threads)
 * race on it and must be serialised by the caller. Each call overwrites every
 * logit it reads, so nothing needs clearing between calls.
 * Each call made outside a stream capture looks up the array's device address
 * in the current CUDA context (so a device reset, which may move the array,
 * or another context on the device is followed); a call made during a capture
 * uses the address found by the last uncaptured call in the same context and
 * returns TFMOE_ERR_CUDA if there is none.
 *
 * Arguments (DEVICE pointers, caller-owned): x bf16 [T][hidden] and router_w
 * bf16 [num_experts][hidden], both 16-byte aligned; router_bias fp32
 * [num_experts] or NULL; outputs ids_out int32 [T][top_k] and weights_out fp32
 * [T][top_k]. hidden must be a positive multiple of 32, 1 <= top_k <= 32,
 * top_k <= num_experts <= 256. Stream-ordered on cuda_stream; T == 0 is a no-op.
 */
#define TFMOE_ROUTE_NOALLOC_MAX_LOGITS (1 << 20)
TFMOE_API tfmoe_status tfmoe_route_noalloc(const uint16_t *x, int32_t T, int32_t hidden,
                                           const uint16_t *router_w, const float *router_bias,
                                           int32_t num_experts, int32_t top_k,
                                           int32_t *ids_out, float *weights_out, void *cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* TFMOE_H */
