/*
 * tfmoe_oracle.c -- plain fp64 CPU oracle for the forward pass of one
 * mixture-of-experts FFN layer with NVFP4 weights and BF16 activations
 * (W4A16).
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark load this library. The CUDA library never links,
 * includes or calls it, and the two share no source.
 *
 * What it computes, and where each step comes from:
 *
 *  - W4A16: weights are NVFP4 (4-bit floats carrying a scale), inputs stay
 *    BF16 and the arithmetic is done at higher precision, not on FP4
 *    operands [TensorFold 1.0.12 GLM-5.3-Flash post, section "NVFP4 is
 *    neither uniform 4-bit nor all-FP4 compute"].
 *  - Only the experts a token routes to are evaluated; their weights are what
 *    a decode step must stream [DGX Spark GB10 bandwidth-budget page, section
 *    "Mechanism: decode is bandwidth-bound, prefill is compute-bound"].
 *  - The per-layer sequence router -> top-k -> plan -> routed experts ->
 *    weighted combine is the MoE chain of [TensorFold issue #627, comment
 *    "Where the 0.35 ms per step goes"].
 *  - Bit layouts: E2M1 and E4M3 follow the OCP Microscaling (MX) format
 *    definitions; one E4M3 scale per 16 consecutive reduction elements and one
 *    fp32 per-tensor multiplier per (expert, projection).
 *  - The reference is 64-bit, as the error budget of [TensorFold issue #627,
 *    "Description"] is stated against a float64 reference.
 *  - Optional steps on either side of the routed path, from the same MoE
 *    chain [TensorFold issue #627, the per-launch kernel table (add_moe_norm)
 *    and "Where the 0.35 ms per step goes" (the shared expert, run beside the
 *    routed experts)]: a shared expert -- one SwiGLU FFN of width Is in the
 *    same NVFP4 formats that every token passes through with weight 1 -- the
 *    residual add, and an RMS norm of the sum. The pages name these steps but
 *    not their arithmetic; the readings taken here are: the shared expert's a
 *    is rounded to bf16 like a routed expert's; the residual (bf16) is added
 *    in the same fp64 sum as the expert outputs; the layer output (the new
 *    residual stream) is that sum rounded once to bf16; the norm reads that
 *    rounded output: out_norm = bf16_RNE( h * gamma / sqrt(mean(h^2) + eps) ).
 *
 * Rounding points (the only places precision is lost on purpose):
 *   router logit      = fp32( fp64 sum of bf16*bf16 products ) (+ fp32 bias)
 *   gate G, up U      = fp32( fp64 sum over K of x * deq(w) )
 *   a = bf16_RNE( silu(G) * U )   evaluated in fp64 from the fp32 G, U
 *   y = fp64 sum over K of a * deq(w)      (not rounded)
 *   out = bf16_RNE( sum over slots s=0..k-1 of g_s * y_s
 *                   (+ y_shared) (+ residual) )                   in fp64
 *   out_norm = bf16_RNE( out * gamma / sqrt(mean over h of out^2 + eps) )
 *   W4A4 variant (act_fp4): gate/up read NVFP4-quantised x rows and down reads
 *   NVFP4-quantised a rows (the quantiser and its reading are defined below)
 *
 * Parity pins live in the repository's CPU test-suite; every function below
 * is pinned there (format tables, a hand-worked block, closed-form chains,
 * routing invariants and a brute-force dense-equivalent computation).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

/* ------------------------------------------------------------------ */
/* Number formats                                                       */
/* ------------------------------------------------------------------ */

/* E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.
 * Exponent 0 is subnormal: 0.5 * m. Otherwise (1 + m/2) * 2^(e-1). */
double oracle_e2m1(unsigned code)
{
    unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0) ? 0.5 * (double)m : (1.0 + 0.5 * (double)m) * ldexp(1.0, (int)e - 1);
    return s ? -mag : mag;
}

/* E4M3 ("fn" variant): bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0
 * mantissa. Exponent 0 is subnormal (m/8) * 2^-6. Exponent 15 with mantissa 7
 * is NaN; there is no infinity, so the largest value is 448. */
double oracle_e4m3(unsigned byte)
{
    unsigned s = (byte >> 7) & 1u, e = (byte >> 3) & 15u, m = byte & 7u;
    if (e == 15u && m == 7u) return NAN;
    double mag = (e == 0) ? ((double)m / 8.0) * ldexp(1.0, -6)
                          : (1.0 + (double)m / 8.0) * ldexp(1.0, (int)e - 7);
    return s ? -mag : mag;
}

double oracle_bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bfloat16 (ties to even), directly from the
 * double: bf16 keeps 8 significant bits and fp32's exponent range, so the
 * quantum is 2^(e-8) for |v| in [2^(e-1), 2^e), and 2^-133 below 2^-126. */
uint16_t oracle_round_bf16(double v)
{
    if (isnan(v)) return 0x7FC0u;
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0) return sign;
    int e;
    (void)frexp(a, &e);               /* a = f * 2^e, f in [0.5, 1) */
    int q_exp = e - 8;
    if (q_exp < -133) q_exp = -133;
    double r = ldexp(rint(ldexp(a, -q_exp)), q_exp);   /* rint: nearest, ties to even */
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);
    float f = (float)r;               /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFFu));
}

/* One weight row of an NVFP4 matrix, decoded to fp64:
 * deq[c] = E2M1(code c) * E4M3(scale of block c/16) * global.
 * Element c sits in byte c/2, low nibble when c is even. */
static void dequant_row(const uint8_t *codes, const uint8_t *scales, float global, int K, double *deq)
{
    for (int c = 0; c < K; ++c) {
        uint8_t byte = codes[c / 2];
        unsigned nib = (c % 2 == 0) ? (byte & 0x0Fu) : (byte >> 4);
        deq[c] = oracle_e2m1(nib) * oracle_e4m3(scales[c / 16]) * (double)global;
    }
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* ------------------------------------------------------------------ */
/* NVFP4 activations (the W4A4 variant)                                 */
/* ------------------------------------------------------------------ */
/*
 * The pages name an all-FP4 prefill (FP4 tensor cores) beside the W4A16 path but give no
 * recipe for quantising activations. The reading taken here quantises an activation row the
 * way the weights are stored: E2M1 codes, one E4M3 scale per 16 consecutive elements, one
 * fp32 multiplier per row (per token for x, per routed pair for a), every decision in fp32:
 *   g   = fl32(amax_row / 2688)             (2688 = 6 * 448; g = 1 for an all-zero row)
 *   s_b = E4M3_RNE(min(fl32(amax_b / fl32(6 g)), 448))
 *   q_i = E2M1_RNE(fl32(v_i / fl32(s_b g)))  (saturating at +-6; 0 when s_b g = 0)
 *   deq_i = E2M1(q_i) * s_b * g             (exact in fp64)
 */

/* E2M1 code of the value nearest to v, ties to the code with an even mantissa bit,
 * saturating at +-6; the sign bit is set for every v < 0 (so tiny negatives give -0). */
unsigned oracle_e2m1_rne(double v)
{
    const double a = fabs(v);
    unsigned c;
    if (a <= 0.25) c = 0;            /* 0.25: between 0 (m=0) and 0.5 (m=1) -> 0 */
    else if (a < 0.75) c = 1;
    else if (a <= 1.25) c = 2;       /* 0.75 -> 1.0 (m=0); 1.25: 1.0 (m=0) against 1.5 (m=1) */
    else if (a < 1.75) c = 3;
    else if (a <= 2.5) c = 4;        /* 1.75 -> 2.0; 2.5: 2.0 (m=0) against 3.0 (m=1) */
    else if (a < 3.5) c = 5;
    else if (a <= 5.0) c = 6;        /* 3.5 -> 4.0; 5.0: 4.0 (m=0) against 6.0 (m=1) */
    else c = 7;                      /* up to 6 and beyond: saturate */
    return (v < 0.0 ? 8u : 0u) | c;
}

/* E4M3 byte of the value nearest to v >= 0 (ties to even), values above 448 clamped to 448.
 * The quantum is 2^(e-3) for v in [2^e, 2^(e+1)), e >= -6, and 2^-9 below 2^-6. */
unsigned oracle_e4m3_rne(double v)
{
    if (!(v > 0.0)) return 0;
    if (v >= 448.0) return 0x7Eu;
    int e;
    (void)frexp(v, &e);              /* v = f 2^e, f in [0.5, 1): leading bit 2^(e-1) */
    int q_exp = (e - 1) - 3;
    if (q_exp < -9) q_exp = -9;
    double r = ldexp(rint(ldexp(v, -q_exp)), q_exp);
    if (r > 448.0) r = 448.0;
    for (unsigned b = 0; b < 0x7Fu; ++b)
        if (oracle_e4m3(b) == r) return b;
    return 0x7Eu;                    /* not reached: every rounded value is an E4M3 value */
}

/* One activation row of K values (each exactly a float) in NVFP4, as the comment above
 * defines: codes [K] (one per byte here), scales [K/16], the row's fp32 multiplier and the
 * dequantised values [K]. */
int oracle_quant_act_row(const double *v, int32_t K, uint8_t *codes, uint8_t *scales, float *g_out, double *deq)
{
    if (!v || K <= 0 || K % 16) return 1;
    float amax = 0.0f;
    for (int i = 0; i < K; ++i) {
        const float a = fabsf((float)v[i]);
        if (a > amax) amax = a;
    }
    const float g = amax > 0.0f ? amax / 2688.0f : 1.0f;
    const float six_g = 6.0f * g;
    for (int b = 0; b < K / 16; ++b) {
        float amax_b = 0.0f;
        for (int i = 16 * b; i < 16 * b + 16; ++i) {
            const float a = fabsf((float)v[i]);
            if (a > amax_b) amax_b = a;
        }
        float ratio = amax_b / six_g;
        if (ratio > 448.0f) ratio = 448.0f;
        const unsigned sb = oracle_e4m3_rne((double)ratio);
        const double sbv = oracle_e4m3(sb);
        const float S = (float)sbv * g;
        if (scales) scales[b] = (uint8_t)sb;
        for (int i = 16 * b; i < 16 * b + 16; ++i) {
            const unsigned c = (S > 0.0f) ? oracle_e2m1_rne((double)((float)v[i] / S)) : 0u;
            if (codes) codes[i] = (uint8_t)c;
            if (deq) deq[i] = oracle_e2m1(c) * sbv * (double)g;
        }
    }
    if (g_out) *g_out = g;
    return 0;
}

/* ------------------------------------------------------------------ */
/* The layer                                                            */
/* ------------------------------------------------------------------ */

typedef struct {
    int32_t hidden, intermediate, num_experts, top_k;
    const uint16_t *router_w;      /* bf16 [E][H] */
    const float *router_bias;      /* fp32 [E] or NULL */
    const uint8_t *gate_codes, *up_codes;     /* [E][I][H/2] */
    const uint8_t *gate_scales, *up_scales;   /* [E][I][H/16] */
    const float *gate_global, *up_global;     /* [E] */
    const uint8_t *down_codes;                /* [E][H][I/2] */
    const uint8_t *down_scales;               /* [E][H][I/16] */
    const float *down_global;                 /* [E] */
    /* Shared expert: shared_intermediate = Is (0: none). */
    int32_t shared_intermediate;
    const uint8_t *sh_gate_codes, *sh_up_codes;     /* [Is][H/2] */
    const uint8_t *sh_gate_scales, *sh_up_scales;   /* [Is][H/16] */
    float sh_gate_global, sh_up_global;
    const uint8_t *sh_down_codes;                   /* [H][Is/2] */
    const uint8_t *sh_down_scales;                  /* [H][Is/16] */
    float sh_down_global;
} oracle_layer;

/* Inputs of the steps after the combine; any pointer may be NULL (step skipped). */
typedef struct {
    const uint16_t *residual;   /* bf16 [T][H], added to the layer output */
    const uint16_t *norm_w;     /* bf16 [H], gamma of the RMS norm of the layer output */
    double eps;                 /* the norm's epsilon */
    int32_t act_fp4;            /* 1: the W4A4 variant, x and a quantised to NVFP4 (routed experts) */
} oracle_epilogue;

/* Outputs. Every pointer except out may be NULL. Per-pair arrays are indexed
 * by pair = t*k + s, s the slot (0 = highest logit). */
typedef struct {
    uint16_t *out;      /* bf16 [T][H] */
    double *out64;      /* [T][H] value before the final rounding */
    double *S;          /* [T][H] sum_s g_s * sum_j |a_s[j] * deq(Wd)[h][j]| */
    float *logits;      /* [T][E] */
    int32_t *ids;       /* [T][k] */
    double *g;          /* [T][k] */
    float *G, *U;       /* [T][k][I] */
    uint16_t *a;        /* bf16 [T][k][I] */
    double *y;          /* [T][k][H] */
    double *yabs;       /* [T][k][H] sum_j |a[j] * deq(Wd)[h][j]| */
    uint16_t *out_norm; /* bf16 [T][H] RMS norm of out (needs epilogue norm_w) */
    uint16_t *a_sh;     /* bf16 [T][Is] shared expert's SwiGLU output */
    double *y_sh;       /* [T][H] shared expert's down projection */
} oracle_outputs;

/* Router logits, top-k (ties to the lower expert index) and the softmax
 * weights over the selected logits for token row x. */
static void route_token(const oracle_layer *L, const uint16_t *x, float *logits, int32_t *ids, double *g)
{
    const int H = L->hidden, E = L->num_experts, k = L->top_k;
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int h = 0; h < H; ++h)
            acc += oracle_bf16_to_double(x[h]) * oracle_bf16_to_double(L->router_w[(size_t)e * H + h]);
        float l = (float)acc;
        if (L->router_bias) l = l + L->router_bias[e];
        logits[e] = l;
    }
    char *taken = (char *)calloc((size_t)E, 1);
    for (int s = 0; s < k; ++s) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || logits[e] > logits[best])) best = e;
        ids[s] = best;
        taken[best] = 1;
    }
    free(taken);
    double lmax = (double)logits[ids[0]], den = 0.0;
    for (int s = 0; s < k; ++s) den += exp((double)logits[ids[s]] - lmax);
    for (int s = 0; s < k; ++s) g[s] = exp((double)logits[ids[s]] - lmax) / den;
}

/* The shared expert for every token: a_sh = bf16(silu(G) * U) with G, U the fp32-rounded
 * fp64 sums over H, then y_sh = the fp64 sum over Is of a_sh * deq(Wd_sh) and its absolute
 * counterpart. The same arithmetic as a routed expert, without routing. */
static void shared_expert(const oracle_layer *L, const double *xd, int32_t T, int nthreads, uint16_t *a_sh,
                          double *y_sh, double *yabs_sh)
{
    const int H = L->hidden, Is = L->shared_intermediate;
#pragma omp parallel num_threads(nthreads)
    {
        double *dg = (double *)malloc(sizeof(double) * H);
        double *du = (double *)malloc(sizeof(double) * H);
#pragma omp for schedule(static)
        for (int j = 0; j < Is; ++j) {
            dequant_row(L->sh_gate_codes + (size_t)j * (H / 2), L->sh_gate_scales + (size_t)j * (H / 16),
                        L->sh_gate_global, H, dg);
            dequant_row(L->sh_up_codes + (size_t)j * (H / 2), L->sh_up_scales + (size_t)j * (H / 16),
                        L->sh_up_global, H, du);
            for (int t = 0; t < T; ++t) {
                const double *xr = xd + (size_t)t * H;
                double sg = 0.0, su = 0.0;
                for (int h = 0; h < H; ++h) { sg += xr[h] * dg[h]; su += xr[h] * du[h]; }
                float G = (float)sg, U = (float)su;
                a_sh[(size_t)t * Is + j] = oracle_round_bf16(silu((double)G) * (double)U);
            }
        }
        free(dg);
        free(du);
    }
#pragma omp parallel num_threads(nthreads)
    {
        double *dd = (double *)malloc(sizeof(double) * Is);
#pragma omp for schedule(static)
        for (int h = 0; h < H; ++h) {
            dequant_row(L->sh_down_codes + (size_t)h * (Is / 2), L->sh_down_scales + (size_t)h * (Is / 16),
                        L->sh_down_global, Is, dd);
            for (int t = 0; t < T; ++t) {
                const uint16_t *ar = a_sh + (size_t)t * Is;
                double s = 0.0, sa = 0.0;
                for (int j = 0; j < Is; ++j) {
                    double term = oracle_bf16_to_double(ar[j]) * dd[j];
                    s += term;
                    sa += fabs(term);
                }
                y_sh[(size_t)t * H + h] = s;
                yabs_sh[(size_t)t * H + h] = sa;
            }
        }
        free(dd);
    }
}

/* RMS norm of one bf16 row: bf16_RNE( v[h] * gamma[h] / sqrt(mean(v^2) + eps) ), in fp64. */
static void rms_norm_row(const uint16_t *v, const uint16_t *gamma, int H, double eps, uint16_t *out)
{
    double ss = 0.0;
    for (int h = 0; h < H; ++h) {
        double f = oracle_bf16_to_double(v[h]);
        ss += f * f;
    }
    double r = 1.0 / sqrt(ss / (double)H + eps);
    for (int h = 0; h < H; ++h)
        out[h] = oracle_round_bf16(oracle_bf16_to_double(v[h]) * r * oracle_bf16_to_double(gamma[h]));
}

int oracle_rms_norm(const uint16_t *v, const uint16_t *gamma, int32_t T, int32_t H, double eps, uint16_t *out)
{
    if (!v || !gamma || !out || T < 0 || H <= 0) return 1;
    for (int t = 0; t < T; ++t) rms_norm_row(v + (size_t)t * H, gamma, H, eps, out + (size_t)t * H);
    return 0;
}

int oracle_forward(const oracle_layer *L, const uint16_t *x, int32_t T, int32_t nthreads,
                   const oracle_epilogue *epi, const oracle_outputs *O)
{
    if (!L || !O || T < 0) return 1;
    const int H = L->hidden, I = L->intermediate, E = L->num_experts, k = L->top_k;
    if (H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || H % 16 || I % 16) return 1;
    const int Is = L->shared_intermediate;
    if (Is < 0 || Is % 16) return 1;
    if (O->out_norm && !(epi && epi->norm_w && O->out)) return 1;
    if (T == 0) return 0;
    if (nthreads <= 0) nthreads = omp_get_max_threads();
    const size_t P = (size_t)T * k;

    float *logits = (float *)malloc(sizeof(float) * (size_t)T * E);
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * P);
    double *g = (double *)malloc(sizeof(double) * P);
    uint16_t *a = (uint16_t *)malloc(sizeof(uint16_t) * P * I);
    double *y = (double *)malloc(sizeof(double) * P * H);
    double *yabs = (double *)malloc(sizeof(double) * P * H);
    double *xd = (double *)malloc(sizeof(double) * (size_t)T * H);
    int32_t *count = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    int32_t *start = (int32_t *)malloc(sizeof(int32_t) * ((size_t)E + 1));
    int32_t *pairs = (int32_t *)malloc(sizeof(int32_t) * P);
    if (!logits || !ids || !g || !a || !y || !yabs || !xd || !count || !start || !pairs) return 2;
    uint16_t *a_sh = NULL;
    double *y_sh = NULL, *yabs_sh = NULL;
    if (Is > 0) {
        a_sh = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)T * Is);
        y_sh = (double *)malloc(sizeof(double) * (size_t)T * H);
        yabs_sh = (double *)malloc(sizeof(double) * (size_t)T * H);
        if (!a_sh || !y_sh || !yabs_sh) return 2;
    }

    /* Step 1: routing, token by token. */
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
    for (int t = 0; t < T; ++t)
        route_token(L, x + (size_t)t * H, logits + (size_t)t * E, ids + (size_t)t * k, g + (size_t)t * k);

    for (size_t i = 0; i < (size_t)T * H; ++i) xd[i] = oracle_bf16_to_double(x[i]);
    const int fp4 = epi && epi->act_fp4;
    if (fp4 && Is > 0) return 1;      /* the W4A4 variant covers the routed experts */
    if (fp4) {                        /* gate/up read the NVFP4-quantised token rows */
        double *row = (double *)malloc(sizeof(double) * H);
        if (!row) return 2;
        for (int t = 0; t < T; ++t) {
            oracle_quant_act_row(xd + (size_t)t * H, H, NULL, NULL, NULL, row);
            memcpy(xd + (size_t)t * H, row, sizeof(double) * H);
        }
        free(row);
    }

    /* Step 2: per-expert pair lists, in (token, slot) order. */
    for (size_t p = 0; p < P; ++p) count[ids[p]]++;
    start[0] = 0;
    for (int e = 0; e < E; ++e) start[e + 1] = start[e] + count[e];
    {
        int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
        for (size_t p = 0; p < P; ++p) { int e = ids[p]; pairs[start[e] + fill[e]++] = (int32_t)p; }
        free(fill);
    }

    /* Step 3: gate and up projections with the SwiGLU activation, one
     * expert at a time, rows in parallel. */
    for (int e = 0; e < E; ++e) {
        if (count[e] == 0) continue;
#pragma omp parallel num_threads(nthreads)
        {
            double *dg = (double *)malloc(sizeof(double) * H);
            double *du = (double *)malloc(sizeof(double) * H);
#pragma omp for schedule(static)
            for (int j = 0; j < I; ++j) {
                size_t row = (size_t)e * I + j;
                dequant_row(L->gate_codes + row * (H / 2), L->gate_scales + row * (H / 16), L->gate_global[e], H, dg);
                dequant_row(L->up_codes + row * (H / 2), L->up_scales + row * (H / 16), L->up_global[e], H, du);
                for (int q = start[e]; q < start[e + 1]; ++q) {
                    int p = pairs[q], t = p / k;
                    const double *xr = xd + (size_t)t * H;
                    double sg = 0.0, su = 0.0;
                    for (int h = 0; h < H; ++h) { sg += xr[h] * dg[h]; su += xr[h] * du[h]; }
                    float G = (float)sg, U = (float)su;
                    if (O->G) O->G[(size_t)p * I + j] = G;
                    if (O->U) O->U[(size_t)p * I + j] = U;
                    a[(size_t)p * I + j] = oracle_round_bf16(silu((double)G) * (double)U);
                }
            }
            free(dg);
            free(du);
        }
    }

    /* Step 4: down projection, rows in parallel; y stays in fp64. Its activation is a, or for
     * the W4A4 variant a's NVFP4-quantised rows. */
    double *ad = NULL;                /* W4A4: the dequantised NVFP4 rows of a */
    if (fp4) {
        ad = (double *)malloc(sizeof(double) * P * I);
        if (!ad) return 2;
        for (size_t i = 0; i < P * I; ++i) ad[i] = oracle_bf16_to_double(a[i]);
        double *row = (double *)malloc(sizeof(double) * I);
        if (!row) return 2;
        for (size_t p = 0; p < P; ++p) {
            oracle_quant_act_row(ad + p * I, I, NULL, NULL, NULL, row);
            memcpy(ad + p * I, row, sizeof(double) * I);
        }
        free(row);
    }
    for (int e = 0; e < E; ++e) {
        if (count[e] == 0) continue;
#pragma omp parallel num_threads(nthreads)
        {
            double *dd = (double *)malloc(sizeof(double) * I);
#pragma omp for schedule(static)
            for (int h = 0; h < H; ++h) {
                size_t row = (size_t)e * H + h;
                dequant_row(L->down_codes + row * (I / 2), L->down_scales + row * (I / 16), L->down_global[e], I, dd);
                for (int q = start[e]; q < start[e + 1]; ++q) {
                    int p = pairs[q];
                    const uint16_t *ar = a + (size_t)p * I;
                    const double *aq = ad ? ad + (size_t)p * I : NULL;
                    double s = 0.0, sa = 0.0;
                    for (int j = 0; j < I; ++j) {
                        double term = (aq ? aq[j] : oracle_bf16_to_double(ar[j])) * dd[j];
                        s += term;
                        sa += fabs(term);
                    }
                    y[(size_t)p * H + h] = s;
                    yabs[(size_t)p * H + h] = sa;
                }
            }
            free(dd);
        }
    }

    /* Step 4b: the shared expert, every token with weight 1. */
    if (Is > 0) shared_expert(L, xd, T, nthreads, a_sh, y_sh, yabs_sh);

    /* Step 5: weighted combine in slot order, then the shared expert's output and the
     * residual, in one fp64 sum rounded once to bf16. */
    const uint16_t *res = epi ? epi->residual : NULL;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int h = 0; h < H; ++h) {
            double acc = 0.0, bound = 0.0;
            for (int s = 0; s < k; ++s) {
                size_t p = (size_t)t * k + s;
                acc += g[p] * y[p * H + h];
                bound += g[p] * yabs[p * H + h];
            }
            size_t o = (size_t)t * H + h;
            if (Is > 0) {
                acc += y_sh[o];
                bound += yabs_sh[o];
            }
            if (res) acc += oracle_bf16_to_double(res[o]);
            if (O->out) O->out[o] = oracle_round_bf16(acc);
            if (O->out64) O->out64[o] = acc;
            if (O->S) O->S[o] = bound;
        }
    }

    /* Step 6: RMS norm of the rounded layer output. */
    if (O->out_norm) oracle_rms_norm(O->out, epi->norm_w, T, H, epi->eps, O->out_norm);
    if (Is > 0) {
        if (O->a_sh) memcpy(O->a_sh, a_sh, sizeof(uint16_t) * (size_t)T * Is);
        if (O->y_sh) memcpy(O->y_sh, y_sh, sizeof(double) * (size_t)T * H);
        free(a_sh); free(y_sh); free(yabs_sh);
    }

    if (O->logits) memcpy(O->logits, logits, sizeof(float) * (size_t)T * E);
    if (O->ids) memcpy(O->ids, ids, sizeof(int32_t) * P);
    if (O->g) memcpy(O->g, g, sizeof(double) * P);
    if (O->a) memcpy(O->a, a, sizeof(uint16_t) * P * I);
    if (O->y) memcpy(O->y, y, sizeof(double) * P * H);
    if (O->yabs) memcpy(O->yabs, yabs, sizeof(double) * P * H);

    free(logits); free(ids); free(g); free(a); free(y); free(yabs); free(xd); free(ad);
    free(count); free(start); free(pairs);
    return 0;
}

/* Routing alone: the router logits, top-k ids and softmax weights of every
 * token, exactly as step 1 of oracle_forward computes them (the same
 * route_token), without the expert projections. For checks of the routing of
 * batches whose full forward would take the oracle too long. */
int oracle_route(const oracle_layer *L, const uint16_t *x, int32_t T, int32_t nthreads,
                 float *logits, int32_t *ids, double *g)
{
    if (!L || T < 0 || !logits || !ids || !g) return 1;
    const int H = L->hidden, E = L->num_experts, k = L->top_k;
    if (H <= 0 || E <= 0 || k <= 0 || k > E) return 1;
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 4)
    for (int t = 0; t < T; ++t)
        route_token(L, x + (size_t)t * H, logits + (size_t)t * E, ids + (size_t)t * k, g + (size_t)t * k);
    return 0;
}

int oracle_max_threads(void) { return omp_get_max_threads(); }
