/*
 * moe_oracle.c -- CPU oracle for the gpt-oss-style MXFP4 expert-FFN MoE layer.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the package's
 * smoke check and the CPU-baseline leg of the benchmark may load this library.
 * It shares no code, header, table or helper with the CUDA path; it is a plain,
 * slow, obviously-correct restatement of what the layer computes, in double
 * precision, one element at a time.
 *
 * Sources (web pages, cited by title and section):
 *   [P2] MoE-Infinity PR #152, "expert offloading Phase 2 -- MXFP4 dequant-on-copy
 *        execution", section "Changes": mxfp4_dequantize golden test at rel-err 0.0;
 *        the native forward keeps the scales, bias, [N, K//2] packed layout, gate/up
 *        split, clamped SwiGLU and fp32 accumulation of the resident path.
 *   [P3] FreeToken PR #838, "feat(gguf): serve gpt-oss gguf checkpoints on gpt_oss":
 *        review item "NVFP4 down scale vs. down bias" (the result is sum w*(s*y + b),
 *        never sum w*s*(y + b)); review item "w2_bias with
 *        apply_router_weight_on_input" (with the router weight on the input both
 *        expert biases must be absent); section "What it does" (swiglu alpha 1.702
 *        and limit 7 are family constants; gate_up_bias [E, 2I] and down_bias [E, H];
 *        gate/up bias added before the gated activation, down bias before the
 *        routing weight; swigluoai is the uninterleaved spelling of the same math).
 *   [P5] onnxruntime/mobius PR #719, "Add native GPT-OSS MXFP4 QMoE export",
 *        sections "Summary" and "Validation": blocks [E, N, K/32, 16] (the same
 *        bytes as [E, N, K/2]); E8M0 bytes 0x00..0xfe are valid, 0xff is rejected.
 *   [P4] transformers PR #49431, "Restore GPT-OSS's router-masked expert-parallel
 *        plan": the MXFP4 experts consume routing data (ids and weights), not a
 *        dispatch of expert ids.
 *   [P3'] FreeToken PR #838, section "What it does" and the loader notes: the gpt-oss
 *        router is the module mlp.router, whose bias loads with the dense state dict.
 *   [MX] OCP Microscaling Formats (MX) v1.0: FP4 E2M1 element (1 sign, 2 exponent
 *        bits with bias 1, 1 mantissa bit, no inf/NaN) and E8M0 scale (2^(b-127),
 *        0xff = NaN).
 *   [F8] OCP 8-bit Floating Point Specification (OFP8) v1.0: the E4M3 format (1 sign,
 *        4 exponent bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 NaN,
 *        largest magnitude 448).
 *   [N4] NVFP4 as NVIDIA publishes it: blocks of 16 E2M1 elements sharing one E4M3
 *        scale, plus one fp32 scale per tensor ("weight_scale_2"); [P3] review item
 *        "NVFP4 down scale vs. down bias" fixes where that fp32 scale enters.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   R1  element kk of a packed row lives in byte kk/2; the LOW nibble holds the
 *       even element, the HIGH nibble the odd one.
 *   R2  top-k takes the k largest logits in order (value descending, ties to the
 *       lower expert index), then a softmax over those k values only.
 *   R3  gate/up rows of the fused gate_up projection are interleaved:
 *       gate = h[2i], up = h[2i+1].
 *   R4  clamped SwiGLU: g = min(gate, limit), u = clamp(up, -limit, limit),
 *       a = (u + 1) * g * sigmoid(alpha * g).
 *   R5  a 0xff scale byte decodes to NaN (the pages reject it as invalid).
 *   R6  NVFP4 experts: W[e, n, kk] = E2M1(code) * E4M3(scale[e, n, kk/16]) with the
 *       packing of R1; each projection's fp32 weight_scale_2 multiplies the expert's
 *       matrix product before its bias is added (h = s*acc + b, y = s*acc + b).  The
 *       fused gate_up bank carries two per expert (gate rows, up rows: index 0 and 1
 *       of the per-expert triple the review indexes, down being index 2).
 *   R7  the standalone NVFP4 dequant returns bf16 rounded once (nearest, ties to even)
 *       from the exact product E2M1 * E4M3 * weight_scale_2.
 *   R8  the router is a linear layer with bias: logits[t, e] = x[t] . W_r[e] + b_r[e],
 *       x and W_r bf16 [T, H] / [E, H], b_r fp32 [E] (a bf16 bias converts exactly).
 *
 * Function that is not pinned by anything outside itself: none -- every entry
 * point is checked against hand-written values, closed forms, invariants or a
 * library routine by the CPU tests.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- planted mistakes (only the non-vacuity tests set these) ---------------- */
enum {
    ORACLE_DEFECT_NONE = 0,
    ORACLE_DEFECT_NIBBLE_SWAP = 1,     /* high nibble taken as the even element      */
    ORACLE_DEFECT_E8M0_BIAS_126 = 2,   /* 2^(b-126) instead of 2^(b-127)              */
    ORACLE_DEFECT_GATE_ZERO = 3,       /* gate projection weights zeroed              */
    ORACLE_DEFECT_NO_CLAMP = 4,        /* SwiGLU without the limit clamps             */
    ORACLE_DEFECT_UNINTERLEAVED = 5,   /* gate = h[i], up = h[I + i]                  */
    ORACLE_DEFECT_DOWN_BIAS_UNWEIGHTED = 6, /* sum (w*y + b) instead of sum w*(y + b) */
    ORACLE_DEFECT_WOI_BIAS_WEIGHTED = 7,    /* router-weight-on-input: down bias scaled
                                               by the routing weight                  */
    ORACLE_DEFECT_DOWN_BIAS_IN_SCALE = 8,   /* down bias multiplied by the row's first
                                               E8M0 block scale (scale after bias)    */
    ORACLE_DEFECT_NVFP4_SCALE_AFTER_BIAS = 9, /* NVFP4: y = s*(acc + b), the mistake the
                                                 [P3] review item describes           */
    ORACLE_DEFECT_NVFP4_BLOCK32 = 10,       /* NVFP4: one scale per 32 elements (the
                                               first 16-block's scale for both halves) */
    ORACLE_DEFECT_NVFP4_GU_SCALE_SWAP = 11, /* NVFP4: gate rows take the up scale and
                                               the other way round                    */
    ORACLE_DEFECT_OPERAND_E4M3_HI_ONLY = 12, /* both projections' activation operands
                                               kept to one E4M3 term per element at a
                                               power-of-two scale per 32-element block
                                               (2^(e-7), e the exponent of the block's
                                               largest magnitude): a kernel that drops
                                               the second term of a two-term split    */
};

enum { ORACLE_FMT_MXFP4 = 0, ORACLE_FMT_NVFP4 = 1 };

enum { ORACLE_FLAG_WEIGHT_ON_INPUT = 1 };

/* ---- element formats [MX] ---------------------------------------------------- */

/* E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.
 * Exponent field 0 is subnormal: magnitude = m * 0.5. */
double oracle_e2m1_value(int code)
{
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag;
    if (e == 0)
        mag = 0.5 * (double)m;
    else
        mag = ldexp(1.0 + 0.5 * (double)m, e - 1);
    return sign ? -mag : mag;
}

/* E8M0: 2^(b - 127); 0xff is NaN (invalid per [P5] Validation; reading R5). */
double oracle_e8m0_value(int b, int defect)
{
    if (b == 255)
        return NAN;
    return ldexp(1.0, b - (defect == ORACLE_DEFECT_E8M0_BIAS_126 ? 126 : 127));
}

/* E4M3 [F8]: bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa.
 * Exponent field 0 is subnormal: magnitude = m/8 * 2^-6.  Exponent and mantissa
 * all ones is NaN (there are no infinities). */
double oracle_e4m3_value(int b)
{
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 15;
    int m = b & 7;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* double -> bfloat16 bits, round to nearest, ties to even, with subnormals
 * and overflow to infinity.  bf16 keeps 8 significant bits; the spacing of
 * representable values in [2^e, 2^(e+1)) is 2^(e-7), and below 2^-126 it is
 * the fixed subnormal spacing 2^-133. */
uint16_t oracle_double_to_bf16(double v)
{
    if (isnan(v))
        return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80);
    int e2;
    frexp(a, &e2);           /* a in [2^(e2-1), 2^e2) */
    int e = e2 - 1;
    if (e < -126)
        e = -126;
    double q = ldexp(1.0, e - 7);
    double r = nearbyint(a / q) * q; /* default rounding mode: ties to even */
    if (r >= ldexp(1.0, 128))
        return (uint16_t)(sign | 0x7F80);
    float f = (float)r;     /* exact: every bf16 value is a float */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

double oracle_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* One weight element W[e, n, kk] of a packed bank: blocks [E, N, K/2],
 * scales [E, N, K/32] ([P2] Changes: [N, K//2] layout; [P5] Summary: blocks
 * [E, N, K/32, 16]).  Reading R1 for the nibble order. */
static double weight_elem(const uint8_t *blocks, const uint8_t *scales,
                          int64_t N, int64_t K, int64_t e, int64_t n, int64_t kk,
                          int defect)
{
    int64_t row = e * N + n;
    uint8_t byte = blocks[row * (K / 2) + kk / 2];
    int even = (kk % 2) == 0;
    if (defect == ORACLE_DEFECT_NIBBLE_SWAP)
        even = !even;
    int code = even ? (byte & 0xF) : (byte >> 4);
    int s = scales[row * (K / 32) + kk / 32];
    return oracle_e2m1_value(code) * oracle_e8m0_value(s, defect);
}

/* One weight element of a packed NVFP4 bank (reading R6): blocks [E, N, K/2] with
 * the nibble order of R1, E4M3 scales [E, N, K/16], one per 16 elements [N4]. */
static double weight_elem_nvfp4(const uint8_t *blocks, const uint8_t *scales,
                                int64_t N, int64_t K, int64_t e, int64_t n, int64_t kk,
                                int defect)
{
    int64_t row = e * N + n;
    uint8_t byte = blocks[row * (K / 2) + kk / 2];
    int even = (kk % 2) == 0;
    if (defect == ORACLE_DEFECT_NIBBLE_SWAP)
        even = !even;
    int code = even ? (byte & 0xF) : (byte >> 4);
    int64_t blk = kk / 16;
    if (defect == ORACLE_DEFECT_NVFP4_BLOCK32)
        blk = (kk / 32) * 2;
    return oracle_e2m1_value(code) * oracle_e4m3_value(scales[row * (K / 16) + blk]);
}

static double weight_elem_fmt(int fmt, const uint8_t *blocks, const uint8_t *scales,
                              int64_t N, int64_t K, int64_t e, int64_t n, int64_t kk,
                              int defect)
{
    if (fmt == ORACLE_FMT_NVFP4)
        return weight_elem_nvfp4(blocks, scales, N, K, e, n, kk, defect);
    return weight_elem(blocks, scales, N, K, e, n, kk, defect);
}

/* NVFP4 dequant (reading R7): out[e, n, kk] = bf16(E2M1 * E4M3 * s2[e]), s2 = 1
 * when scale2 is NULL.  E2M1 * E4M3 has at most 6 significant bits, so the product
 * with an fp32 s2 (24 bits) is exact in double and oracle_double_to_bf16 rounds it
 * once. */
void oracle_nvfp4_dequantize(const uint8_t *blocks, const uint8_t *scales, const float *scale2,
                             uint16_t *out, int64_t E, int64_t N, int64_t K, int defect)
{
    /* rows are independent; OpenMP only spreads them over the host's cores */
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t e = 0; e < E; ++e)
        for (int64_t n = 0; n < N; ++n) {
            double s2 = scale2 ? (double)scale2[e] : 1.0;
            for (int64_t kk = 0; kk < K; ++kk)
                out[(e * N + n) * K + kk] = oracle_double_to_bf16(
                    weight_elem_nvfp4(blocks, scales, N, K, e, n, kk, defect) * s2);
        }
}

/* ---- standalone dequant-on-copy [P2] Changes ------------------------------- */
/* out[e, n, kk] = bf16(E2M1(code) * 2^(s - 127)); every value with s <= 252 is
 * exactly representable, so the golden test's rel-err 0.0 means bit-exact. */
void oracle_dequantize(const uint8_t *blocks, const uint8_t *scales, uint16_t *out,
                       int64_t E, int64_t N, int64_t K, int defect)
{
    /* rows are independent; OpenMP only spreads them over the host's cores */
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t e = 0; e < E; ++e)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t kk = 0; kk < K; ++kk)
                out[(e * N + n) * K + kk] = oracle_double_to_bf16(
                    weight_elem(blocks, scales, N, K, e, n, kk, defect));
}

/* ---- top-k routing (reading R2) --------------------------------------------- */
/* ids[t, j] in selection order; weights[t, j] = exp(l_j - l_max) / sum over the
 * k selected of exp(l_i - l_max), computed in double and stored as float. */
void oracle_route(const float *logits, int64_t T, int64_t E, int k,
                  int32_t *ids, float *weights)
{
    char *taken = (char *)malloc((size_t)E);
    double *ex = (double *)malloc(sizeof(double) * (size_t)k);
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int64_t best = -1;
            for (int64_t i = 0; i < E; ++i) {
                if (taken[i])
                    continue;
                /* strictly greater keeps the lower index on ties */
                if (best < 0 || l[i] > l[best])
                    best = i;
            }
            taken[best] = 1;
            ids[t * k + j] = (int32_t)best;
        }
        double lmax = (double)l[ids[t * k]];
        double sum = 0.0;
        for (int j = 0; j < k; ++j) {
            ex[j] = exp((double)l[ids[t * k + j]] - lmax);
            sum += ex[j];
        }
        for (int j = 0; j < k; ++j)
            weights[t * k + j] = (float)(ex[j] / sum);
    }
    free(ex);
    free(taken);
}

/* ---- router logits (reading R8; [P3'] mlp.router with its bias) -------------- */
/* out[t, e] = sum_c x[t, c] * W[e, c] + b[e] in double; x, W bf16 bits; b may be NULL. */
void oracle_router_logits(const uint16_t *x, const uint16_t *w, const float *b, int64_t T,
                          int64_t H, int64_t E, double *out)
{
    for (int64_t t = 0; t < T; ++t)
        for (int64_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t c = 0; c < H; ++c)
                acc += oracle_bf16_to_double(x[t * H + c]) * oracle_bf16_to_double(w[e * H + c]);
            out[t * E + e] = acc + (b ? (double)b[e] : 0.0);
        }
}

/* ---- clamped SwiGLU (reading R4; constants from [P3] What it does) ---------- */
double oracle_swiglu(double gate, double up, double alpha, double limit, int defect)
{
    double g = gate, u = up;
    if (defect != ORACLE_DEFECT_NO_CLAMP) {
        g = gate < limit ? gate : limit;
        u = up < -limit ? -limit : (up > limit ? limit : up);
    }
    return (u + 1.0) * g / (1.0 + exp(-alpha * g));
}

/* ---- planted mistake 12 (model of a dropped second split term) --------------- */
/* Round to the nearest E4M3 value [F8], ties to even: 3 fraction bits in the normal
 * range (|r| >= 2^-6), the fixed subnormal spacing 2^-9 below it; magnitudes stay far
 * below 448 here, so there is no saturation. */
static double e4m3_round(double r)
{
    double a = fabs(r);
    if (a == 0.0)
        return r;
    int e2;
    frexp(a, &e2);              /* a in [2^(e2-1), 2^e2) */
    int e = e2 - 1;
    if (e < -6)
        e = -6;
    double q = ldexp(1.0, e - 3);
    return copysign(nearbyint(a / q) * q, r);
}

/* v[0..n) in blocks of 32: each block scaled by 2^(e-7), e = floor(log2 of its
 * largest magnitude), rounded to E4M3 and scaled back. */
static void keep_e4m3_hi_term(double *v, int64_t n)
{
    for (int64_t b0 = 0; b0 < n; b0 += 32) {
        double amax = 0.0;
        for (int64_t i = b0; i < b0 + 32 && i < n; ++i)
            amax = fmax(amax, fabs(v[i]));
        if (amax == 0.0)
            continue;
        int e2;
        frexp(amax, &e2);
        double S = ldexp(1.0, (e2 - 1) - 7);
        for (int64_t i = b0; i < b0 + 32 && i < n; ++i)
            v[i] = e4m3_round(v[i] / S) * S;
    }
}

/* ---- formulation A: per-token loop, weights decoded on the fly -------------- */
/* For each listed token t (token_list[r], r < n_list):
 *   weight on output (flags = 0):
 *     out[r] = sum_j w[t,j] * ( W_d[e] . act( W_gu[e] . x[t] + b_gu[e] ) + b_d[e] )
 *   weight on input (flags = ORACLE_FLAG_WEIGHT_ON_INPUT):
 *     out[r] = sum_j ( W_d[e] . act( W_gu[e] . (w[t,j] x[t]) + b_gu[e] ) + b_d[e] )
 *   where e = ids[t, j], act splits gate/up (reading R3) and applies the clamped
 *   SwiGLU.  Biases may be NULL (zero).  [P3] requires both biases absent in the
 *   weight-on-input mode; the oracle still defines that case the way the review's
 *   test reference does (biases added unweighted) so that the planted mistake
 *   ORACLE_DEFECT_WOI_BIAS_WEIGHTED has something to differ from.
 *   x is bf16 bits [T, H]; W_gu [E, 2I, H] packed; W_d [E, H, I] packed;
 *   out is double [n_list, H].
 *   env (optional, may be NULL) receives the magnitude envelope of the down
 *   projection, the sum over j of |w_eff| * (sum_i |a_i * W_d[e, c, i]| + |b_d[e, c]|)
 *   with w_eff the routing weight applied to that slot's output (1 with the weight on
 *   the input).  It bounds |out| by the triangle inequality and scales the error a
 *   rounded activation operand can cause (MoE-Infinity PR #152, Changes: the parity
 *   test pairs an fp32 golden with a magnitude envelope). */
/* fmt selects the weight format; gu_s2 [E, 2] (gate, up) and d_s2 [E] are the
 * NVFP4 per-expert fp32 scales (NULL: 1), unused for MXFP4. */
static void forward_tokens_impl(int fmt, const uint16_t *x, int64_t T, int64_t H, int64_t I,
                                int64_t E, int k, const int32_t *ids, const float *w,
                                const uint8_t *gu_blocks, const uint8_t *gu_scales,
                                const float *gu_s2, const float *gu_bias,
                                const uint8_t *d_blocks, const uint8_t *d_scales,
                                const float *d_s2, const float *d_bias,
                                double alpha, double limit, int flags,
                                const int64_t *token_list, int64_t n_list, double *out,
                                double *env, int defect)
{
    (void)T;
    (void)E;
    int64_t N_gu = 2 * I;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_list; ++r) {
        int64_t t = token_list[r];
        double *xin = (double *)malloc(sizeof(double) * (size_t)H);
        double *h = (double *)malloc(sizeof(double) * (size_t)N_gu);
        double *a = (double *)malloc(sizeof(double) * (size_t)I);
        double *o = out + r * H;
        double *ev = env ? env + r * H : NULL;
        for (int64_t c = 0; c < H; ++c) {
            o[c] = 0.0;
            if (ev)
                ev[c] = 0.0;
        }
        for (int j = 0; j < k; ++j) {
            int64_t e = ids[t * k + j];
            double wj = (double)w[t * k + j];
            int woi = (flags & ORACLE_FLAG_WEIGHT_ON_INPUT) != 0;
            for (int64_t c = 0; c < H; ++c)
                xin[c] = oracle_bf16_to_double(x[t * H + c]) * (woi ? wj : 1.0);
            if (defect == ORACLE_DEFECT_OPERAND_E4M3_HI_ONLY)
                keep_e4m3_hi_term(xin, H);
            /* gate_up projection with bias before the activation [P3] */
            for (int64_t n = 0; n < N_gu; ++n) {
                double acc = 0.0;
                int zero_row = 0;
                if (defect == ORACLE_DEFECT_GATE_ZERO)
                    zero_row = (n % 2) == 0; /* interleaved: even rows are gate */
                if (!zero_row)
                    for (int64_t c = 0; c < H; ++c)
                        acc += xin[c] * weight_elem_fmt(fmt, gu_blocks, gu_scales, N_gu, H, e, n, c, defect);
                /* NVFP4: the row's weight_scale_2 before the bias (reading R6) */
                double s2 = 1.0;
                if (fmt == ORACLE_FMT_NVFP4 && gu_s2) {
                    int role = (int)(n % 2); /* 0 gate, 1 up (reading R3) */
                    if (defect == ORACLE_DEFECT_NVFP4_GU_SCALE_SWAP)
                        role = 1 - role;
                    s2 = (double)gu_s2[e * 2 + role];
                }
                h[n] = s2 * acc + (gu_bias ? (double)gu_bias[e * N_gu + n] : 0.0);
            }
            for (int64_t i = 0; i < I; ++i) {
                double gate, up;
                if (defect == ORACLE_DEFECT_UNINTERLEAVED) {
                    gate = h[i];
                    up = h[I + i];
                } else {
                    gate = h[2 * i];
                    up = h[2 * i + 1];
                }
                a[i] = oracle_swiglu(gate, up, alpha, limit, defect);
            }
            if (defect == ORACLE_DEFECT_OPERAND_E4M3_HI_ONLY)
                keep_e4m3_hi_term(a, I);
            /* down projection; bias added before the routing weight [P3] */
            for (int64_t c = 0; c < H; ++c) {
                double acc = 0.0, mag = 0.0;
                for (int64_t i = 0; i < I; ++i) {
                    double term = a[i] * weight_elem_fmt(fmt, d_blocks, d_scales, H, I, e, c, i, defect);
                    acc += term;
                    mag += fabs(term);
                }
                double b = d_bias ? (double)d_bias[e * H + c] : 0.0;
                /* NVFP4: y = s*acc + b (reading R6; [P3] NVFP4 down scale vs. down bias) */
                double s2 = (fmt == ORACLE_FMT_NVFP4 && d_s2) ? (double)d_s2[e] : 1.0;
                if (defect == ORACLE_DEFECT_NVFP4_SCALE_AFTER_BIAS)
                    b *= s2;
                acc *= s2;
                mag *= fabs(s2);
                if (ev)
                    ev[c] += (woi ? 1.0 : fabs(wj)) * (mag + fabs(b));
                if (defect == ORACLE_DEFECT_DOWN_BIAS_IN_SCALE)
                    b *= oracle_e8m0_value(d_scales[(e * H + c) * (I / 32)], 0);
                if (woi) {
                    if (defect == ORACLE_DEFECT_WOI_BIAS_WEIGHTED)
                        o[c] += acc + wj * b;
                    else
                        o[c] += acc + b;
                } else if (defect == ORACLE_DEFECT_DOWN_BIAS_UNWEIGHTED) {
                    o[c] += wj * acc + b;
                } else {
                    o[c] += wj * (acc + b); /* sum w * (s*y + b), s = 1 for MXFP4 [P3] */
                }
            }
        }
        free(a);
        free(h);
        free(xin);
    }
}

void oracle_forward_tokens(const uint16_t *x, int64_t T, int64_t H, int64_t I,
                           int64_t E, int k, const int32_t *ids, const float *w,
                           const uint8_t *gu_blocks, const uint8_t *gu_scales,
                           const float *gu_bias, const uint8_t *d_blocks,
                           const uint8_t *d_scales, const float *d_bias,
                           double alpha, double limit, int flags,
                           const int64_t *token_list, int64_t n_list, double *out,
                           double *env, int defect)
{
    forward_tokens_impl(ORACLE_FMT_MXFP4, x, T, H, I, E, k, ids, w, gu_blocks, gu_scales, NULL,
                        gu_bias, d_blocks, d_scales, NULL, d_bias, alpha, limit, flags,
                        token_list, n_list, out, env, defect);
}

/* Formulation A for NVFP4 experts (reading R6): gu_scales E4M3 [E, 2I, H/16],
 * gu_s2 fp32 [E, 2] (gate, up; NULL = 1), d_scales E4M3 [E, H, I/16], d_s2 fp32 [E]
 * (NULL = 1).  Everything else as oracle_forward_tokens. */
void oracle_nvfp4_forward_tokens(const uint16_t *x, int64_t T, int64_t H, int64_t I,
                                 int64_t E, int k, const int32_t *ids, const float *w,
                                 const uint8_t *gu_blocks, const uint8_t *gu_scales,
                                 const float *gu_s2, const float *gu_bias,
                                 const uint8_t *d_blocks, const uint8_t *d_scales,
                                 const float *d_s2, const float *d_bias,
                                 double alpha, double limit, int flags,
                                 const int64_t *token_list, int64_t n_list, double *out,
                                 double *env, int defect)
{
    forward_tokens_impl(ORACLE_FMT_NVFP4, x, T, H, I, E, k, ids, w, gu_blocks, gu_scales, gu_s2,
                        gu_bias, d_blocks, d_scales, d_s2, d_bias, alpha, limit, flags,
                        token_list, n_list, out, env, defect);
}

/* ---- formulation B: group pairs by expert over a pre-decoded bank ----------- */
/* Same result as formulation A (up to summation order), computed the way a
 * grouped kernel organises it: every (token, slot) pair is assigned to its
 * expert, each expert's pairs go through the expert's two projections as a
 * small dense matrix product over the fully decoded double-precision bank, and
 * the rows are scattered back and summed per token in slot order.  Only meant
 * for small shapes (the decoded bank is E*3*H*I doubles).  No planted mistakes. */
int oracle_forward_grouped(const uint16_t *x, int64_t T, int64_t H, int64_t I,
                           int64_t E, int k, const int32_t *ids, const float *w,
                           const uint8_t *gu_blocks, const uint8_t *gu_scales,
                           const float *gu_bias, const uint8_t *d_blocks,
                           const uint8_t *d_scales, const float *d_bias,
                           double alpha, double limit, int flags, double *out)
{
    int64_t N_gu = 2 * I;
    int64_t P = T * k;
    double *Wgu = (double *)malloc(sizeof(double) * (size_t)(E * N_gu * H));
    double *Wd = (double *)malloc(sizeof(double) * (size_t)(E * H * I));
    double *ybuf = (double *)malloc(sizeof(double) * (size_t)(P * H));
    double *h = (double *)malloc(sizeof(double) * (size_t)N_gu);
    double *a = (double *)malloc(sizeof(double) * (size_t)I);
    double *xin = (double *)malloc(sizeof(double) * (size_t)H);
    if (!Wgu || !Wd || !ybuf || !h || !a || !xin) {
        free(Wgu); free(Wd); free(ybuf); free(h); free(a); free(xin);
        return -1;
    }
    for (int64_t e = 0; e < E; ++e) {
        for (int64_t n = 0; n < N_gu; ++n)
            for (int64_t c = 0; c < H; ++c)
                Wgu[(e * N_gu + n) * H + c] = weight_elem(gu_blocks, gu_scales, N_gu, H, e, n, c, 0);
        for (int64_t c = 0; c < H; ++c)
            for (int64_t i = 0; i < I; ++i)
                Wd[(e * H + c) * I + i] = weight_elem(d_blocks, d_scales, H, I, e, c, i, 0);
    }
    int woi = (flags & ORACLE_FLAG_WEIGHT_ON_INPUT) != 0;
    for (int64_t e = 0; e < E; ++e) {
        for (int64_t p = 0; p < P; ++p) { /* pairs p = t*k + j in ascending order */
            if (ids[p] != e)
                continue;
            int64_t t = p / k;
            double wj = (double)w[p];
            for (int64_t c = 0; c < H; ++c)
                xin[c] = oracle_bf16_to_double(x[t * H + c]) * (woi ? wj : 1.0);
            for (int64_t n = 0; n < N_gu; ++n) {
                double acc = 0.0;
                const double *wr = Wgu + (e * N_gu + n) * H;
                for (int64_t c = 0; c < H; ++c)
                    acc += wr[c] * xin[c];
                h[n] = acc + (gu_bias ? (double)gu_bias[e * N_gu + n] : 0.0);
            }
            for (int64_t i = 0; i < I; ++i)
                a[i] = oracle_swiglu(h[2 * i], h[2 * i + 1], alpha, limit, 0);
            for (int64_t c = 0; c < H; ++c) {
                double acc = 0.0;
                const double *wr = Wd + (e * H + c) * I;
                for (int64_t i = 0; i < I; ++i)
                    acc += wr[i] * a[i];
                double y = acc + (d_bias ? (double)d_bias[e * H + c] : 0.0);
                ybuf[p * H + c] = woi ? y : wj * y;
            }
        }
    }
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < H; ++c) {
            double s = 0.0;
            for (int j = 0; j < k; ++j)
                s += ybuf[(t * k + j) * H + c];
            out[t * H + c] = s;
        }
    free(Wgu); free(Wd); free(ybuf); free(h); free(a); free(xin);
    return 0;
}

/* Number of OpenMP threads the forward loop may use (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
