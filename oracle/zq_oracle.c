/*
 * zq_oracle.c -- plain, slow CPU oracle for the ZeroQuant fused quantized
 * linear layer.  TEST INFRASTRUCTURE ONLY: only tests/, the smoke check and
 * the bench's CPU-baseline leg may load it.  It shares no code with the CUDA
 * library and the CUDA library never calls it.
 *
 * Source: "ZeroQuant: Efficient and Affordable Post-Training Quantization for
 * Large-Scale Transformers" (arXiv 2206.01861), section-by-section summary
 * page, Section 3.4 "Detailed, Sentence-Based Technical Breakdown":
 *   - Eq. 2 (symmetric uniform quantizer) and its prose,
 *   - "Group-wise Weight Quantization" (g contiguous row groups, one scale each),
 *   - "Token-wise Activation Quantization" (one scale per token row),
 *   - "Quantization-Optimized Transformer Kernels" (fused LN + quant, INT32
 *     accumulator, dequantization by weight-group scale x token scale in the
 *     GEMM epilogue, Fig. 2 fused == unfused).
 *
 * Readings where the pages are silent or garbled (each one is listed with its
 * reason in the design notes of this repository):
 *   R1 Eq. 2 as printed gives only {-1,0,1}; the prose says "normalise, then
 *      scale to the integer range".  We use S = amax/qmax and
 *      q = rne(x * (qmax/amax)), one IEEE fp32 division per row/group and one
 *      fp32 multiply per element.
 *   R2 Clamp to [-qmax, qmax] (qmax = 127 or 7): symmetric, and the absmax
 *      scale never produces -128/-8 anyway.
 *   R3 LayerNorm statistics are fp32 sums in a fixed order that does not
 *      depend on how a kernel splits the row: chunks of 8 consecutive values
 *      summed in order, chunk sums combined by a zero-padded pairwise tree;
 *      the variance is the biased two-pass sum of (x - mean)^2
 *      (see zqo_ln_row_stats).
 *   R4 The fused kernel quantizes its fp16 LayerNorm output (Fig. 2: fused and
 *      unfused compute the same output).
 *   R5 Scales are fp32.
 *   R6 group(o) = floor(o*g/N): g contiguous groups even when g does not
 *      divide N.
 *   R7 INT4: two's-complement nibbles, two per byte; of each eight
 *      consecutive k, byte i holds k = i (low nibble) and k = 4 + i (high).
 *   R8 "round" = round half to even.
 *   R9 Epilogue: y = fp16( ((f32(acc)*s_tok[t]) * s_grp[group(o)]) + f32(bias[o]) ),
 *      each a separate IEEE round-to-nearest op (no contraction).
 *   R12 Bias-add + quant (the token quantization fused into a bias-add,
 *      "Kernel fusion for token-wise activation quantization"): v = f32(x) +
 *      f32(bias), one fp32 add; y = fp16(v); then the token quantization.
 *   R13 GeLU + quant: GeLU is its exact form, gelu(v) = v * Phi(v) =
 *      0.5 v (1 + erf(v / sqrt 2)) = 0.5 v erfc(-v / sqrt 2), on v of R12;
 *      y = fp16(gelu(v)).  Here it is evaluated in double (erfc form) and
 *      rounded once to fp16; a kernel evaluating it in fp32 (with its math
 *      library's erfc) may differ by one fp16 ulp, and its codes are then
 *      those of the token quantization of its own y.
 *   R14 Static (per-tensor) activation quantization, the prior PTQ scheme the
 *      pages contrast with token-wise quantization: calibration keeps
 *      moving averages x_max = m x_max + (1-m) max(batch), x_min likewise
 *      (m = 0.95), started from the first batch's max and min, fp32; the
 *      range is A = max(|x_max|, |x_min|); every token then uses
 *      s = A/127 and q = clamp(rne(x * (127/A)), -127, 127).
 *   R15 FP16 activations with quantized weights (W8A16, W4/8A16; the summary
 *      page's "Main Quantitative Results" and "INT4/INT8 Mixed-Precision
 *      Quantization"): the layer is X (q S)^T + b with the dequantized
 *      weights q * S[group(o)].  Evaluated here in double: acc = sum_k
 *      x[t,k] q[o,k] (every product exact), y = acc * S + b, rounded once to
 *      fp16.  A tensor-core kernel sums the products in fp32 in its own
 *      order and applies S after the sum, so it agrees within a rounding
 *      bound, not bit for bit.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * fp16 values cross the interface as their uint16 bit patterns.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if defined(__FAST_MATH__)
#error "the oracle must be built without fast-math"
#endif

/* ---------------------------------------------------------------- fp16 */

static uint16_t d2h(double d) {
    _Float16 h = (_Float16)d; /* one IEEE round to nearest even */
    uint16_t bits;
    memcpy(&bits, &h, 2);
    return bits;
}

static float h2f(uint16_t bits) {
    _Float16 h;
    memcpy(&h, &bits, 2);
    return (float)h; /* exact */
}

static uint16_t f2h(float f) {
    _Float16 h = (_Float16)f; /* IEEE round to nearest even */
    uint16_t bits;
    memcpy(&bits, &h, 2);
    return bits;
}

/* Round to nearest, ties to even (R8); the default FE_TONEAREST mode. */
static float rne(float v) { return nearbyintf(v); }

static int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* ------------------------------------------- Eq. 2, one scale per set */

/* The symmetric quantizer of Eq. 2 under readings R1, R2, R8 for one set of
 * values that shares one scale (a weight group or a token row).
 * amax is max|x| over the set; returns S and writes inv = qmax/amax. */
static float eq2_scale(float amax, int qmax, float *inv) {
    if (amax == 0.0f) {
        *inv = 0.0f;
        return 0.0f;
    }
    *inv = (float)qmax / amax;
    return amax / (float)qmax;
}

static int eq2_quantize(float x, float inv, int qmax) {
    if (inv == 0.0f) return 0;
    float v = x * inv;
    return clampi((int)rne(v), -qmax, qmax);
}

/* ------------------------------------- group-wise weight quantization */

/* Group index of output row o when N rows are split into g contiguous
 * groups (R6). */
int zqo_group_of(int o, int N, int g) { return (int)(((int64_t)o * g) / N); }

/* W: fp16 bits [N*K] row-major, rows = outputs.  bits = 8 or 4.
 * q: int8 [N*K] (values in [-qmax, qmax]); s_grp: fp32 [g].
 * Returns 0, or -1 on bad arguments. */
int zqo_quantize_weights_groupwise(const uint16_t *W, int N, int K, int g, int bits,
                                   int8_t *q, float *s_grp) {
    if (N < 1 || K < 1 || g < 1 || g > N || (bits != 8 && bits != 4)) return -1;
    const int qmax = bits == 8 ? 127 : 7;
    float *amax = (float *)calloc((size_t)g, sizeof(float));
    if (!amax) return -1;
    /* S_i = max|W_i| over the rows of group i */
    for (int o = 0; o < N; ++o) {
        int gi = zqo_group_of(o, N, g);
        for (int k = 0; k < K; ++k) {
            float a = fabsf(h2f(W[(size_t)o * K + k]));
            if (a > amax[gi]) amax[gi] = a;
        }
    }
    float *inv = (float *)malloc((size_t)g * sizeof(float));
    if (!inv) { free(amax); return -1; }
    for (int i = 0; i < g; ++i) s_grp[i] = eq2_scale(amax[i], qmax, &inv[i]);
    for (int o = 0; o < N; ++o) {
        int gi = zqo_group_of(o, N, g);
        for (int k = 0; k < K; ++k)
            q[(size_t)o * K + k] = (int8_t)eq2_quantize(h2f(W[(size_t)o * K + k]), inv[gi], qmax);
    }
    free(inv);
    free(amax);
    return 0;
}

/* R7: INT4 codes, two per byte.  Row o is cut into blocks of eight
 * consecutive k; block m is stored in bytes 4m..4m+3 of the row, and byte
 * 4m+i holds q[o, 8m+i] in its low nibble and q[o, 8m+4+i] in its high
 * nibble (two's complement).  K must be a multiple of 8. */
int zqo_pack_int4(const int8_t *q, int N, int K, uint8_t *packed) {
    if (K % 8) return -1;
    for (int o = 0; o < N; ++o)
        for (int m = 0; m < K / 8; ++m)
            for (int i = 0; i < 4; ++i) {
                unsigned lo = (unsigned)q[(size_t)o * K + 8 * m + i] & 0xFu;
                unsigned hi = (unsigned)q[(size_t)o * K + 8 * m + 4 + i] & 0xFu;
                packed[(size_t)o * (K / 2) + 4 * m + i] = (uint8_t)(lo | (hi << 4));
            }
    return 0;
}

static int sext4(unsigned v) { return v >= 8 ? (int)v - 16 : (int)v; }

/* Inverse of zqo_pack_int4: sign-extend each nibble. */
int zqo_unpack_int4(const uint8_t *packed, int N, int K, int8_t *q) {
    if (K % 8) return -1;
    for (int o = 0; o < N; ++o)
        for (int m = 0; m < K / 8; ++m)
            for (int i = 0; i < 4; ++i) {
                unsigned b = packed[(size_t)o * (K / 2) + 4 * m + i];
                q[(size_t)o * K + 8 * m + i] = (int8_t)sext4(b & 0xFu);
                q[(size_t)o * K + 8 * m + 4 + i] = (int8_t)sext4(b >> 4);
            }
    return 0;
}

/* -------------------------------------------- LayerNorm (reading R3) */

/* Pairwise tree over n values (n a power of two): level l adds v[c + 2^l]
 * into v[c] for every c that is a multiple of 2^(l+1).  Returns v[0]. */
static float tree_sum(float *v, int n) {
    for (int step = 1; step < n; step *= 2)
        for (int c = 0; c < n; c += 2 * step) v[c] = v[c] + v[c + step];
    return v[0];
}

static int pow2_at_least(int n) {
    int p = 1;
    while (p < n) p *= 2;
    return p;
}

/* Row sum in the fixed order of reading R3: the row is cut into chunks of
 * eight consecutive values (the last one shorter when K is not a multiple of
 * 8), each chunk summed in index order, and the chunk sums, padded with
 * zeros to a power of two, combined by the pairwise tree.  With sq != 0 the
 * summands are (x - mean)^2: the first one squared, the rest accumulated with
 * fused multiply-adds. */
static float chunk_tree_sum(const uint16_t *x, int K, int sq, float mean) {
    int nchunk = (K + 7) / 8;
    int P = pow2_at_least(nchunk);
    float *cs = (float *)calloc((size_t)P, sizeof(float));
    for (int c = 0; c < nchunk; ++c) {
        int k0 = 8 * c, k1 = k0 + 8 < K ? k0 + 8 : K;
        float acc;
        if (sq) {
            float d = h2f(x[k0]) - mean;
            acc = d * d;
            for (int k = k0 + 1; k < k1; ++k) {
                d = h2f(x[k]) - mean;
                acc = fmaf(d, d, acc);
            }
        } else {
            acc = h2f(x[k0]);
            for (int k = k0 + 1; k < k1; ++k) acc = acc + h2f(x[k]);
        }
        cs[c] = acc;
    }
    float r = tree_sum(cs, P);
    free(cs);
    return r;
}

/* mean and rstd of one row (reading R3, all fp32, biased variance):
 *   mean = S/K with S the fixed-order sum of x,
 *   var  = Q/K with Q the fixed-order sum of (x - mean)^2 (two passes),
 *   rstd = 1/sqrt(var + eps). */
void zqo_ln_row_stats(const uint16_t *x, int K, float eps, float *mean_out, float *rstd_out,
                      double *mean_d_out, double *var_d_out) {
    float mean = chunk_tree_sum(x, K, 0, 0.0f) / (float)K;
    float var = chunk_tree_sum(x, K, 1, mean) / (float)K;
    float r = sqrtf(var + eps);
    *rstd_out = 1.0f / r;
    *mean_out = mean;
    if (mean_d_out) *mean_d_out = (double)mean;
    if (var_d_out) *var_d_out = (double)var;
}

/* Unfused step 1 of Fig. 2: y = fp16(LN(x)) per row.  gamma/beta may be
 * NULL (gamma = NULL means the identity: y = x, the quant-only mode). */
int zqo_layernorm(const uint16_t *X, const uint16_t *gamma, const uint16_t *beta, int T, int K,
                  float eps, uint16_t *Y) {
    if (T < 0 || K < 1) return -1;
    for (int t = 0; t < T; ++t) {
        const uint16_t *x = X + (size_t)t * K;
        uint16_t *y = Y + (size_t)t * K;
        if (!gamma) {
            memcpy(y, x, (size_t)K * 2);
            continue;
        }
        float mean, rstd;
        zqo_ln_row_stats(x, K, eps, &mean, &rstd, NULL, NULL);
        for (int k = 0; k < K; ++k) {
            float d = h2f(x[k]) - mean;
            float n = d * rstd;
            float s = n * h2f(gamma[k]);
            float b = beta ? h2f(beta[k]) : 0.0f;
            y[k] = f2h(s + b);
        }
    }
    return 0;
}

/* Unfused step 2 of Fig. 2: token-wise symmetric INT8 quantization of fp16
 * rows, one scale per row (Token-wise Activation Quantization). */
int zqo_token_quant(const uint16_t *Y, int T, int K, int8_t *q, float *s_tok) {
    if (T < 0 || K < 1) return -1;
    for (int t = 0; t < T; ++t) {
        const uint16_t *y = Y + (size_t)t * K;
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(h2f(y[k]));
            if (a > amax) amax = a;
        }
        float inv;
        s_tok[t] = eq2_scale(amax, 127, &inv);
        for (int k = 0; k < K; ++k) q[(size_t)t * K + k] = (int8_t)eq2_quantize(h2f(y[k]), inv, 127);
    }
    return 0;
}

/* The fused LN + token quantization of Fig. 2 (right), written as its own
 * single pass per row so that the Fig. 2 equality (fused == unfused) is a
 * real check.  Y_ln may be NULL. */
int zqo_ln_quant(const uint16_t *X, const uint16_t *gamma, const uint16_t *beta, int T, int K,
                 float eps, int8_t *q, float *s_tok, uint16_t *Y_ln) {
    if (T < 0 || K < 1) return -1;
    uint16_t *row = (uint16_t *)malloc((size_t)K * 2);
    if (!row) return -1;
    for (int t = 0; t < T; ++t) {
        const uint16_t *x = X + (size_t)t * K;
        float mean = 0.0f, rstd = 1.0f;
        if (gamma) zqo_ln_row_stats(x, K, eps, &mean, &rstd, NULL, NULL);
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            uint16_t yb;
            if (gamma) {
                float v = ((h2f(x[k]) - mean) * rstd) * h2f(gamma[k]);
                yb = f2h(v + (beta ? h2f(beta[k]) : 0.0f));
            } else {
                yb = x[k];
            }
            row[k] = yb;
            float a = fabsf(h2f(yb));
            if (a > amax) amax = a;
        }
        float inv;
        s_tok[t] = eq2_scale(amax, 127, &inv);
        for (int k = 0; k < K; ++k) q[(size_t)t * K + k] = (int8_t)eq2_quantize(h2f(row[k]), inv, 127);
        if (Y_ln) memcpy(Y_ln + (size_t)t * K, row, (size_t)K * 2);
    }
    free(row);
    return 0;
}

/* ------------------------------------------------ INT32 GEMM (exact) */

/* acc[t,o] = sum_k xq[t,k]*wq[o,k], summed in int64 and checked to fit
 * int32 (the INT32 accumulator of the INT8 GEMM).  Returns 0, or -2 if a
 * sum does not fit int32. */
/* GeLU, exact form (R13), in double: v * Phi(v) with Phi(v) = 0.5 erfc(-v / sqrt 2),
 * the same function as 0.5 v (1 + erf(v / sqrt 2)) without its cancellation
 * for negative v. */
double zqo_gelu(double v) { return 0.5 * v * erfc(-v / sqrt(2.0)); }

/* The token quantization fused into a bias-add (act = 0) or into a GeLU
 * (act = 1), R12 / R13: per row, y = fp16(act(f32(x) + f32(bias))), then
 * absmax -> scale -> codes exactly as zqo_token_quant.  bias and Y may be
 * NULL. */
int zqo_bias_act_quant(const uint16_t *X, const uint16_t *bias, int T, int K, int act, int8_t *q,
                       float *s_tok, uint16_t *Y) {
    if (T < 0 || K < 1 || act < 0 || act > 1) return -1;
    uint16_t *row = (uint16_t *)malloc((size_t)K * 2);
    if (!row) return -1;
    for (int t = 0; t < T; ++t) {
        const uint16_t *x = X + (size_t)t * K;
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            float v = h2f(x[k]);
            if (bias) v = v + h2f(bias[k]);
            const uint16_t yb = act == 1 ? d2h(zqo_gelu((double)v)) : f2h(v);
            row[k] = yb;
            float a = fabsf(h2f(yb));
            if (a > amax) amax = a;
        }
        float inv;
        s_tok[t] = eq2_scale(amax, 127, &inv);
        for (int k = 0; k < K; ++k) q[(size_t)t * K + k] = (int8_t)eq2_quantize(h2f(row[k]), inv, 127);
        if (Y) memcpy(Y + (size_t)t * K, row, (size_t)K * 2);
    }
    free(row);
    return 0;
}

/* Static calibration (R14) over nb batches of T x K stored one after the
 * other; writes the calibrated range A. */
int zqo_static_calibrate(const uint16_t *X, int nb, int T, int K, float momentum, float *A) {
    if (nb < 1 || T < 1 || K < 1) return -1;
    float xmax = 0.0f, xmin = 0.0f;
    for (int b = 0; b < nb; ++b) {
        const uint16_t *x = X + (size_t)b * T * K;
        float bmax = h2f(x[0]), bmin = h2f(x[0]);
        for (size_t i = 1; i < (size_t)T * K; ++i) {
            const float v = h2f(x[i]);
            if (v > bmax) bmax = v;
            if (v < bmin) bmin = v;
        }
        if (b == 0) {
            xmax = bmax;
            xmin = bmin;
        } else {
            xmax = momentum * xmax + (1.0f - momentum) * bmax;
            xmin = momentum * xmin + (1.0f - momentum) * bmin;
        }
    }
    *A = fmaxf(fabsf(xmax), fabsf(xmin));
    return 0;
}

/* Static quantization with the calibrated range A (R14): one scale for every
 * token, written to s_tok so that the GEMM's dequantization is unchanged. */
int zqo_static_quant(const uint16_t *X, int T, int K, float A, int8_t *q, float *s_tok) {
    if (T < 0 || K < 1 || !(A >= 0.0f)) return -1;
    float inv;
    const float s = eq2_scale(A, 127, &inv);
    for (int t = 0; t < T; ++t) {
        s_tok[t] = s;
        for (int k = 0; k < K; ++k)
            q[(size_t)t * K + k] = (int8_t)eq2_quantize(h2f(X[(size_t)t * K + k]), inv, 127);
    }
    return 0;
}

int zqo_gemm_i32(const int8_t *xq, const int8_t *wq, int T, int N, int K, int32_t *acc) {
    for (int t = 0; t < T; ++t)
        for (int o = 0; o < N; ++o) {
            int64_t s = 0;
            const int8_t *a = xq + (size_t)t * K, *b = wq + (size_t)o * K;
            for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)b[k];
            if (s > INT32_MAX || s < INT32_MIN) return -2;
            acc[(size_t)t * N + o] = (int32_t)s;
        }
    return 0;
}

/* ----------------------------------------------- dequant epilogue (R9) */

/* y[t,o] = fp16( ((f32(acc)*s_tok[t]) * s_grp[group(o)]) + f32(bias[o]) ).
 * bias may be NULL (treated as 0). */
int zqo_dequant(const int32_t *acc, const float *s_tok, const float *s_grp, int g,
                const uint16_t *bias, int T, int N, uint16_t *Y) {
    if (g < 1 || g > N) return -1;
    for (int t = 0; t < T; ++t)
        for (int o = 0; o < N; ++o) {
            float a = (float)acc[(size_t)t * N + o];
            float v = a * s_tok[t];
            v = v * s_grp[zqo_group_of(o, N, g)];
            v = v + (bias ? h2f(bias[o]) : 0.0f);
            Y[(size_t)t * N + o] = f2h(v);
        }
    return 0;
}

/* GEMM + dequant for one token row at a time (the fused form of Fig. 2,
 * written without an int32 intermediate buffer). */
int zqo_linear_q(const int8_t *xq, const float *s_tok, const int8_t *wq, const float *s_grp, int g,
                 const uint16_t *bias, int T, int N, int K, uint16_t *Y) {
    if (g < 1 || g > N) return -1;
    for (int t = 0; t < T; ++t)
        for (int o = 0; o < N; ++o) {
            int64_t s = 0;
            for (int k = 0; k < K; ++k) s += (int64_t)xq[(size_t)t * K + k] * wq[(size_t)o * K + k];
            if (s > INT32_MAX || s < INT32_MIN) return -2;
            float v = (float)(int32_t)s * s_tok[t];
            v = v * s_grp[zqo_group_of(o, N, g)];
            v = v + (bias ? h2f(bias[o]) : 0.0f);
            Y[(size_t)t * N + o] = f2h(v);
        }
    return 0;
}

/* Reports the rounding mode so a test can confirm round-to-nearest. */
/* FP16 activations times group-wise quantized weights (R15): acc and y in
 * double, Y = fp16(y).  q is int8 [N][K] (INT4 weights: unpacked first). */
int zqo_gemm_a16(const uint16_t *X, const int8_t *q, const float *s_grp, int g,
                 const uint16_t *bias, int T, int N, int K, double *acc, double *y, uint16_t *Y) {
    if (T < 0 || N < 1 || K < 1 || g < 1 || g > N) return -1;
    for (int t = 0; t < T; ++t)
        for (int o = 0; o < N; ++o) {
            double sum = 0.0;
            for (int k = 0; k < K; ++k)
                sum += (double)h2f(X[(size_t)t * K + k]) * (double)q[(size_t)o * K + k];
            const double v = sum * (double)s_grp[zqo_group_of(o, N, g)] +
                             (bias ? (double)h2f(bias[o]) : 0.0);
            acc[(size_t)t * N + o] = sum;
            y[(size_t)t * N + o] = v;
            Y[(size_t)t * N + o] = d2h(v);
        }
    return 0;
}

int zqo_rounding_is_nearest(void) { return fegetround() == FE_TONEAREST; }
