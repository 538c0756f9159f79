/*
 * mfp8_oracle.c — CPU oracle for the FP8_DYNAMIC quantized Linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file.  Only the tests, the smoke check and the bench's CPU
 * baseline leg use it.  It shares no code, header, table or constant with the
 * CUDA library; the two meet only through the seeded input tensors.
 *
 * What it computes, and where that is stated:
 *
 *   - The number format.  "MOSS-VL quantization README" (github OpenMOSS/
 *     MOSS-VL, quantization/), FP8-Dynamic recipe section: weights are
 *     float8_e4m3fn.  "MOSS-VL-Realtime-FP8 mixed-precision strategy"
 *     article, section "252 个主力 Linear 层为什么用 FP8 E4M3": an 8-bit float
 *     with 4 exponent and 3 mantissa bits.  The "fn" variant is finite-only:
 *     no infinities, one NaN pattern per sign (S.1111.111), exponent bias 7,
 *     largest finite value 1.75 * 2^8 = 448.
 *   - Weights: one static scale per output channel; activations: one scale
 *     per token computed at run time.  Same README section ("channel-wise
 *     static", "FP8 per-token dynamic"), and the Realtime-FP8 article's
 *     "channel-wise 静态 scale" / "per-token 动态激活量化" paragraph.
 *   - The pages fix neither the scale formula, the rounding mode, the
 *     saturation rule nor the accumulator precision.  The readings used here:
 *       scale s = fl32(max|x| / 448), raised to FLT_MIN when smaller;
 *       code    = e4m3( fl32(x / s) ), round-to-nearest-even, values that
 *                 round past 448 saturate to 448, NaN stays NaN, the sign of
 *                 zero is kept;
 *       result  = (sum_k dec(a_k) * dec(w_k)) * s_a * s_w, exact sum,
 *                 no bias term.
 *
 * The exact sum: every e4m3 value is an integer multiple of 2^-9 whose
 * magnitude is at most 448 = 229376 * 2^-9, so each product is an integer
 * multiple of 2^-18 below 2^35.6 units and a K = 12288 sum stays under
 * 2^49.2 units.  Both an int64 sum and an fp64 sum in any order are exact.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off (no -ffast-math: IEEE division,
 * no flush-to-zero).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- bf16 -- */

/* A bf16 value is the upper half of an IEEE binary32: widening is exact. */
float orc_bf16_to_f32(uint16_t h) {
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

/* ---------------------------------------------------------------- e4m3 -- */

/* Decode one float8_e4m3fn code from the format definition:
 *   code = s | eeee | mmm, bias 7;
 *   e == 0          -> (-1)^s * m * 2^-9          (subnormal)
 *   e == 15, m == 7 -> NaN                        (the only non-finite code)
 *   otherwise       -> (-1)^s * (1 + m/8) * 2^(e-7)
 */
double orc_e4m3_decode(uint8_t code) {
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Encode one fp32 value to float8_e4m3fn: round to nearest, ties to even,
 * on the 3-bit mantissa (subnormals on the fixed 2^-9 grid); magnitudes that
 * round above 448 (and infinities) become 448; NaN becomes NaN; the sign is
 * kept, also for results that round to zero. */
uint8_t orc_e4m3_encode(float v) {
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    if (isnan(v)) return (uint8_t)(sign | 0x7F);
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a == 0.0) return sign;

    /* a lies in [2^E, 2^(E+1)). */
    int fe;
    frexp(a, &fe);
    int E = fe - 1;
    /* Spacing of representable values around a: 2^(E-3) for normals
     * (E >= -6), the subnormal step 2^-9 below. */
    int q = (E < -6) ? -9 : E - 3;
    double steps = nearbyint(ldexp(a, -q)); /* default mode: ties to even */
    double r = ldexp(steps, q);             /* exact rounded magnitude */
    if (r == 0.0) return sign;

    int re;
    frexp(r, &re);
    int RE = re - 1;
    uint8_t code;
    if (RE < -6) {
        code = (uint8_t)ldexp(r, 9); /* subnormal: m = r / 2^-9, 1..7 */
    } else {
        int mant = (int)ldexp(ldexp(r, -RE) - 1.0, 3);
        code = (uint8_t)(((RE + 7) << 3) | mant);
    }
    return (uint8_t)(sign | code);
}

void orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

void orc_e4m3_decode_array(const uint8_t* c, int64_t n, double* out) {
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = orc_e4m3_decode(c[i]);
}

/* Encode every fp32 bit pattern in [lo, hi) and write the codes. */
void orc_e4m3_encode_bits_range(uint64_t lo, uint64_t hi, uint8_t* out) {
    int64_t n = (int64_t)(hi - lo);
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i) {
        uint32_t bits = (uint32_t)(lo + (uint64_t)i);
        float f;
        memcpy(&f, &bits, sizeof f);
        out[i] = orc_e4m3_encode(f);
    }
}

/* --------------------------------------------------------------- scales -- */

/* One scale for one row of bf16 values (a token of X, or an output channel
 * of W): s = fl32(max_k |x_k| / 448), no smaller than FLT_MIN. */
float orc_row_scale(const uint16_t* row, int64_t K) {
    float amax = 0.0f;
    int64_t k;
    for (k = 0; k < K; ++k) {
        float a = fabsf(orc_bf16_to_f32(row[k]));
        if (a > amax) amax = a;
    }
    float s = amax / 448.0f;
    if (s < FLT_MIN) s = FLT_MIN;
    return s;
}

/* Quantize R rows of K bf16 values, one scale per row:
 *   s[r] = orc_row_scale(row r),  Q[r,k] = e4m3(fl32(x[r,k] / s[r])).
 * Used for the weights (rows = output channels, once) and for the
 * activations (rows = tokens, every call) alike: the rule is the same, only
 * when it runs differs. */
void orc_quantize_rows(const uint16_t* X, int64_t R, int64_t K, uint8_t* Q, float* s) {
    int64_t r;
#pragma omp parallel for schedule(dynamic, 16)
    for (r = 0; r < R; ++r) {
        const uint16_t* row = X + r * K;
        float sr = orc_row_scale(row, K);
        int64_t k;
        for (k = 0; k < K; ++k) {
            float q = orc_bf16_to_f32(row[k]) / sr;
            Q[r * K + k] = orc_e4m3_encode(q);
        }
        s[r] = sr;
    }
}

/* ---------------------------------------------------- FP8 KV cache -- */

/* fp32 -> bf16: round to nearest, ties to even, on the 16 low bits dropped
 * (a carry out of the mantissa moves into the exponent, up to infinity); a
 * NaN stays a NaN (its quiet bit set). */
uint16_t orc_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lower = u & 0xFFFFu, upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

/* The FP8 e4m3 KV cache ("MOSS-VL quantization README", SGLang paragraph:
 * --kv-cache-dtype fp8_e4m3; the pages give only the flag).  Reading: a K or
 * V tensor [T tokens][H heads][D] in bf16 gets one scale per (token, head)
 * row of D values, by the same rule as the activations (orc_quantize_rows):
 * s = fl32(absmax / 448) floored at FLT_MIN, q = e4m3(fl32(x / s)). */
void orc_kv_quantize(const uint16_t* KV, int64_t T, int64_t H, int64_t D, uint8_t* Q, float* s) {
    orc_quantize_rows(KV, T * H, D, Q, s);
}

/* Dequantize (reading): out = bf16(fl32(dec(q) * s)), the product rounded
 * to fp32 (the decoded value is exact in fp32) and then to bf16. */
void orc_kv_dequantize(const uint8_t* Q, const float* s, int64_t T, int64_t H, int64_t D, uint16_t* out) {
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < T * H; ++r) {
        int64_t k;
        for (k = 0; k < D; ++k) {
            float v = (float)orc_e4m3_decode(Q[r * D + k]) * s[r];
            out[r * D + k] = orc_f32_to_bf16(v);
        }
    }
}

/* ------------------------------------------------- INT8 KV cache (HQQ) -- */

/* The INT8 KV cache of the "MOSS-VL quantization README", KV8 section: the
 * cache_config of generation_config.json names the hqq backend with nbits 8,
 * axis_key = axis_value = 0, q_group_size 64 and residual_length 128, and the
 * text says the history is kept quantized while a short bf16 tail of recent
 * positions is not.  The pages give these settings, not HQQ's optimizer.
 *
 * Readings (all of them this project's):
 *  - a K or V tensor of one layer is [T tokens][H heads][D]; axis 0 is the
 *    token axis, so a group is 64 consecutive tokens of one (head, channel)
 *    column, and a tensor of T tokens (T % 64 == 0) has T/64 groups per
 *    column: scale and zero are [T/64][H][D];
 *  - the fit is the asymmetric min-max one with an integer zero point,
 *    in fp32 with each rounding stated (rint = nearest, ties to even):
 *      range = fl32(max - min)
 *      s = max(fl32(range / 255), FLT_MIN)     when range > 0
 *      s = max(|min|, FLT_MIN)                 for a constant group
 *      z = rint(fl32(-min / s)) + 0            (+0, never -0)
 *      q = min(255, max(0, rint(fl32(fl32(x / s) + z))))   (NaN -> 0)
 *    so the group's minimum gets code 0, its maximum 255 or 254 (the
 *    rounded zero point moves the grid by at most half a step), and a
 *    constant group is reproduced exactly;
 *  - dequantize: x' = bf16(fl32(fl32(q - z) * s)) (q - z is exact).
 * The values must be finite with max - min finite in fp32. */
static void kv8_fit(float mn, float mx, float* s_out, float* z_out) {
    float range = mx - mn, s;
    if (range > 0.0f) {
        s = range / 255.0f;
        if (s < FLT_MIN) s = FLT_MIN;
    } else {
        s = fabsf(mn);
        if (s < FLT_MIN) s = FLT_MIN;
    }
    *s_out = s;
    *z_out = rintf(-mn / s) + 0.0f;
}

static uint8_t kv8_code(float x, float s, float z) {
    float t = x / s;
    t = t + z;
    float q = rintf(t);
    q = fmaxf(q, 0.0f); /* NaN -> 0 */
    q = fminf(q, 255.0f);
    return (uint8_t)q;
}

void orc_kv8_quantize(const uint16_t* KV, int64_t T, int64_t H, int64_t D, uint8_t* Q, float* scale, float* zero) {
    const int64_t C = H * D, G = T / 64;
    int64_t gc;
#pragma omp parallel for schedule(static)
    for (gc = 0; gc < G * C; ++gc) {
        const int64_t g = gc / C, c = gc % C;
        const uint16_t* x = KV + g * 64 * C + c; /* token 64g, column c */
        float mn = orc_bf16_to_f32(x[0]), mx = mn, s, z;
        int t;
        for (t = 1; t < 64; ++t) {
            float v = orc_bf16_to_f32(x[t * C]);
            if (v < mn) mn = v;
            if (v > mx) mx = v;
        }
        kv8_fit(mn, mx, &s, &z);
        for (t = 0; t < 64; ++t) Q[(g * 64 + t) * C + c] = kv8_code(orc_bf16_to_f32(x[t * C]), s, z);
        scale[gc] = s;
        zero[gc] = z;
    }
}

/* The cache read (the README's KV8 caveat: the quantized history is
 * dequantized and the bf16 tail appended): out [Tq + Tr][H][D] holds the Tq
 * quantized tokens dequantized, then the Tr residual tokens as they are. */
void orc_kv8_read(const uint8_t* Q, const float* scale, const float* zero, int64_t Tq, const uint16_t* resid,
                  int64_t Tr, int64_t H, int64_t D, uint16_t* out) {
    const int64_t C = H * D;
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < Tq * C; ++i) {
        const int64_t t = i / C, c = i % C, gc = (t / 64) * C + c;
        const float d = (float)Q[i] - zero[gc];
        out[i] = orc_f32_to_bf16(d * scale[gc]);
    }
    memcpy(out + Tq * C, resid, (size_t)(Tr * C) * sizeof(uint16_t));
}

/* How many of the T positions a cache holds quantized (reading of
 * residual_length 128 with groups of 64 along the tokens): the latest 128
 * positions always stay bf16, and older ones are quantized in whole groups,
 * so Tq = 64 * floor((T - 128) / 64) for T >= 128, else 0. */
int64_t orc_kv8_history_tokens(int64_t T) {
    return T < 128 ? 0 : 64 * ((T - 128) / 64);
}

/* ------------------------------------- producers of the activations -- */

/* RMSNorm, the producer of the q/k/v and gate/up inputs ("MOSS-VL-Realtime-FP8
 * mixed-precision strategy" article: the norms stay in high precision and
 * feed the FP8 Linears).  The pages fix neither the formula's rounding nor
 * eps; reading: y = x * g / sqrt(mean_k(x^2) + eps), computed exactly here
 * (fp64; the result is the unrounded value the bf16 output approximates).
 * X [M, K] and g [K] are bf16 bit patterns; y [M, K] fp64. */
void orc_rmsnorm(const uint16_t* X, const uint16_t* g, int64_t M, int64_t K, double eps, double* y) {
    int64_t m;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        const uint16_t* row = X + m * K;
        double ss = 0.0;
        int64_t k;
        for (k = 0; k < K; ++k) {
            double v = (double)orc_bf16_to_f32(row[k]);
            ss += v * v;
        }
        double r = 1.0 / sqrt(ss / (double)K + eps);
        for (k = 0; k < K; ++k)
            y[m * K + k] = (double)orc_bf16_to_f32(row[k]) * r * (double)orc_bf16_to_f32(g[k]);
    }
}

/* The gated MLP activation before down_proj (not named on the pages;
 * reading: SiLU(gate) * up, SiLU(v) = v / (1 + e^-v)), on the packed
 * gate_up output GU [M, 2I] (gate in columns 0 .. I-1, up in I .. 2I-1, the
 * README's packed gate_up_proj), exactly in fp64: y [M, I]. */
void orc_silu_mul(const uint16_t* GU, int64_t M, int64_t I, double* y) {
    int64_t m;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        int64_t k;
        for (k = 0; k < I; ++k) {
            double gv = (double)orc_bf16_to_f32(GU[m * 2 * I + k]);
            double uv = (double)orc_bf16_to_f32(GU[m * 2 * I + I + k]);
            y[m * I + k] = gv / (1.0 + exp(-gv)) * uv;
        }
    }
}

/* ----------------------------------------------------------------- GEMM -- */

/* y_ref[m,n] = (sum_k dec(X8[m,k]) * dec(W8[n,k])) * s_a[m] * s_w[n]
 * s_abs[m,n] = (sum_k |dec(X8[m,k]) * dec(W8[n,k])|) * s_a[m] * s_w[n]
 * X8 is [M,K], W8 is [N,K] (output-channel-major, the Linear layout), both
 * row-major.  The sums are exact (see the header).  Either output pointer may
 * be NULL. */
void orc_linear_ref(const uint8_t* X8, const float* s_a, int64_t M,
                    const uint8_t* W8, const float* s_w, int64_t N, int64_t K,
                    double* y_ref, double* s_abs) {
    double* xd = (double*)malloc(sizeof(double) * (size_t)(M * K));
    int64_t i;
    for (i = 0; i < M * K; ++i) xd[i] = orc_e4m3_decode(X8[i]);

    int64_t n;
#pragma omp parallel
    {
        double* wd = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 8)
        for (n = 0; n < N; ++n) {
            int64_t k, m;
            for (k = 0; k < K; ++k) wd[k] = orc_e4m3_decode(W8[n * K + k]);
            for (m = 0; m < M; ++m) {
                const double* xr = xd + m * K;
                double dot = 0.0, dabs = 0.0;
                for (k = 0; k < K; ++k) {
                    double p = xr[k] * wd[k];
                    dot += p;
                    dabs += fabs(p);
                }
                double sc = (double)s_a[m] * (double)s_w[n];
                if (y_ref) y_ref[m * N + n] = dot * sc;
                if (s_abs) s_abs[m * N + n] = dabs * sc;
            }
        }
        free(wd);
    }
    free(xd);
}

/* The same contraction with integers only: each code value times 2^9 is an
 * integer, so dot[m,n] * 2^18 = sum_k int(X8) * int(W8) exactly.  Writes the
 * integer sums. */
void orc_dot_int64(const uint8_t* X8, int64_t M, const uint8_t* W8, int64_t N, int64_t K,
                   int64_t* dot_units) {
    int64_t n;
#pragma omp parallel for schedule(dynamic, 8)
    for (n = 0; n < N; ++n) {
        int64_t m, k;
        for (m = 0; m < M; ++m) {
            int64_t acc = 0;
            for (k = 0; k < K; ++k) {
                int64_t a = (int64_t)ldexp(orc_e4m3_decode(X8[m * K + k]), 9);
                int64_t b = (int64_t)ldexp(orc_e4m3_decode(W8[n * K + k]), 9);
                acc += a * b;
            }
            dot_units[m * N + n] = acc;
        }
    }
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
