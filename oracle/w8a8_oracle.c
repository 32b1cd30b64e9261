/*
 * w8a8_oracle.c -- plain CPU oracle for the W8A8 quantized linear layer.
 *
 * TEST INFRASTRUCTURE. This file exists so that the CUDA path can be checked
 * against something slow and obviously correct. Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg load it; the product
 * library never links, calls or includes anything from here, and this file
 * includes nothing from the product sources.
 *
 * What it computes (sources are the pages this library is built from):
 *   - PDMIX glossary entry ("PDMIX 阶段间混合量化算法 量化术语百科词条"),
 *     §2.3, eqs. Q_prefill and Q_decode, symbol list (Qmin, Qmax = -128, 127),
 *     §2.1 (one shared per-channel weight).
 *   - PDMIX Parameter Configuration Workflow Guide, §3 bullets and Step 3
 *     table (prefill per-token symmetric, decode per-tensor asymmetric with an
 *     exported zero point, MinMax statistics, int8 per-channel symmetric
 *     MinMax weight), Step 2 YAML.
 *   - LLM.int8() paper summary (blog.rainlin.top), §一.1 absmax equation,
 *     §一.2 four-term zero-point expansion, §二 vector-wise equation, the
 *     architecture figure's steps (1)-(4) and its 16-bit decomposition, and the
 *     mixed-precision decomposition formula Y.
 *
 * Rules kept here on purpose:
 *   - every float step is one IEEE fp32 operation rounded to nearest even; the
 *     file is compiled with -O2 -ffp-contract=off -fno-fast-math, so no FMA
 *     appears unless written as fmaf();
 *   - rounding to an integer is nearbyintf() under FE_TONEAREST (half to even);
 *   - integer products are accumulated in int64_t; the caller checks they fit;
 *   - bf16 is handled as raw uint16_t bits: bf16 -> fp32 is a 16-bit shift
 *     (exact), fp32 -> bf16 is round-to-nearest-even on the bit pattern;
 *   - OpenMP splits work over independent output rows only, so every result is
 *     identical for any thread count.
 *
 * Readings where the pages are silent or garbled are marked "reading:".
 */
#include <fenv.h>
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_DT_BF16 0
#define ORACLE_DT_FP32 1

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp32                                                             */
/* ------------------------------------------------------------------------ */

float oracle_bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

uint16_t oracle_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u) {
        return (uint16_t)((u >> 16) | 0x0040u); /* keep NaN a (quiet) NaN */
    }
    /* round to nearest, ties to even, on the 16 bits that are dropped */
    uint32_t keep_lsb = (u >> 16) & 1u;
    u += 0x7fffu + keep_lsb;
    return (uint16_t)(u >> 16);
}

static float load_elem(const void *base, int dtype, int64_t idx) {
    if (dtype == ORACLE_DT_BF16) return oracle_bf16_to_f32(((const uint16_t *)base)[idx]);
    return ((const float *)base)[idx];
}

int oracle_round_mode_ok(void) { return fegetround() == FE_TONEAREST; }

/* round-half-even of an fp32 value, then clamped into [-1024, 1024] so that
 * the later integer add of a zero point cannot overflow; the final clamp to
 * the int8 range makes this pre-clamp invisible. A NaN (0 * inf, possible
 * only with an infinite r given to the static quantizer, which its contract
 * excludes) is given code 0 here so that the C stays defined. */
static int rne_clamped(float p) {
    if (p != p) return 0;
    float t = nearbyintf(p);
    if (t < -1024.0f) t = -1024.0f;
    if (t > 1024.0f) t = 1024.0f;
    return (int)t;
}

static int clamp_int(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* ------------------------------------------------------------------------ */
/* Symmetric absmax quantizer of one vector (C1).                            */
/* LLM.int8() summary §一.1 (X_i8 = round(127*X / max|X|)) and step (2) of the */
/* architecture figure (X * (127 / C_x)); PDMIX Q_prefill with Z_token = 0    */
/* (configuration guide: prefill is per-token symmetric).                     */
/* reading: scale by r = 127/a (one division per vector) rather than         */
/* dividing each element by S; a == 0 gives S = r = 0 and all-zero codes.    */
/* reading: so does an absmax so small (below 127/FLT_MAX, ~3.7e-37) that     */
/* 127/a overflows fp32: no finite scale resolves such values on the grid.    */
/* ------------------------------------------------------------------------ */
static void absmax_quant_vector(const void *base, int dtype, int64_t start, int64_t stride,
                                int64_t len, const unsigned char *skip, int8_t *q,
                                int64_t q_stride, float *S_out) {
    float a = 0.0f;
    for (int64_t i = 0; i < len; ++i) {
        if (skip && skip[i]) continue;
        float v = fabsf(load_elem(base, dtype, start + i * stride));
        if (v > a) a = v;
    }
    float S = 0.0f, r = 0.0f;
    if (a > 0.0f && 127.0f / a <= FLT_MAX) {
        S = a / 127.0f;
        r = 127.0f / a;
    }
    for (int64_t i = 0; i < len; ++i) {
        int code = 0;
        if (!(skip && skip[i])) {
            float p = load_elem(base, dtype, start + i * stride) * r;
            code = clamp_int(rne_clamped(p), -127, 127);
        }
        q[i * q_stride] = (int8_t)code;
    }
    *S_out = S;
}

/* Per-token dynamic symmetric quantization of X [M, K] (row stride ldx):
 * one scale per row. PDMIX glossary §2.3 eq. Q_prefill; configuration guide
 * Step 3 row qconfig.act.scope. Outputs Xq [M, K] dense, S_x [M]. */
void oracle_quant_per_token(const void *X, int dtype, int64_t M, int64_t K, int64_t ldx,
                            int8_t *Xq, float *S_x) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        absmax_quant_vector(X, dtype, m * ldx, 1, K, NULL, Xq + m * K, 1, &S_x[m]);
    }
}

/* Per-output-channel symmetric weight quantization. W is [K, N] as on the
 * pages (out = X * W), row stride ldw; one scale per column n over all K.
 * Configuration guide Step 2 YAML (weight: per_channel, int8, symmetric,
 * minmax); LLM.int8() summary step (1) (C_w per column of W) and step (2).
 * Outputs Wq [N, K] (K contiguous), s_w [N], colsum[n] = sum_k Wq[n, k]. */
void oracle_quant_weight_per_channel(const void *W, int dtype, int64_t K, int64_t N,
                                     int64_t ldw, int8_t *Wq, float *s_w, int32_t *colsum) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        absmax_quant_vector(W, dtype, n, ldw, K, NULL, Wq + n * K, 1, &s_w[n]);
        int64_t s = 0;
        for (int64_t k = 0; k < K; ++k) s += Wq[n * K + k];
        colsum[n] = (int32_t)s;
    }
}

/* ------------------------------------------------------------------------ */
/* Asymmetric MinMax calibration (C2), PDMIX decode.                         */
/* Glossary §2.3 eq. Q_decode and symbol list ([Qmin, Qmax] = [-128, 127]);  */
/* configuration guide: decode exports per-tensor asymmetric parameters with  */
/* a zero point, statistics from the MinMax observer.                        */
/* reading: the range includes 0 (lo = min(0, min x), hi = max(0, max x)),    */
/* so that real 0 has an exact code; 255 steps over [-128, 127];              */
/* Z = clamp(-128 - rne(lo * r), -128, 127). hi == lo (all zeros) gives       */
/* S = r = 1, Z = 0.                                                          */
/* ------------------------------------------------------------------------ */
void oracle_calibrate_static(const void *X, int dtype, int64_t T, int64_t K, int64_t ldx,
                             float *S, float *r, int32_t *Z) {
    float lo = 0.0f, hi = 0.0f;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t k = 0; k < K; ++k) {
            float v = load_elem(X, dtype, t * ldx + k);
            if (v < lo) lo = v;
            if (v > hi) hi = v;
        }
    }
    float d = hi - lo;
    if (hi == lo || !(255.0f / d <= FLT_MAX)) { /* reading: a range whose 255/d
                                                 * overflows fp32 counts as empty */
        *S = 1.0f;
        *r = 1.0f;
        *Z = 0;
        return;
    }
    *S = d / 255.0f;
    *r = 255.0f / d;
    *Z = clamp_int(-128 - rne_clamped(lo * *r), -128, 127);
}

/* Per-tensor static asymmetric quantization (C3): q = clamp(rne(x * r) + Z,
 * -128, 127). Glossary §2.3 eq. Q_decode; saturation beyond the calibrated
 * range is exactly this clamp (glossary §2.4, last paragraph). */
void oracle_quant_per_tensor(const void *X, int dtype, int64_t M, int64_t K, int64_t ldx,
                             float r, int32_t Z, int8_t *Xq) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) {
            float p = load_elem(X, dtype, m * ldx + k) * r;
            Xq[m * K + k] = (int8_t)clamp_int(rne_clamped(p) + Z, -128, 127);
        }
    }
}

/* Per-tensor static dequantization: x = S * (q - Z), the inverse that the
 * linear quantizer q = round(x / S) + Z of glossary §2.3 implies (the same
 * x ~ S (q - Z) the four-term expansion of the LLM.int8() summary §一.2
 * expands). The difference q - Z is an exact small integer, so the only
 * rounding is the one fp32 product; out_dtype 0 then rounds it to bf16. */
void oracle_dequant_per_tensor(const int8_t *Xq, int64_t M, int64_t K, float S, int32_t Z, int out_dtype,
                               void *out) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) {
            float y = S * (float)((int32_t)Xq[m * K + k] - Z);
            if (out_dtype == 0)
                ((uint16_t *)out)[m * K + k] = oracle_f32_to_bf16(y);
            else
                ((float *)out)[m * K + k] = y;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Integer GEMM (C4): acc[m, n] = sum_k Xq[m, k] * Wq[n, k], int64.           */
/* LLM.int8() summary step (3): INT8 x INT8 products accumulated in INT32.    */
/* ------------------------------------------------------------------------ */
void oracle_gemm_i64(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                     int64_t *acc) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k) s += (int64_t)Xq[m * K + k] * (int64_t)Wq[n * K + k];
            acc[m * N + n] = s;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Zero-point correction (C5) and the dequant epilogue (C7).                 */
/* LLM.int8() summary §一.2: C = A B + A zp_b + B zp_a + zp_a zp_b; with a     */
/* symmetric weight zp_b = 0 and x = S (q - Z) this leaves                    */
/* acc - Z * colsum[n]. Vector-wise dequant (§二 equation and step (4)) is     */
/* the outer-product rescale S_x[m] * s_w[n].                                 */
/* Fixed fp32 order, per element:                                             */
/*   c   = acc - Z * colsum[n]            (exact, int64, must fit int32)      */
/*   f   = (float) c                      (RN)                                */
/*   sc  = S_x[m] * s_w[n]                (RN)                                */
/*   add = side ? side[m, n] : 0; if bias: add = add + bias[n]   (RN)         */
/*   y   = fmaf(f, sc, add)               (one rounding)                      */
/* Returns 0, or -1 when some corrected accumulator leaves the int32 range.   */
/* ------------------------------------------------------------------------ */
int oracle_epilogue(const int64_t *acc, int64_t M, int64_t N, const float *S_x, int s_x_per_row,
                    const int32_t *Z, const int32_t *colsum, const float *s_w, const float *bias,
                    const float *side, float *y) {
    int bad = 0;
    const int64_t z = Z ? (int64_t)(*Z) : 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t m = 0; m < M; ++m) {
        const float sx = s_x_per_row ? S_x[m] : S_x[0];
        for (int64_t n = 0; n < N; ++n) {
            int64_t c = acc[m * N + n];
            if (z != 0) c -= z * (int64_t)colsum[n];
            if (c > INT32_MAX || c < INT32_MIN) bad = 1;
            float f = (float)(int32_t)c;
            float sc = sx * s_w[n];
            float add = 0.0f;
            if (side) add = side[m * N + n];
            if (bias) add = add + bias[n];
            y[m * N + n] = fmaf(f, sc, add);
        }
    }
    return bad ? -1 : 0;
}

void oracle_f32_to_bf16_array(const float *y, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(y[i]);
}

/* ------------------------------------------------------------------------ */
/* LLM.int8() mixed-precision decomposition (C8).                            */
/* Summary, 16-bit decomposition step (1) and mixed-precision decomposition  */
/* steps 1-2: a feature column of X is an outlier when its magnitude exceeds  */
/* the threshold (6.0).                                                       */
/* reading: a column is an outlier when ANY element has |x| > threshold      */
/* (strict); the figure's column holding 12 next to 45 and 37 is selected.    */
/* reading: outlier columns become zeros in Xq (same math as dropping them),  */
/* and the row scale is the absmax over the remaining columns.                */
/* Outputs: Xq [M, K], S_x [M], idx [cap] (ascending), *n_out = number of     */
/* outlier columns (may exceed cap; then only cap are stored), Xo [M, cap]    */
/* bf16 gathered outlier values. Returns 0, or -2 when n_out > cap.           */
/* ------------------------------------------------------------------------ */
int oracle_outlier_split(const uint16_t *X, int64_t M, int64_t K, int64_t ldx, float threshold,
                         int32_t cap, int8_t *Xq, float *S_x, int32_t *idx, int32_t *n_out,
                         uint16_t *Xo) {
    unsigned char *is_out = (unsigned char *)calloc((size_t)(K > 0 ? K : 1), 1);
    if (!is_out) return -3;
    for (int64_t k = 0; k < K; ++k) {
        for (int64_t m = 0; m < M; ++m) {
            if (fabsf(oracle_bf16_to_f32(X[m * ldx + k])) > threshold) {
                is_out[k] = 1;
                break;
            }
        }
    }
    int32_t count = 0;
    for (int64_t k = 0; k < K; ++k) {
        if (is_out[k]) {
            if (count < cap) idx[count] = (int32_t)k;
            ++count;
        }
    }
    *n_out = count;
    const int32_t stored = count < cap ? count : cap;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        absmax_quant_vector(X, ORACLE_DT_BF16, m * ldx, 1, K, is_out, Xq + m * K, 1, &S_x[m]);
        for (int32_t j = 0; j < stored; ++j) Xo[m * cap + j] = X[m * ldx + idx[j]];
    }
    free(is_out);
    return count > cap ? -2 : 0;
}

/* The 16-bit side product of the decomposition: side[m, n] =
 * sum over j ascending of Xo[m, j] * W[idx[j], n], each step one fmaf from
 * 0.0f, bf16 inputs widened exactly to fp32. LLM.int8() summary, 16-bit
 * decomposition step (2) (X_F16 * W_F16 = Out_F16) and the final sum.
 * reading: the pages' FP16 side path runs on bf16 inputs with fp32
 * accumulation; W is the unquantized [K, N] weight, row stride ldw. */
void oracle_outlier_side(const uint16_t *Xo, int64_t M, int32_t n_used, int32_t cap,
                         const int32_t *idx, const uint16_t *W, int64_t ldw, int64_t N,
                         float *side) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            float s = 0.0f;
            for (int32_t j = 0; j < n_used; ++j) {
                float xv = oracle_bf16_to_f32(Xo[m * cap + j]);
                float wv = oracle_bf16_to_f32(W[(int64_t)idx[j] * ldw + n]);
                s = fmaf(xv, wv, s);
            }
            side[m * N + n] = s;
        }
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
