/*
 * oracle.c -- plain, slow CPU reference of the per-layer routed-expert step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header or table with the CUDA path.
 *
 * Sources (the FreeToken pages):
 *   - offload backend: experts in host RAM, an LRU cache of expert slots on the
 *     GPU, misses streamed over PCIe   (florigen.ai, "FreeTokenは何をしているのか";
 *     pirouter.ai, "32 GB に 65 GB が載る仕組み")
 *   - cache unit (layer, expert), least-recently-used replacement, contents follow
 *     the router                       (ai-hardware-zukan, "GPUに載らない分をどう間に合わせるか")
 *   - one global LRU expert cache      (gaming-st.com, "技術的背景")
 *   - routed experts NVFP4 = E2M1 values with block scaling
 *                                      (florigen.ai, "NVFP4で約135GBまで縮める")
 *   - hybrid split q = m*B_P/B_H from equal finish times, valid for B_H > B_P;
 *     hybrid chosen when B_H/B_P exceeds the threshold 2.0
 *                                      (ai-hardware-zukan, "GPUに載らない分をどう間に合わせるか";
 *                                       florigen.ai, "CPU/PCIe ratio 1.70x")
 * Where the pages are silent the readings are: softmax over all E logits,
 * k largest logits (ties to the lower id), gates renormalised over the
 * selected k, selected ids processed in ascending order, shared expert with
 * unit weight, SwiGLU h = silu(gate) * up, per-row fp32 activation scale for
 * the W4A4 (prefill) path, LRU order within one lookup batch: hits stamped
 * first in ascending id, then misses in ascending id take the lowest free slot
 * or evict the slot with the smallest stamp.
 *
 * Precision: fp64 throughout, except the NVFP4 activation quantizer, which is
 * fp32 with round-to-nearest-even in a fixed operation order, so that its
 * integer decisions are taken in the same precision as the kernel's.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------ number formats -- */
/* E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; no inf/NaN.
 * exponent 0 is subnormal: value = m * 0.5. */
EXPORT double orc_e2m1(int code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E4M3 ("fn"): 1 sign, 4 exponent (bias 7), 3 mantissa bits; no inf;
 * S.1111.111 is NaN; exponent 0 is subnormal: value = m/8 * 2^-6. */
EXPORT double orc_e4m3(int byte) {
    int s = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

static double bf16_val(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* ------------------------------------------------------- record layout -- */
static int64_t up256(int64_t x) { return (x + 255) / 256 * 256; }

/* Byte offsets: [4] 3 fp32 tensor scales (gate, up, down) at the record head,
 * then [0] W13 codes [2F x d/2], [1] W13 scales [2F x d/16], [2] W2 codes
 * [d x F/2], [3] W2 scales [d x F/16]; [5] record size.  Every section starts
 * on a 256-byte boundary.  W13 row 2j = gate_j, 2j+1 = up_j. */
EXPORT void orc_record_layout(int d, int F, int64_t *off) {
    int64_t w13_rows = 2 * (int64_t)F, w2_rows = d;
    off[4] = 0;
    off[0] = up256(3 * 4);
    off[1] = off[0] + up256(w13_rows * d / 2);
    off[2] = off[1] + up256(w13_rows * d / 16);
    off[3] = off[2] + up256(w2_rows * F / 2);
    off[5] = off[3] + up256(w2_rows * F / 16);
}

static float rec_tensor_scale(const uint8_t *rec, const int64_t *off, int which) {
    float t;
    memcpy(&t, rec + off[4] + 4 * which, 4);
    return t;
}

/* Dequantised element (row r, column k) of a matrix with K columns. */
static double dq(const uint8_t *codes, const uint8_t *scales, int64_t K, int64_t r, int64_t k,
                 double tscale) {
    uint8_t byte = codes[r * (K / 2) + k / 2];
    int code = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    return orc_e2m1(code) * orc_e4m3(scales[r * (K / 16) + k / 16]) * tscale;
}

/* Full dequantised matrix (for tests): which = 0 gate [F x d], 1 up [F x d], 2 down [d x F]. */
EXPORT void orc_dequant_matrix(const uint8_t *rec, int d, int F, int which, double *out) {
    int64_t off[6];
    orc_record_layout(d, F, off);
    double ts = rec_tensor_scale(rec, off, which);
    if (which < 2) {
        for (int64_t j = 0; j < F; ++j)
            for (int64_t k = 0; k < d; ++k)
                out[j * d + k] = dq(rec + off[0], rec + off[1], d, 2 * j + which, k, ts);
    } else {
        for (int64_t i = 0; i < d; ++i)
            for (int64_t j = 0; j < F; ++j)
                out[i * F + j] = dq(rec + off[2], rec + off[3], F, i, j, ts);
    }
}

/* ------------------------------------------------------------- routing -- */
/* Router for T rows: logits z = W_r x (fp64 accumulation of exact bf16
 * products), softmax over all E, the k largest logits (ties: lower id),
 * gates renormalised over the selection when renorm != 0.  Output ids are in
 * ascending order.  gap[t] = z_(k) - z_(k+1) (+inf when k == E).
 * Non-finite logits (the pages say nothing about them; reading taken): a NaN
 * logit is replaced by -inf before the selection and the softmax, so the
 * order (value descending, id ascending) is total and k distinct ids in
 * [0, E) always come out; gates follow IEEE arithmetic on those values (NaN
 * when the largest logit is +inf or every logit is -inf).
 * Returns 0, or -1 on bad arguments. */
EXPORT int orc_route(const uint16_t *Wr, const uint16_t *x, int T, int E, int d, int k,
                     int renorm, int32_t *idx, double *gates, double *logits, double *gap) {
    if (T < 0 || E <= 0 || d <= 0 || k <= 0 || k > E) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        double *z = (double *)malloc(sizeof(double) * E);
        char *taken = (char *)calloc((size_t)E, 1);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * k);
        const uint16_t *xr = x + (int64_t)t * d;
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            const uint16_t *w = Wr + (int64_t)e * d;
            for (int K = 0; K < d; ++K) acc += bf16_val(w[K]) * bf16_val(xr[K]);
            z[e] = isnan(acc) ? -INFINITY : acc;
        }
        /* selection: repeatedly take the largest remaining logit, lower id on ties */
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || z[e] > z[best])) best = e;
            taken[best] = 1;
            sel[j] = best;
        }
        if (gap) {
            int nxt = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (nxt < 0 || z[e] > z[nxt])) nxt = e;
            gap[t] = nxt < 0 ? INFINITY : z[sel[k - 1]] - z[nxt];
        }
        /* softmax over all E */
        double zmax = z[0];
        for (int e = 1; e < E; ++e) zmax = z[e] > zmax ? z[e] : zmax;
        double denom = 0.0;
        for (int e = 0; e < E; ++e) denom += exp(z[e] - zmax);
        double selsum = 0.0;
        for (int j = 0; j < k; ++j) selsum += exp(z[sel[j]] - zmax) / denom;
        /* ascending id order */
        int j = 0;
        for (int e = 0; e < E; ++e) {
            if (!taken[e]) continue;
            double p = exp(z[e] - zmax) / denom;
            idx[(int64_t)t * k + j] = e;
            gates[(int64_t)t * k + j] = renorm ? p / selsum : p;
            ++j;
        }
        if (logits)
            for (int e = 0; e < E; ++e) logits[(int64_t)t * E + e] = z[e];
        free(z);
        free(taken);
        free(sel);
    }
    return 0;
}

/* ---------------------------------------------------------- expert FFN -- */
static double silu(double v) { return v / (1.0 + exp(-v)); }

/* W4A16 expert: g_j = sum_K W1[j,K] x_K, u_j = sum_K W3[j,K] x_K,
 * h_j = silu(g_j) * u_j, y_i = sum_j W2[i,j] h_j; x given as fp64. */
static void expert_from_f64(const uint8_t *rec, int d, int F, const double *xv, double *y,
                            double *h_out) {
    int64_t off[6];
    orc_record_layout(d, F, off);
    double tg = rec_tensor_scale(rec, off, 0), tu = rec_tensor_scale(rec, off, 1);
    double td = rec_tensor_scale(rec, off, 2);
    double *h = (double *)malloc(sizeof(double) * F);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < F; ++j) {
        double g = 0.0, u = 0.0;
        for (int64_t K = 0; K < d; ++K) {
            g += dq(rec + off[0], rec + off[1], d, 2 * j, K, tg) * xv[K];
            u += dq(rec + off[0], rec + off[1], d, 2 * j + 1, K, tu) * xv[K];
        }
        h[j] = silu(g) * u;
    }
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < F; ++j) acc += dq(rec + off[2], rec + off[3], F, i, j, td) * h[j];
        y[i] = acc;
    }
    if (h_out) memcpy(h_out, h, sizeof(double) * F);
    free(h);
}

EXPORT void orc_expert_w4a16(const uint8_t *rec, int d, int F, const uint16_t *x, double *y,
                             double *h_out) {
    double *xv = (double *)malloc(sizeof(double) * d);
    for (int K = 0; K < d; ++K) xv[K] = bf16_val(x[K]);
    expert_from_f64(rec, d, F, xv, y, h_out);
    free(xv);
}

/* ------------------------------------------- MXFP4 and BF16 expert records -- */
/* The formats the pages name for other checkpoints (florigen, "NVFP4で約135GBまで縮める":
 * shared experts kept in BF16; pages' model tables: gpt-oss and DeepSeek-V4
 * routed experts in MXFP4).  MXFP4 as the OCP microscaling formats define it:
 * E2M1 elements, one E8M0 scale per 32 consecutive elements, no tensor scale. */

/* E8M0: an 8-bit biased exponent, value 2^(code - 127); code 255 is NaN. */
EXPORT double orc_e8m0(int code) {
    if (code == 255) return NAN;
    return ldexp(1.0, code - 127);
}

/* MXFP4 record offsets: [0] W13 codes [2F x d/2] (row 2j = gate_j, 2j+1 = up_j),
 * [1] W13 E8M0 scales [2F x d/32], [2] W2 codes [d x F/2], [3] W2 scales
 * [d x F/32]; [4] record size; every section on a 256-byte boundary. */
EXPORT void orc_mx_record_layout(int d, int F, int64_t *off) {
    int64_t w13_rows = 2 * (int64_t)F, w2_rows = d;
    off[0] = 0;
    off[1] = off[0] + up256(w13_rows * d / 2);
    off[2] = off[1] + up256(w13_rows * d / 32);
    off[3] = off[2] + up256(w2_rows * F / 2);
    off[4] = off[3] + up256(w2_rows * F / 32);
}

static double dq_mx(const uint8_t *codes, const uint8_t *scales, int64_t K, int64_t r, int64_t k) {
    uint8_t byte = codes[r * (K / 2) + k / 2];
    int code = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    return orc_e2m1(code) * orc_e8m0(scales[r * (K / 32) + k / 32]);
}

/* Full dequantised matrix of an MXFP4 record: which = 0 gate [F x d], 1 up, 2 down [d x F]. */
EXPORT void orc_dequant_matrix_mx(const uint8_t *rec, int d, int F, int which, double *out) {
    int64_t off[5];
    orc_mx_record_layout(d, F, off);
    if (which < 2) {
        for (int64_t j = 0; j < F; ++j)
            for (int64_t k = 0; k < d; ++k) out[j * d + k] = dq_mx(rec + off[0], rec + off[1], d, 2 * j + which, k);
    } else {
        for (int64_t i = 0; i < d; ++i)
            for (int64_t j = 0; j < F; ++j) out[i * F + j] = dq_mx(rec + off[2], rec + off[3], F, i, j);
    }
}

/* W4A16 expert over an MXFP4 record, in fp64 (same SwiGLU as expert_from_f64). */
EXPORT void orc_expert_mx_w4a16(const uint8_t *rec, int d, int F, const uint16_t *x, double *y) {
    int64_t off[5];
    orc_mx_record_layout(d, F, off);
    double *h = (double *)malloc(sizeof(double) * F);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < F; ++j) {
        double g = 0.0, u = 0.0;
        for (int64_t K = 0; K < d; ++K) {
            const double xv = bf16_val(x[K]);
            g += dq_mx(rec + off[0], rec + off[1], d, 2 * j, K) * xv;
            u += dq_mx(rec + off[0], rec + off[1], d, 2 * j + 1, K) * xv;
        }
        h[j] = silu(g) * u;
    }
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < F; ++j) acc += dq_mx(rec + off[2], rec + off[3], F, i, j) * h[j];
        y[i] = acc;
    }
    free(h);
}

/* Expert over a BF16 record (W13 [2F x d], rows interleaved gate/up, then W2 [d x F]), fp64. */
EXPORT void orc_expert_bf16(const uint16_t *rec, int d, int F, const uint16_t *x, double *y) {
    const uint16_t *w13 = rec, *w2 = rec + 2 * (int64_t)F * d;
    double *h = (double *)malloc(sizeof(double) * F);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < F; ++j) {
        double g = 0.0, u = 0.0;
        for (int64_t K = 0; K < d; ++K) {
            const double xv = bf16_val(x[K]);
            g += bf16_val(w13[(2 * j) * d + K]) * xv;
            u += bf16_val(w13[(2 * j + 1) * d + K]) * xv;
        }
        h[j] = silu(g) * u;
    }
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < F; ++j) acc += bf16_val(w2[i * (int64_t)F + j]) * h[j];
        y[i] = acc;
    }
    free(h);
}

/* ------------------------------------------- NVFP4 activation quantizer -- */
/* fp32, round-to-nearest-even, in this order:
 *   s_t = amax(row) / 2688 (1 if amax = 0); r = amax(block) / (6 s_t);
 *   sb = E4M3(r) RNE saturating; denom = value(sb) * s_t; code = E2M1(x/denom) RNE saturating;
 *   all codes 0 when value(sb) = 0. */
EXPORT float orc_tensor_scale_f32(const float *x, int64_t n) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    return amax > 0.0f ? amax / 2688.0f : 1.0f;
}

/* E4M3 code of r >= 0, RNE, saturating to 448 (code 0x7E). */
EXPORT int orc_e4m3_rne(float r) {
    if (!(r < 448.0f)) return 0x7E;
    if (r < 0.015625f) {                 /* below 2^-6: subnormal grid m * 2^-9, m = 0..8 */
        return (int)nearbyintf(r * 512.0f); /* m = 8 is the smallest normal, code 0x08 */
    }
    int ex;
    frexpf(r, &ex);                      /* r = f * 2^ex, f in [0.5, 1) */
    int E = ex - 1;                      /* r in [2^E, 2^(E+1)) */
    float q = ldexpf(1.0f, E - 3);       /* mantissa step */
    int n = (int)nearbyintf(r / q);      /* in [8, 16] */
    if (n == 16) { E += 1; n = 8; }
    int code = ((E + 7) << 3) | (n - 8);
    return code > 0x7E ? 0x7E : code;
}

/* E2M1 code of v, RNE with ties to the even code, saturating to +-6. */
EXPORT int orc_e2m1_rne(float v) {
    float a = fabsf(v);
    int m;
    if (a <= 0.25f) m = 0;
    else if (a < 0.75f) m = 1;
    else if (a <= 1.25f) m = 2;
    else if (a < 1.75f) m = 3;
    else if (a <= 2.5f) m = 4;
    else if (a < 3.5f) m = 5;
    else if (a <= 5.0f) m = 6;
    else m = 7;
    return (signbit(v) ? 8 : 0) | m;
}

/* Quantize n values (n a multiple of 16) with tensor scale s_t. codes: n/2
 * bytes, element 2i in the low nibble; scales: n/16 E4M3 bytes. */
EXPORT void orc_nvfp4_quantize(const float *x, int64_t n, float s_t, uint8_t *codes,
                               uint8_t *scales) {
    float six_st = 6.0f * s_t;
    for (int64_t b = 0; b < n / 16; ++b) {
        const float *blk = x + b * 16;
        float bmax = 0.0f;
        for (int j = 0; j < 16; ++j) {
            float a = fabsf(blk[j]);
            if (a > bmax) bmax = a;
        }
        float r = bmax / six_st;
        int sb = orc_e4m3_rne(r);
        scales[b] = (uint8_t)sb;
        float sval = (float)orc_e4m3(sb);
        float denom = sval * s_t;
        for (int j = 0; j < 8; ++j) {
            int lo = 0, hi = 0;
            if (sval != 0.0f) {
                lo = orc_e2m1_rne(blk[2 * j] / denom);
                hi = orc_e2m1_rne(blk[2 * j + 1] / denom);
            }
            codes[b * 8 + j] = (uint8_t)(lo | (hi << 4));
        }
    }
}

/* value of quantized element i */
static double dq_act(const uint8_t *codes, const uint8_t *scales, int64_t i, double s_t) {
    int code = (i % 2 == 0) ? (codes[i / 2] & 0xF) : (codes[i / 2] >> 4);
    return orc_e2m1(code) * orc_e4m3(scales[i / 16]) * s_t;
}

/* W4A4 expert for one row (the prefill path): x is quantized with its own
 * row scale, the products are taken in fp64, h is rounded to fp32 and
 * quantized with its own row scale before the down projection. */
EXPORT void orc_expert_w4a4(const uint8_t *rec, int d, int F, const uint16_t *x, double *y) {
    int64_t off[6];
    orc_record_layout(d, F, off);
    float *xf = (float *)malloc(sizeof(float) * d);
    uint8_t *xc = (uint8_t *)malloc((size_t)d / 2), *xs = (uint8_t *)malloc((size_t)d / 16);
    double *xv = (double *)malloc(sizeof(double) * d);
    for (int K = 0; K < d; ++K) xf[K] = (float)bf16_val(x[K]);
    float sx = orc_tensor_scale_f32(xf, d);
    orc_nvfp4_quantize(xf, d, sx, xc, xs);
    for (int K = 0; K < d; ++K) xv[K] = dq_act(xc, xs, K, sx);

    double tg = rec_tensor_scale(rec, off, 0), tu = rec_tensor_scale(rec, off, 1);
    double td = rec_tensor_scale(rec, off, 2);
    float *hf = (float *)malloc(sizeof(float) * F);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < F; ++j) {
        double g = 0.0, u = 0.0;
        for (int64_t K = 0; K < d; ++K) {
            g += dq(rec + off[0], rec + off[1], d, 2 * j, K, tg) * xv[K];
            u += dq(rec + off[0], rec + off[1], d, 2 * j + 1, K, tu) * xv[K];
        }
        hf[j] = (float)(silu(g) * u);
    }
    uint8_t *hc = (uint8_t *)malloc((size_t)F / 2), *hs = (uint8_t *)malloc((size_t)F / 16);
    float sh = orc_tensor_scale_f32(hf, F);
    orc_nvfp4_quantize(hf, F, sh, hc, hs);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < F; ++j)
            acc += dq(rec + off[2], rec + off[3], F, i, j, td) * dq_act(hc, hs, j, sh);
        y[i] = acc;
    }
    free(xf); free(xc); free(xs); free(xv); free(hf); free(hc); free(hs);
}

/* ------------------------------------------ MXFP4 activation quantizer -- */
/* OCP microscaling, per block of 32 consecutive values: shared exponent
 * e = floor(log2(amax)) - 2 (2 = the largest E2M1 exponent), clamped to
 * [-127, 127], stored as the E8M0 code e + 127; element code = E2M1 of
 * x / 2^e, RNE, saturating to +-6.  An all-zero block gets code 0 and zero
 * elements.  Every step is exact in fp32 (amax, the exponent, the division by
 * a power of two), so the codes do not depend on the precision it runs in.
 * n a multiple of 32; codes n/2 bytes (element 2i in the low nibble), scales n/32. */
EXPORT void orc_mx_quantize(const float *x, int64_t n, uint8_t *codes, uint8_t *scales) {
    for (int64_t b = 0; b < n / 32; ++b) {
        const float *blk = x + b * 32;
        float amax = 0.0f;
        for (int j = 0; j < 32; ++j) {
            float a = fabsf(blk[j]);
            if (a > amax) amax = a;
        }
        int e = -127;
        if (amax > 0.0f) {
            int ex;
            frexpf(amax, &ex); /* amax = f * 2^ex, f in [0.5, 1): floor(log2 amax) = ex - 1 */
            e = ex - 1 - 2;
            if (e < -127) e = -127;
            if (e > 127) e = 127;
        }
        scales[b] = (uint8_t)(e + 127);
        for (int j = 0; j < 16; ++j) {
            int lo = 0, hi = 0;
            if (amax > 0.0f) {
                lo = orc_e2m1_rne(ldexpf(blk[2 * j], -e));
                hi = orc_e2m1_rne(ldexpf(blk[2 * j + 1], -e));
            }
            codes[b * 16 + j] = (uint8_t)(lo | (hi << 4));
        }
    }
}

static double dq_act_mx(const uint8_t *codes, const uint8_t *scales, int64_t i) {
    int code = (i % 2 == 0) ? (codes[i / 2] & 0xF) : (codes[i / 2] >> 4);
    return orc_e2m1(code) * orc_e8m0(scales[i / 32]);
}

/* W4A4 expert over an MXFP4 record for one row (the prefill path with MXFP4
 * records): x is MXFP4-quantized per block of 32, the products are taken in
 * fp64, h is rounded to fp32 and MXFP4-quantized before the down projection
 * (the same steps as the NVFP4 W4A4 expert, with E8M0 block scales and no
 * row scale). */
EXPORT void orc_expert_mx_w4a4(const uint8_t *rec, int d, int F, const uint16_t *x, double *y) {
    int64_t off[5];
    orc_mx_record_layout(d, F, off);
    float *xf = (float *)malloc(sizeof(float) * d);
    uint8_t *xc = (uint8_t *)malloc((size_t)d / 2), *xs = (uint8_t *)malloc((size_t)d / 32);
    double *xv = (double *)malloc(sizeof(double) * d);
    for (int K = 0; K < d; ++K) xf[K] = (float)bf16_val(x[K]);
    orc_mx_quantize(xf, d, xc, xs);
    for (int K = 0; K < d; ++K) xv[K] = dq_act_mx(xc, xs, K);
    float *hf = (float *)malloc(sizeof(float) * F);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < F; ++j) {
        double g = 0.0, u = 0.0;
        for (int64_t K = 0; K < d; ++K) {
            g += dq_mx(rec + off[0], rec + off[1], d, 2 * j, K) * xv[K];
            u += dq_mx(rec + off[0], rec + off[1], d, 2 * j + 1, K) * xv[K];
        }
        hf[j] = (float)(silu(g) * u);
    }
    uint8_t *hc = (uint8_t *)malloc((size_t)F / 2), *hs = (uint8_t *)malloc((size_t)F / 32);
    orc_mx_quantize(hf, F, hc, hs);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < F; ++j) acc += dq_mx(rec + off[2], rec + off[3], F, i, j) * dq_act_mx(hc, hs, j);
        y[i] = acc;
    }
    free(xf); free(xc); free(xs); free(xv); free(hf); free(hc); free(hs);
}

/* ------------------------------------------------------------ one layer -- */
/* Record of (layer, expert) in a host pool of P records: index (layer*E + expert) mod P. */
static const uint8_t *pool_record(const uint8_t *pool, int64_t P, int64_t rec_bytes, int layer,
                                  int E, int e) {
    return pool + (((int64_t)layer * E + e) % P) * rec_bytes;
}

/* One expert on one bf16 row in the record's format: 0 NVFP4, 1 MXFP4 (W4A16,
 * or W4A4 with w4a4), 2 BF16 (weights and activations as they are, both paths). */
static void expert_fmt(const uint8_t *rec, int fmt, int w4a4, int d, int F, const uint16_t *x, double *y) {
    if (fmt == 1 && w4a4) orc_expert_mx_w4a4(rec, d, F, x, y);
    else if (fmt == 1) orc_expert_mx_w4a16(rec, d, F, x, y);
    else if (fmt == 2) orc_expert_bf16((const uint16_t *)rec, d, F, x, y);
    else if (w4a4) orc_expert_w4a4(rec, d, F, x, y);
    else orc_expert_w4a16(rec, d, F, x, y, NULL);
}

/* One MoE layer on T independent rows: route, then
 * y = sum over selected e in ascending id of g_e * E_e(x) + S(x).
 * fmt: the routed records' format (0 NVFP4, 1 MXFP4); shared_fmt: the shared
 * record's (0, 1 or 2 BF16).  w4a4 = 0: decode path (W4A16); 1: prefill path
 * (W4A4: NVFP4 or MXFP4 activations to match the records; a BF16 shared
 * expert is not quantized).  shared_rec may be NULL (no shared expert). */
EXPORT int orc_moe_layer_fmt(const uint8_t *pool, int64_t P, int layer, int E, int d, int F, int k,
                             int renorm, const uint16_t *Wr_layer, const uint8_t *shared_rec,
                             const uint16_t *x, int T, int w4a4, int fmt, int shared_fmt, int32_t *idx,
                             double *gates, double *y) {
    if (fmt < 0 || fmt > 1 || shared_fmt < 0 || shared_fmt > 2 || (shared_fmt != fmt && shared_fmt != 2)) return 1;
    int64_t off[6];
    if (fmt == 1) orc_mx_record_layout(d, F, off);
    else orc_record_layout(d, F, off);
    const int64_t rec_bytes = fmt == 1 ? off[4] : off[5];
    int rc = orc_route(Wr_layer, x, T, E, d, k, renorm, idx, gates, NULL, NULL);
    if (rc) return rc;
    double *ye = (double *)malloc(sizeof(double) * d);
    for (int t = 0; t < T; ++t) {
        const uint16_t *xr = x + (int64_t)t * d;
        double *yr = y + (int64_t)t * d;
        for (int i = 0; i < d; ++i) yr[i] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = idx[(int64_t)t * k + j];
            expert_fmt(pool_record(pool, P, rec_bytes, layer, E, e), fmt, w4a4, d, F, xr, ye);
            double g = gates[(int64_t)t * k + j];
            for (int i = 0; i < d; ++i) yr[i] += g * ye[i];
        }
        if (shared_rec) {
            expert_fmt(shared_rec, shared_fmt, w4a4, d, F, xr, ye);
            for (int i = 0; i < d; ++i) yr[i] += ye[i];
        }
    }
    free(ye);
    return 0;
}

/* The layer with NVFP4 records throughout. */
EXPORT int orc_moe_layer(const uint8_t *pool, int64_t P, int layer, int E, int d, int F, int k,
                         int renorm, const uint16_t *Wr_layer, const uint8_t *shared_rec,
                         const uint16_t *x, int T, int w4a4, int32_t *idx, double *gates,
                         double *y) {
    return orc_moe_layer_fmt(pool, P, layer, E, d, F, k, renorm, Wr_layer, shared_rec, x, T, w4a4, 0, 0,
                             idx, gates, y);
}

/* --------------------------------------------------------- LRU simulator -- */
typedef struct {
    int64_t L, E, C;
    int32_t *map;    /* [L*E] slot of key, -1 if absent */
    int32_t *owner;  /* [C] key in slot, -1 if free */
    uint64_t *stamp; /* [C] last-use clock of slot */
    uint64_t clock;
} orc_lru;

EXPORT orc_lru *orc_lru_new(int64_t L, int64_t E, int64_t C) {
    if (L <= 0 || E <= 0 || C <= 0) return NULL;
    orc_lru *s = (orc_lru *)calloc(1, sizeof(orc_lru));
    s->L = L; s->E = E; s->C = C;
    s->map = (int32_t *)malloc(sizeof(int32_t) * L * E);
    s->owner = (int32_t *)malloc(sizeof(int32_t) * C);
    s->stamp = (uint64_t *)calloc((size_t)C, sizeof(uint64_t));
    for (int64_t i = 0; i < L * E; ++i) s->map[i] = -1;
    for (int64_t i = 0; i < C; ++i) s->owner[i] = -1;
    return s;
}

EXPORT void orc_lru_free(orc_lru *s) {
    if (!s) return;
    free(s->map); free(s->owner); free(s->stamp); free(s);
}

EXPORT void orc_lru_state(const orc_lru *s, int32_t *map, int32_t *owner, uint64_t *stamp,
                          uint64_t *clock) {
    if (map) memcpy(map, s->map, sizeof(int32_t) * s->L * s->E);
    if (owner) memcpy(owner, s->owner, sizeof(int32_t) * s->C);
    if (stamp) memcpy(stamp, s->stamp, sizeof(uint64_t) * s->C);
    if (clock) *clock = s->clock;
}

/* One lookup batch of layer `layer`: experts[0..n) distinct and ascending.
 * Hits get ++clock in ascending id; then each miss, in ascending id, takes the
 * free slot with the lowest index, or else the slot with the smallest stamp
 * (ties: lowest index), evicting its owner, and gets ++clock.
 * Per entry: ev_slot, ev_hit (1/0), ev_evicted (evicted key or -1).
 * Returns the number of misses, or -1 on bad input (not ascending, out of
 * range, n > C). */
EXPORT int orc_lru_batch(orc_lru *s, int layer, const int32_t *experts, int n, int32_t *ev_slot,
                         int32_t *ev_hit, int64_t *ev_evicted) {
    if (layer < 0 || layer >= s->L || n < 0 || n > s->C) return -1;
    for (int i = 0; i < n; ++i) {
        if (experts[i] < 0 || experts[i] >= s->E) return -1;
        if (i > 0 && experts[i] <= experts[i - 1]) return -1;
    }
    for (int i = 0; i < n; ++i) {
        int64_t key = (int64_t)layer * s->E + experts[i];
        int32_t slot = s->map[key];
        ev_hit[i] = slot >= 0;
        ev_slot[i] = slot;
        ev_evicted[i] = -1;
        if (slot >= 0) s->stamp[slot] = ++s->clock;
    }
    int misses = 0;
    for (int i = 0; i < n; ++i) {
        if (ev_hit[i]) continue;
        ++misses;
        int64_t key = (int64_t)layer * s->E + experts[i];
        int64_t victim = -1;
        for (int64_t c = 0; c < s->C; ++c)
            if (s->owner[c] < 0) { victim = c; break; }
        if (victim < 0) {
            victim = 0;
            for (int64_t c = 1; c < s->C; ++c)
                if (s->stamp[c] < s->stamp[victim]) victim = c;
            int32_t old = s->owner[victim];
            s->map[old] = -1;
            ev_evicted[i] = old;
        }
        s->owner[victim] = (int32_t)key;
        s->map[key] = (int32_t)victim;
        s->stamp[victim] = ++s->clock;
        ev_slot[i] = (int32_t)victim;
    }
    return misses;
}

/* ------------------------------------------------------------- planner -- */
/* Split m missing experts between the PCIe transfer (bandwidth B_P) and the
 * host-side processing (bandwidth B_H, of which max(B_H - B_P, 0) is left
 * while the DMA reads host memory).  Equal finish times,
 * q/B_P = (m - q)/(B_H - B_P), give q = m*B_P/B_H for B_H > B_P.
 * mode 1 (hybrid) iff B_H/B_P > threshold, else 0 (offload: all m over PCIe).
 * q_real: the real-valued formula (m when B_H <= B_P); q: the executed count,
 * round half up of q_real in hybrid mode, m in offload mode.
 * t_finish: finish time of the executed split for experts of expert_bytes. */
EXPORT int orc_plan_split(int m, double B_P, double B_H, double threshold, double expert_bytes,
                          int *q, int *cpu, int *mode, double *q_real, double *t_finish) {
    if (m < 0 || !(B_P > 0) || !(B_H >= 0) || !(expert_bytes > 0)) return -1;
    double qr = (B_H > B_P) ? (double)m * B_P / B_H : (double)m;
    int md = (B_H > B_P && B_H / B_P > threshold) ? 1 : 0;
    int qi = md ? (int)floor(qr + 0.5) : m;
    if (qi > m) qi = m;
    *q = qi;
    *cpu = m - qi;
    *mode = md;
    *q_real = qr;
    double t_pcie = qi * expert_bytes / B_P;
    double t_cpu = (m - qi) > 0 ? (m - qi) * expert_bytes / (B_H - B_P) : 0.0;
    *t_finish = t_pcie > t_cpu ? t_pcie : t_cpu;
    return 0;
}
