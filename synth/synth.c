/*
 * synth.c -- seeded synthetic inputs for the per-layer routed-expert step.
 *
 * This module makes INPUTS only: random draws, the NVFP4 encoding of the
 * synthetic expert weights, bf16 rounding of router weights and hidden states,
 * and the AR(1) hidden-state recurrence.  It holds none of the step's own
 * arithmetic (no routing, no decode of NVFP4, no expert FFN, no cache).  Both
 * the CPU oracle and the CUDA path are fed from the bytes written here.
 *
 * Random numbers: SplitMix64 (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014; constants as in Vigna's
 * public-domain splitmix64.c) used as a counter-based generator: a stream key
 * is hashed from (seed, purpose, a, b, c, d) and draw i of the stream is
 * mix(key ^ mix(i)).  Normals use the Box-Muller transform (Box & Muller,
 * 1958) on the uniforms at counters 2i and 2i+1, cosine branch only.
 *
 * Weight encoding (NVFP4: E2M1 values, one E4M3 scale per 16 consecutive
 * elements of a row, one fp32 scale per matrix; the format the FreeToken
 * pages name for routed experts in "NVFP4で約135GBまで縮める"), in fp32 with
 * round-to-nearest-even, in this order:
 *   s_t   = amax(tensor) / 2688            (2688 = 6 * 448; s_t = 1 if amax = 0)
 *   r     = amax(block) / (6 * s_t)
 *   sb    = E4M3(r), RNE, saturating to 448
 *   denom = value(sb) * s_t
 *   code  = E2M1(x / denom), RNE, saturating to 6   (all codes 0 if value(sb) = 0)
 *
 * Expert record (one contiguous block per (layer, expert)):
 *   3 fp32 tensor scales (gate, up, down), padded to 256 B
 *   W13 codes  [2F x d/2] bytes, rows interleaved: row 2j = gate_j, 2j+1 = up_j;
 *              two codes per byte, element 2i in the low nibble
 *   W13 scales [2F x d/16] E4M3 bytes
 *   W2 codes   [d x F/2] bytes (row = output dim, K = F)
 *   W2 scales  [d x F/16]
 * each section starting on a 256-byte boundary, the whole padded to 256 B.
 * (The gate/up half -- tensor scales and W13 -- is a contiguous prefix.)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

/* ---------------------------------------------------------------- RNG -- */
static inline uint64_t mix64(uint64_t x) {
    x += 0x9E3779B97F4A7C15ull;
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return x ^ (x >> 31);
}

EXPORT uint64_t synth_key(uint64_t seed, uint64_t purpose, uint64_t a, uint64_t b,
                          uint64_t c, uint64_t d) {
    uint64_t k = mix64(seed);
    k = mix64(k ^ purpose);
    k = mix64(k ^ a);
    k = mix64(k ^ b);
    k = mix64(k ^ c);
    k = mix64(k ^ d);
    return k;
}

static inline double uniform01(uint64_t key, uint64_t i) {
    uint64_t u = mix64(key ^ mix64(i));
    return ((double)(u >> 11) + 0.5) * (1.0 / 9007199254740992.0); /* (0,1) */
}

static inline double normal01(uint64_t key, uint64_t i) {
    double u1 = uniform01(key, 2 * i), u2 = uniform01(key, 2 * i + 1);
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

/* n draws of N(0, sigma^2), rounded to fp32. */
EXPORT void synth_normals_f32(uint64_t key, int64_t n, double sigma, float *out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)(sigma * normal01(key, (uint64_t)i));
}

/* --------------------------------------------------------------- bf16 -- */
static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

EXPORT void synth_to_bf16(const float *x, int64_t n, uint16_t *out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(x[i]);
}

/* Router weights of one layer: [E x d] N(0, sigma^2) rounded to bf16. */
EXPORT void synth_router_bf16(uint64_t seed, int32_t layer, int32_t E, int32_t d, double sigma,
                              uint16_t *out) {
    uint64_t key = synth_key(seed, 2, (uint64_t)layer, 0, 0, 0);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)E * d; ++i)
        out[i] = f32_to_bf16_rne((float)(sigma * normal01(key, (uint64_t)i)));
}

/* Hidden-state noise eps in R^d for (purpose, stream, layer, t, attempt), N(0,1) in fp32. */
EXPORT void synth_noise_f32(uint64_t seed, int32_t purpose, int32_t stream, int32_t layer,
                            int64_t t, int32_t attempt, int32_t d, float *out) {
    uint64_t key = synth_key(seed, (uint64_t)purpose, (uint64_t)stream, (uint64_t)layer,
                             (uint64_t)t, (uint64_t)attempt);
    for (int32_t i = 0; i < d; ++i) out[i] = (float)normal01(key, (uint64_t)i);
}

/* One AR(1) step in fp32: x_t = rho*x_{t-1} + sqrt(1-rho^2)*eps_t; x_0 = eps_0 (t == 0). */
EXPORT void synth_ar1_step(const float *x_prev, const float *eps, int32_t d, int64_t t,
                           float rho, float *x_out) {
    float c = sqrtf(1.0f - rho * rho);
    for (int32_t i = 0; i < d; ++i) x_out[i] = (t == 0) ? eps[i] : rho * x_prev[i] + c * eps[i];
}

/* ------------------------------------------------------- NVFP4 encode -- */
/* Non-negative finite E4M3 ("fn" variant: bias 7, no inf, 0x7F NaN) values, by code. */
static float g_e4m3_pos[127];
static int g_tables_ready = 0;
static const float g_e2m1_mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

static void build_tables(void) {
    if (g_tables_ready) return;
    for (int c = 0; c < 127; ++c) {
        int e = (c >> 3) & 0xF, m = c & 7;
        g_e4m3_pos[c] = e == 0 ? ldexpf((float)m, -9) : ldexpf(1.0f + m / 8.0f, e - 7);
    }
    g_tables_ready = 1;
}

/* RNE to the nearest of an ascending table; ties go to the even index. */
static int rne_index(const float *tab, int n, float v) {
    int lo = 0, hi = n - 1;
    if (v >= tab[hi]) return hi; /* saturate */
    while (hi - lo > 1) {        /* tab[lo] <= v < tab[hi] */
        int mid = (lo + hi) >> 1;
        if (tab[mid] <= v) lo = mid; else hi = mid;
    }
    float dl = v - tab[lo], dh = tab[hi] - v;
    if (dl < dh) return lo;
    if (dh < dl) return hi;
    return (lo & 1) ? hi : lo;
}

static inline uint8_t e4m3_encode_pos(float r) { return (uint8_t)rne_index(g_e4m3_pos, 127, r); }

static inline uint8_t e2m1_encode(float v) {
    uint8_t s = signbit(v) ? 8 : 0;
    return (uint8_t)(s | rne_index(g_e2m1_mag, 8, fabsf(v)));
}

/* Encode a row-major [rows x K] fp32 matrix.  Row r, element k goes to
 * codes[(out_row(r)) * K/2 + k/2] (low nibble for even k), scales likewise
 * with one byte per 16 elements; out_row(r) = r*row_mul + row_add. */
static float encode_matrix(const float *w, int64_t rows, int64_t K, int64_t row_mul,
                           int64_t row_add, uint8_t *codes, uint8_t *scales) {
    float amax = 0.0f;
    for (int64_t i = 0; i < rows * K; ++i) amax = fmaxf(amax, fabsf(w[i]));
    float s_t = amax > 0.0f ? amax / 2688.0f : 1.0f;
    float six_st = 6.0f * s_t;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t orow = r * row_mul + row_add;
        for (int64_t b = 0; b < K / 16; ++b) {
            const float *blk = w + r * K + b * 16;
            float bmax = 0.0f;
            for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf(blk[j]));
            float ratio = bmax / six_st;
            uint8_t sb = e4m3_encode_pos(ratio);
            scales[orow * (K / 16) + b] = sb;
            float denom = g_e4m3_pos[sb] * s_t;
            uint8_t *cb = codes + orow * (K / 2) + b * 8;
            for (int j = 0; j < 8; ++j) {
                uint8_t lo = 0, hi = 0;
                if (g_e4m3_pos[sb] != 0.0f) {
                    lo = e2m1_encode(blk[2 * j] / denom);
                    hi = e2m1_encode(blk[2 * j + 1] / denom);
                }
                cb[j] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
    return s_t;
}

static inline int64_t align256(int64_t x) { return (x + 255) & ~(int64_t)255; }

/* Section offsets of one record: [w13 codes, w13 scales, w2 codes, w2 scales, tensor scales, total]. */
EXPORT void synth_record_layout(int32_t d, int32_t F, int64_t *off) {
    int64_t dd = d, ff = F;
    off[4] = 0;                     /* tensor scales at the head */
    off[0] = align256(12);
    off[1] = off[0] + align256(2 * ff * dd / 2);
    off[2] = off[1] + align256(2 * ff * dd / 16);
    off[3] = off[2] + align256(dd * ff / 2);
    off[5] = off[3] + align256(dd * ff / 16);
}

/* One expert record from N(0, sigma^2) fp32 draws keyed by (purpose, layer, expert, matrix).
 * purpose 1 = routed expert, 5 = shared expert.  Writes off[5] bytes at rec. */
EXPORT void synth_expert_record(uint64_t seed, int32_t purpose, int32_t layer, int32_t expert,
                                int32_t d, int32_t F, double sigma, uint8_t *rec) {
    build_tables();
    int64_t off[6];
    synth_record_layout(d, F, off);
    memset(rec, 0, (size_t)off[5]);
    int64_t n = (int64_t)F * d;
    float *w = (float *)malloc((size_t)n * sizeof(float));
    float ts[3];
    for (int m = 0; m < 3; ++m) {
        uint64_t key = synth_key(seed, (uint64_t)purpose, (uint64_t)layer, (uint64_t)expert,
                                 (uint64_t)m, 0);
        synth_normals_f32(key, n, sigma, w);
        if (m < 2) /* gate (m=0) -> rows 2j, up (m=1) -> rows 2j+1; [F x d] */
            ts[m] = encode_matrix(w, F, d, 2, m, rec + off[0], rec + off[1]);
        else       /* down: [d x F] */
            ts[m] = encode_matrix(w, d, F, 1, 0, rec + off[2], rec + off[3]);
    }
    memcpy(rec + off[4], ts, sizeof ts);
    free(w);
}

/* ------------------------------------------------------- MXFP4 encode -- */
/* MXFP4 (OCP Microscaling formats: E2M1 elements, one E8M0 scale 2^(c - 127)
 * per 32 consecutive elements, no tensor scale).  Per block: shared exponent
 * e = floor(log2(amax)) - 2 (2 = the largest E2M1 exponent), clamped to
 * [-127, 127]; scale code e + 127; element code E2M1(x / 2^e), RNE, saturating
 * to 6.  An all-zero block gets scale code 0 and zero codes. */
static void encode_matrix_mx(const float *w, int64_t rows, int64_t K, int64_t row_mul,
                             int64_t row_add, uint8_t *codes, uint8_t *scales) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t orow = r * row_mul + row_add;
        for (int64_t b = 0; b < K / 32; ++b) {
            const float *blk = w + r * K + b * 32;
            float amax = 0.0f;
            for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(blk[j]));
            int e = -127;
            if (amax > 0.0f) {
                int ex;
                frexpf(amax, &ex); /* amax = m * 2^ex, m in [0.5, 1): floor(log2 amax) = ex - 1 */
                e = ex - 1 - 2;
                if (e < -127) e = -127;
                if (e > 127) e = 127;
            }
            scales[orow * (K / 32) + b] = (uint8_t)(e + 127);
            uint8_t *cb = codes + orow * (K / 2) + b * 16;
            for (int j = 0; j < 16; ++j) {
                uint8_t lo = 0, hi = 0;
                if (amax > 0.0f) {
                    lo = e2m1_encode(ldexpf(blk[2 * j], -e));
                    hi = e2m1_encode(ldexpf(blk[2 * j + 1], -e));
                }
                cb[j] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* MXFP4 codes and scales of a row-major [rows x K] fp32 matrix (K a multiple of 32). */
EXPORT void synth_mx_encode(const float *w, int64_t rows, int64_t K, uint8_t *codes, uint8_t *scales) {
    build_tables();
    encode_matrix_mx(w, rows, K, 1, 0, codes, scales);
}

/* Section offsets of one MXFP4 record: [w13 codes, w13 scales, w2 codes, w2 scales, total];
 * the same row order as the NVFP4 record (W13 row 2j = gate_j, 2j+1 = up_j). */
EXPORT void synth_mx_record_layout(int32_t d, int32_t F, int64_t *off) {
    int64_t dd = d, ff = F;
    off[0] = 0;
    off[1] = off[0] + align256(2 * ff * dd / 2);
    off[2] = off[1] + align256(2 * ff * dd / 32);
    off[3] = off[2] + align256(dd * ff / 2);
    off[4] = off[3] + align256(dd * ff / 32);
}

/* The MXFP4 record of the same fp32 draws as synth_expert_record. */
EXPORT void synth_expert_record_mx(uint64_t seed, int32_t purpose, int32_t layer, int32_t expert,
                                   int32_t d, int32_t F, double sigma, uint8_t *rec) {
    build_tables();
    int64_t off[5];
    synth_mx_record_layout(d, F, off);
    memset(rec, 0, (size_t)off[4]);
    int64_t n = (int64_t)F * d;
    float *w = (float *)malloc((size_t)n * sizeof(float));
    for (int m = 0; m < 3; ++m) {
        uint64_t key = synth_key(seed, (uint64_t)purpose, (uint64_t)layer, (uint64_t)expert,
                                 (uint64_t)m, 0);
        synth_normals_f32(key, n, sigma, w);
        if (m < 2)
            encode_matrix_mx(w, F, d, 2, m, rec + off[0], rec + off[1]);
        else
            encode_matrix_mx(w, d, F, 1, 0, rec + off[2], rec + off[3]);
    }
    free(w);
}

/* A BF16 expert record of the same fp32 draws (the checkpoints keep shared
 * experts in BF16): W13 [2F x d] (row 2j = gate_j, 2j+1 = up_j), then W2 [d x F],
 * bf16 RNE; 2 * 3dF bytes. */
EXPORT void synth_expert_record_bf16(uint64_t seed, int32_t purpose, int32_t layer, int32_t expert,
                                     int32_t d, int32_t F, double sigma, uint16_t *rec) {
    int64_t n = (int64_t)F * d;
    float *w = (float *)malloc((size_t)n * sizeof(float));
    for (int m = 0; m < 3; ++m) {
        uint64_t key = synth_key(seed, (uint64_t)purpose, (uint64_t)layer, (uint64_t)expert,
                                 (uint64_t)m, 0);
        synth_normals_f32(key, n, sigma, w);
        if (m < 2) {
            for (int64_t j = 0; j < F; ++j)
                for (int64_t i = 0; i < d; ++i) rec[(2 * j + m) * d + i] = f32_to_bf16_rne(w[j * d + i]);
        } else {
            for (int64_t i = 0; i < n; ++i) rec[2 * n + i] = f32_to_bf16_rne(w[i]);
        }
    }
    free(w);
}

/* The fp32 draws behind matrix m of a record (for checking the encoding). */
EXPORT void synth_expert_matrix_f32(uint64_t seed, int32_t purpose, int32_t layer,
                                    int32_t expert, int32_t m, int32_t d, int32_t F,
                                    double sigma, float *out) {
    uint64_t key = synth_key(seed, (uint64_t)purpose, (uint64_t)layer, (uint64_t)expert,
                             (uint64_t)m, 0);
    synth_normals_f32(key, (int64_t)F * d, sigma, out);
}

/* Fill n_dst records by repeating the first n_src records of buf (record i := record i mod n_src). */
EXPORT void synth_replicate_records(uint8_t *buf, int64_t record_bytes, int64_t n_src,
                                    int64_t n_dst) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = n_src; i < n_dst; ++i)
        memcpy(buf + i * record_bytes, buf + (i % n_src) * record_bytes, (size_t)record_bytes);
}

/* T prefill rows of one layer (i.i.d. N(0,1), attempt 0), bf16 [T x d]. */
EXPORT void synth_prefill_rows_bf16(uint64_t seed, int32_t layer, int32_t T, int32_t d,
                                    uint16_t *out) {
#pragma omp parallel for schedule(static)
    for (int32_t t = 0; t < T; ++t) {
        uint64_t key = synth_key(seed, 4, 0, (uint64_t)layer, (uint64_t)t, 0);
        for (int32_t i = 0; i < d; ++i)
            out[(int64_t)t * d + i] = f32_to_bf16_rne((float)normal01(key, (uint64_t)i));
    }
}
