// NVFP4 and MXFP4 activation quantizers (the W4A4 prefill path) and the prefill combine.
//
// The routed experts of the checkpoint are W4A4 NVFP4 (florigen.ai,
// "NVFP4で約135GBまで縮める"): activations are quantized like the weights --
// E2M1 values, one E4M3 scale per 16 consecutive elements, one fp32 scale --
// here with one fp32 scale per row (a token's x, or a token's h for one
// expert).  In fp32 with round-to-nearest-even, in this order:
//   s_t = amax(row) / 2688 (1 if amax = 0); r = amax(block) / (6 s_t);
//   sb = E4M3(r), saturating; denom = value(sb) * s_t; code = E2M1(v / denom),
//   saturating; all codes 0 when value(sb) = 0.
// The conversions are the hardware RNE ones (cvt.rn.satfinite.{e4m3x2,e2m1x2}.f32).
// The rows are written in expert-grouped order (a token's x once per expert
// that it selected, then once more for the shared expert) as NVFP4 codes,
// block scales and row scales: the operands of the block-scaled tensor-core
// GEMMs, which apply s_t in their epilogue.
#include "moe_internal.cuh"

namespace moe {

namespace {

__device__ __forceinline__ uint32_t e4m3_code(float r) {  // r >= 0
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(out) : "f"(r), "f"(0.0f));
    return out & 0xffu;
}
__device__ __forceinline__ float e4m3_value(uint32_t code) {
    uint32_t r;
    const uint16_t s = (uint16_t)code;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(s));
    return __low2float(*reinterpret_cast<__half2 *>(&r));
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// One warp quantizes one row of n values (n a multiple of 16) and writes the
// NVFP4 encoding itself: codes (two per byte, even element in the low nibble),
// one E4M3 scale per 16 values and the row's fp32 scale s_t.
template <typename LoadFn>
__device__ void quant_row_codes(LoadFn load, int n, uint8_t *codes, uint8_t *scales, float *st) {
    const int lane = threadIdx.x & 31;
    float amax = 0.f;
    for (int i = lane; i < n; i += 32) amax = fmaxf(amax, fabsf(load(i)));
    amax = warp_max(amax);
    const float s_t = amax > 0.f ? amax / 2688.0f : 1.0f;
    const float six_st = 6.0f * s_t;
    for (int b = lane; b < n / 16; b += 32) {
        float v[16];
        float bmax = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            v[j] = load(16 * b + j);
            bmax = fmaxf(bmax, fabsf(v[j]));
        }
        const uint32_t sc = e4m3_code(bmax / six_st);
        const float sval = e4m3_value(sc);
        const float denom = sval * s_t;
        uint32_t word[2] = {0u, 0u};
        if (sval != 0.f) {
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
                uint16_t c;
                asm("{\n\t.reg .b8 c8;\n\t"
                    "cvt.rn.satfinite.e2m1x2.f32 c8, %2, %1;\n\t"
                    "cvt.u16.u8 %0, c8;\n\t}"
                    : "=h"(c)
                    : "f"(v[j] / denom), "f"(v[j + 1] / denom));
                word[j >> 3] |= (uint32_t)(c & 0xffu) << (4 * (j & 7));
            }
        }
        *reinterpret_cast<uint2 *>(codes + 8 * b) = make_uint2(word[0], word[1]);
        scales[b] = (uint8_t)sc;
    }
    if (lane == 0) *st = s_t;
}

// MXFP4 activations (OCP microscaling; the W4A4 path over MXFP4 records): one
// E8M0 scale 2^e per 32 values, e = floor(log2 amax(block)) - 2 clamped to
// [-127, 127] (-127 for an all-zero block), codes E2M1(v * 2^-e), RNE and
// saturating, no row scale.  Multiplying by the power of two 2^-e is exact
// (or, below fp32's normal range, correctly rounded like the oracle's ldexpf),
// so every decision is the oracle's.
__device__ __forceinline__ int mx_exponent(float amax) {
    const uint32_t eb = (__float_as_uint(amax) >> 23) & 0xffu;
    if (amax == 0.f || eb == 0u) return -127;  // zero or subnormal: floor(log2) - 2 < -127
    const int e = (int)eb - 127 - 2;
    return e > 127 ? 127 : e;
}
__device__ __forceinline__ float pow2f(int e) {  // 2^e for e in [-149, 127], exact
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(1u << (e + 149));
}
template <typename LoadFn>
__device__ void quant_row_codes_mx(LoadFn load, int n, uint8_t *codes, uint8_t *scales) {
    const int lane = threadIdx.x & 31;
    for (int b = lane; b < n / 32; b += 32) {
        float v[32];
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            v[j] = load(32 * b + j);
            amax = fmaxf(amax, fabsf(v[j]));
        }
        const int e = mx_exponent(amax);
        const float inv = pow2f(-e);
        uint32_t word[4] = {0u, 0u, 0u, 0u};
        if (amax > 0.f) {
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                uint16_t c;
                asm("{\n\t.reg .b8 c8;\n\t"
                    "cvt.rn.satfinite.e2m1x2.f32 c8, %2, %1;\n\t"
                    "cvt.u16.u8 %0, c8;\n\t}"
                    : "=h"(c)
                    : "f"(v[j] * inv), "f"(v[j + 1] * inv));
                word[j >> 3] |= (uint32_t)(c & 0xffu) << (4 * (j & 7));
            }
        }
        *reinterpret_cast<uint4 *>(codes + 16 * b) = make_uint4(word[0], word[1], word[2], word[3]);
        scales[b] = (uint8_t)(e + 127);
    }
}

// Grouped rows of x for the tensor-core GEMMs: row g < T*k is token
// rowrefs[g].t, row T*k + t (shared expert) is token t; one warp per row.
__global__ void quant_x_grouped_kernel(const __nv_bfloat16 *__restrict__ x, int T, int k, int d,
                                       int has_shared, const RowRef *__restrict__ rowrefs,
                                       const int32_t *__restrict__ n_routed, uint8_t *codes, uint8_t *scales,
                                       float *st, int mx) {
    const int g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int tk = T * k;
    if (g >= tk + (has_shared ? T : 0) || (g < tk && g >= *n_routed)) return;
    const int t = g < tk ? rowrefs[g].t : g - tk;
    const __nv_bfloat16 *row = x + (size_t)t * d;
    auto load = [&](int i) { return __bfloat162float(row[i]); };
    if (mx) quant_row_codes_mx(load, d, codes + (size_t)g * (d / 2), scales + (size_t)g * (d / 32));
    else quant_row_codes(load, d, codes + (size_t)g * (d / 2), scales + (size_t)g * (d / 16), st + g);
}

// Grouped h rows (fp32 [rows][F]) -> NVFP4 codes, scales, row scales; one warp per row.
__global__ void quant_h_grouped_kernel(const float *__restrict__ h32, int T, int k, int has_shared,
                                       const int32_t *__restrict__ n_routed, int F, uint8_t *codes,
                                       uint8_t *scales, float *st, int mx) {
    const int g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int tk = T * k;
    if (g >= tk + (has_shared ? T : 0) || (g < tk && g >= *n_routed)) return;
    const float *row = h32 + (size_t)g * F;
    auto load = [&](int i) { return row[i]; };
    if (mx) quant_row_codes_mx(load, F, codes + (size_t)g * (F / 2), scales + (size_t)g * (F / 32));
    else quant_row_codes(load, F, codes + (size_t)g * (F / 2), scales + (size_t)g * (F / 16), st + g);
}

// y[t] = sum over p < k of gates[t][p] * part[t][p] (+ part[t][k], the shared expert); with
// expert parallelism only the selections this rank owns
__global__ void combine_kernel(const float *__restrict__ part, const float *__restrict__ gates,
                               const int32_t *__restrict__ idx, int ep_rank, int ep_size,
                               float *__restrict__ y, int T, int k, int d, int has_shared) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= (int64_t)T * d) return;
    const int t = (int)(i / d), c = (int)(i - (int64_t)t * d);
    const float *pr = part + (size_t)t * (k + 1) * d + c;
    float acc = 0.f;
    for (int p = 0; p < k; ++p)
        if (ep_size == 1 || idx[t * k + p] % ep_size == ep_rank) acc = fmaf(gates[t * k + p], pr[(size_t)p * d], acc);
    if (has_shared) acc += pr[(size_t)k * d];
    y[i] = acc;
}

__global__ void swiglu_split_kernel(const float *__restrict__ sg, int T, int F, uint16_t *__restrict__ hs) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= (int64_t)T * F) return;
    const int t = (int)(i / F), j = (int)(i - (int64_t)t * F);
    const float gt = sg[(size_t)t * 2 * F + 2 * j], up = sg[(size_t)t * 2 * F + 2 * j + 1];
    const float h = gt / (1.0f + expf(-gt)) * up;
    const __nv_bfloat16 hi = __float2bfloat16_rn(h);
    const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
    hs[(size_t)t * 2 * F + j] = __bfloat16_as_ushort(hi);
    hs[(size_t)t * 2 * F + F + j] = __bfloat16_as_ushort(lo);
}

}  // namespace

cudaError_t launch_swiglu_split(const float *sg, int T, int F, uint16_t *hs, cudaStream_t s) {
    const int64_t n = (int64_t)T * F;
    swiglu_split_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(sg, T, F, hs);
    return cudaGetLastError();
}

cudaError_t launch_quant_x_grouped(const __nv_bfloat16 *x, int T, int k, int d, int has_shared,
                                   const RowRef *rowrefs, const int32_t *n_routed, uint8_t *codes,
                                   uint8_t *scales, float *st, int mx, cudaStream_t s) {
    const int rows = T * k + (has_shared ? T : 0);
    const int warps_per_cta = 8;
    quant_x_grouped_kernel<<<(rows + warps_per_cta - 1) / warps_per_cta, warps_per_cta * 32, 0, s>>>(
        x, T, k, d, has_shared, rowrefs, n_routed, codes, scales, st, mx);
    return cudaGetLastError();
}

cudaError_t launch_quant_h_grouped(const float *h32, int T, int k, int has_shared, const int32_t *n_routed,
                                   int F, uint8_t *codes, uint8_t *scales, float *st, int mx, cudaStream_t s) {
    const int rows = T * k + (has_shared ? T : 0);
    const int warps_per_cta = 8;
    quant_h_grouped_kernel<<<(rows + warps_per_cta - 1) / warps_per_cta, warps_per_cta * 32, 0, s>>>(
        h32, T, k, has_shared, n_routed, F, codes, scales, st, mx);
    return cudaGetLastError();
}

cudaError_t launch_combine(const float *part, const float *gates, const int32_t *idx, int ep_rank, int ep_size,
                           float *y, int T, int k, int d, int has_shared, cudaStream_t s) {
    const int64_t n = (int64_t)T * d;
    combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(part, gates, idx, ep_rank, ep_size, y, T, k, d,
                                                               has_shared);
    return cudaGetLastError();
}

}  // namespace moe
