// NVFP4 activation quantizer (the W4A4 prefill path) and the prefill combine.
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
// The expert GEMV consumes each quantized row as its exact dequantized value
// e2m1 * e4m3 * s_t, split into an fp16 (hi, lo) pair, so the products with
// the NVFP4 weights are those of the W4A4 definition up to fp32 rounding.
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
// E2M1 RNE codes of (v0, v1) and their values.
__device__ __forceinline__ float2 e2m1_round_pair(float v0, float v1) {
    uint32_t r;
    asm("{\n\t.reg .b8 c;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c, %2, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, c;\n\t}"
        : "=r"(r)
        : "f"(v0), "f"(v1));
    return __half22float2(*reinterpret_cast<__half2 *>(&r));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ void store_hilo(__half *hi_row, __half *lo_row, int i, float v) {
    const __half hi = __float2half_rn(v);
    hi_row[i] = hi;
    lo_row[i] = __float2half_rn(v - __half2float(hi));
}

// One warp quantizes one row of n values (n a multiple of 16) and writes the
// dequantized row as an fp16 (hi, lo) pair.
template <typename LoadFn>
__device__ void quant_row(LoadFn load, int n, __half *hi_row, __half *lo_row) {
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
        const float sval = e4m3_value(e4m3_code(bmax / six_st));
        const float denom = sval * s_t;
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
            float2 q = make_float2(0.f, 0.f);
            if (sval != 0.f) q = e2m1_round_pair(v[j] / denom, v[j + 1] / denom);
            store_hilo(hi_row, lo_row, 16 * b + j, q.x * sval * s_t);
            store_hilo(hi_row, lo_row, 16 * b + j + 1, q.y * sval * s_t);
        }
    }
}

// x rows (bf16 [T][d]) -> xh [T][2][d]; one warp per row.
__global__ void quant_x_kernel(const __nv_bfloat16 *__restrict__ x, int T, int d, __half *xh) {
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    const __nv_bfloat16 *row = x + (size_t)t * d;
    quant_row([&](int i) { return __bfloat162float(row[i]); }, d, xh + (size_t)t * 2 * d,
              xh + (size_t)t * 2 * d + d);
}

// h rows (fp32 [T][k+1][F]) -> hh [T][k+1][2][F] for the selections that exist
// (p < k, and p = k when there is a shared expert); one warp per row.
__global__ void quant_h_kernel(const float *__restrict__ h32, int T, int k, int F, int has_shared,
                               __half *hh) {
    const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int per_t = k + (has_shared ? 1 : 0);
    if (w >= T * per_t) return;
    const int t = w / per_t, p = w - t * per_t;
    const size_t sel = (size_t)t * (k + 1) + p;
    const float *row = h32 + sel * F;
    quant_row([&](int i) { return row[i]; }, F, hh + sel * 2 * F, hh + sel * 2 * F + F);
}

// y[t] = sum over p < k of gates[t][p] * part[t][p] (+ part[t][k], the shared expert)
__global__ void combine_kernel(const float *__restrict__ part, const float *__restrict__ gates,
                               float *__restrict__ y, int T, int k, int d, int has_shared) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= (int64_t)T * d) return;
    const int t = (int)(i / d), c = (int)(i - (int64_t)t * d);
    const float *pr = part + (size_t)t * (k + 1) * d + c;
    float acc = 0.f;
    for (int p = 0; p < k; ++p) acc = fmaf(gates[t * k + p], pr[(size_t)p * d], acc);
    if (has_shared) acc += pr[(size_t)k * d];
    y[i] = acc;
}

}  // namespace

cudaError_t launch_quant_x(const __nv_bfloat16 *x, int T, int d, __half *xh, cudaStream_t s) {
    const int warps_per_cta = 8;
    quant_x_kernel<<<(T + warps_per_cta - 1) / warps_per_cta, warps_per_cta * 32, 0, s>>>(x, T, d, xh);
    return cudaGetLastError();
}

cudaError_t launch_quant_h(const float *h32, int T, int k, int F, int has_shared, __half *hh,
                           cudaStream_t s) {
    const int rows = T * (k + (has_shared ? 1 : 0));
    const int warps_per_cta = 8;
    quant_h_kernel<<<(rows + warps_per_cta - 1) / warps_per_cta, warps_per_cta * 32, 0, s>>>(
        h32, T, k, F, has_shared, hh);
    return cudaGetLastError();
}

cudaError_t launch_combine(const float *part, const float *gates, float *y, int T, int k, int d,
                           int has_shared, cudaStream_t s) {
    const int64_t n = (int64_t)T * d;
    combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(part, gates, y, T, k, d, has_shared);
    return cudaGetLastError();
}

}  // namespace moe
