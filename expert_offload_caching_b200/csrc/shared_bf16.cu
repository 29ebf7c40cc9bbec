// BF16 shared expert for decode rows (T <= 32).
//
// The pages keep the shared experts in BF16 while the routed experts are
// 4-bit (florigen.ai "NVFP4で約135GBまで縮める").  Such a record is W13
// [2F x d] bf16 (row 2j = gate_j, 2j+1 = up_j), then W2 [d x F] bf16:
//   h_j = silu(W1_j . x) * (W3_j . x);   y_shared = W2 h.
// The shared expert is always used and always resident, so it runs in two
// launches of its own, before the routed experts' launches; it writes the same
// buffers the routed experts do (h as fp16 hi/lo pairs, the output at the
// selection p = k of each row), and the routed combine adds it.  It reads x as
// the route kernel's fp16 (hi, lo) split (device memory; x itself may be
// mapped host memory).
//
// Decode reads each weight once for at most 32 rows: HBM-bound.  One warp per
// output pair: the lanes stride the pair's two weight rows in 16-byte chunks
// (8 bf16; a warp reads 512 contiguous bytes per row and step), each lane keeps
// fp32 partial sums for up to 8 activation rows per pass, and a butterfly of
// shuffles sums them over the warp.
#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kSbWarps = 8;
constexpr int kSbMaxT = kDecodeMaxRows;
constexpr int kSbRows = 8;  // activation rows per pass

// 8 bf16 (one 16-byte chunk of a weight row) -> fp32 (a bf16 is the top half of an fp32)
__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
// 8 fp16 hi + 8 fp16 lo -> fp32 hi + lo
__device__ __forceinline__ void h2x8_sum_to_f32(const uint4 hi, const uint4 lo, float (&f)[8]) {
    const uint32_t a[4] = {hi.x, hi.y, hi.z, hi.w}, b[4] = {lo.x, lo.y, lo.z, lo.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __half22float2(*reinterpret_cast<const __half2 *>(&a[i]));
        const float2 y = __half22float2(*reinterpret_cast<const __half2 *>(&b[i]));
        f[2 * i] = x.x + y.x;
        f[2 * i + 1] = x.y + y.y;
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// MODE kGateUp: warp j computes gate_j and up_j for every row t (activation:
// xh row t) and writes h_tj; MODE kDown: warp i computes output dims 2i and
// 2i+1 (activation: hh at the row's selection).
template <int MODE>
__global__ void __launch_bounds__(kSbWarps * 32)
    shared_bf16_kernel(const uint8_t *rec, int d, int F, int T, const __half *xh, __half *hh,
                       float *part, int64_t sel0, int64_t sel_stride) {
    const int lane = threadIdx.x & 31;
    const int wid = (int)blockIdx.x * kSbWarps + (int)(threadIdx.x >> 5);
    const int npairs = MODE == kGateUp ? F : d / 2;
    if (wid >= npairs) return;
    const int K = MODE == kGateUp ? d : F;
    const int nch = K >> 3;  // 16-byte chunks of a weight row
    const __nv_bfloat16 *W = reinterpret_cast<const __nv_bfloat16 *>(rec) +
                             (MODE == kGateUp ? (size_t)0 : (size_t)2 * F * d);
    const uint4 *r0 = reinterpret_cast<const uint4 *>(W + (size_t)(2 * wid) * K);
    const uint4 *r1 = reinterpret_cast<const uint4 *>(W + (size_t)(2 * wid + 1) * K);

    // rows in groups of kSbRows (one pass over the weight pair per group; later
    // passes find the pair in L1/L2)
    for (int t0 = 0; t0 < T; t0 += kSbRows) {
        float acc0[kSbRows], acc1[kSbRows];
#pragma unroll
        for (int r = 0; r < kSbRows; ++r) acc0[r] = acc1[r] = 0.f;
#pragma unroll 2
        for (int c = lane; c < nch; c += 32) {
            float w0[8], w1[8];
            bf16x8_to_f32(__ldg(r0 + c), w0);
            bf16x8_to_f32(__ldg(r1 + c), w1);
#pragma unroll
            for (int r = 0; r < kSbRows; ++r) {
                const int t = t0 + r;
                if (t < T) {
                    // the row's activation: K fp16 hi, then K fp16 lo
                    const __half *h =
                        MODE == kGateUp ? xh + (size_t)t * 2 * d : hh + (sel0 + t * sel_stride) * 2 * F;
                    float a[8];
                    h2x8_sum_to_f32(reinterpret_cast<const uint4 *>(h)[c], reinterpret_cast<const uint4 *>(h + K)[c],
                                    a);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        acc0[r] = fmaf(w0[i], a[i], acc0[r]);
                        acc1[r] = fmaf(w1[i], a[i], acc1[r]);
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kSbRows; ++r) {
            const int t = t0 + r;
            if (t < T) {
                const float v0 = warp_sum(acc0[r]), v1 = warp_sum(acc1[r]);
                if (lane == r) {
                    const int64_t sel = sel0 + t * sel_stride;
                    if (MODE == kGateUp) {
                        const float h = v0 / (1.0f + expf(-v0)) * v1;
                        const __half hi = __float2half_rn(h);
                        const __half lo = __float2half_rn(h - __half2float(hi));
                        hh[sel * 2 * F + wid] = hi;
                        hh[sel * 2 * F + F + wid] = lo;
                    } else {
                        part[sel * d + 2 * wid] = v0;
                        part[sel * d + 2 * wid + 1] = v1;
                    }
                }
            }
        }
    }
}

}  // namespace

cudaError_t launch_shared_bf16(int mode, const uint8_t *rec, int d, int F, int T, const __half *xh,
                               __half *hh, float *part, int64_t sel0, int64_t sel_stride, cudaStream_t s) {
    if (T < 1 || T > kSbMaxT || d % 64 != 0 || F % 64 != 0 || !rec) return cudaErrorInvalidValue;
    const int npairs = mode == kGateUp ? F : d / 2;
    const unsigned grid = (unsigned)((npairs + kSbWarps - 1) / kSbWarps);
    if (mode == kGateUp)
        shared_bf16_kernel<kGateUp><<<grid, kSbWarps * 32, 0, s>>>(rec, d, F, T, xh, hh, part, sel0, sel_stride);
    else
        shared_bf16_kernel<kDown><<<grid, kSbWarps * 32, 0, s>>>(rec, d, F, T, xh, hh, part, sel0, sel_stride);
    return cudaGetLastError();
}

}  // namespace moe
