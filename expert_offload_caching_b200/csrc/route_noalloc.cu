// moe_route_noalloc: router logits, softmax and top-k for up to 32 rows with no
// caller-provided workspace.
//
// Some callers cannot allocate device memory when they run: a host framework
// that owns the whole device memory pool and hands out only input and output
// buffers, or a process with a fixed memory budget planned before start-up.
// They cannot give moe_layer_init its workspace.  This entry point keeps its
// scratch -- the [T][E] logits and a CTA counter -- in one file-scope array
// built into the library instead, so a call needs nothing but its inputs and
// outputs and never calls cudaMalloc, cudaFree or any allocating routine.
//
// The array is per GPU, 128 KB + 256 B, and stays allocated on every GPU that
// loads the library until the process exits.  Every call shares it, and it
// keeps the last call's contents: each call clears the counter before it
// launches, and calls whose kernels overlap on the GPU (different streams, or
// several threads) race on it -- serialise them.  The first call on a device
// looks up the array's device address (cudaGetSymbolAddress, with that device
// current); make that first call before any stream capture.
//
// What it computes matches the routing part of moe_layer_forward: z = W_r x
// (bf16 inputs, fp32 accumulation), p = softmax(z), the k largest logits with
// ties to the lower id and NaN logits counted as -inf, gates renormalised over
// the k (or the plain softmax probabilities), ids in ascending order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/moe_offload.h"

namespace {

constexpr int kNaMaxRows = 32;
constexpr int kNaMaxE = 1024;
constexpr int kNaMaxK = 32;
constexpr int kNaThreads = 256;
constexpr size_t kNaLogitBytes = sizeof(float) * kNaMaxRows * kNaMaxE;
constexpr size_t kNaScratchBytes = kNaLogitBytes + 256;  // logits, then the CTA counter

// The scratch array.  In host code this name is only a stand-in for the
// symbol: never pass it to a kernel; use the address from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_route_scratch[kNaScratchBytes];

constexpr int kNaMaxDevices = 64;
std::mutex g_na_mutex;
void *g_na_ptr[kNaMaxDevices] = {};

__device__ __forceinline__ float na_warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
// Order-preserving 32-bit key of a float (-0 and +0 equal; NaN is mapped to
// -inf before) and back.
__device__ __forceinline__ uint32_t na_key(float v) {
    const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float na_key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
__device__ __forceinline__ float na_warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__global__ void __launch_bounds__(kNaThreads) route_noalloc_kernel(
    const __nv_bfloat16 *__restrict__ Wr, const __nv_bfloat16 *__restrict__ x, int T, int E, int d,
    int k, int renorm, int32_t *idx, float *gates, unsigned char *scratch) {
    float *z = reinterpret_cast<float *>(scratch);
    unsigned int *ticket = reinterpret_cast<unsigned int *>(scratch + kNaLogitBytes);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int nvec = d >> 3;

    // logits: one warp per router row, every row of x
    for (int e = blockIdx.x * nw + warp; e < E; e += gridDim.x * nw) {
        const uint4 *wrow = reinterpret_cast<const uint4 *>(Wr + (size_t)e * d);
        for (int t = 0; t < T; ++t) {
            const uint4 *xr = reinterpret_cast<const uint4 *>(x + (size_t)t * d);
            float acc = 0.f;
            for (int v = lane; v < nvec; v += 32) {
                const uint4 wv = __ldg(wrow + v), xv = __ldg(xr + v);
                const __nv_bfloat162 *wp = reinterpret_cast<const __nv_bfloat162 *>(&wv);
                const __nv_bfloat162 *xp = reinterpret_cast<const __nv_bfloat162 *>(&xv);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 a = __bfloat1622float2(wp[i]), b = __bfloat1622float2(xp[i]);
                    acc = fmaf(a.x, b.x, acc);
                    acc = fmaf(a.y, b.y, acc);
                }
            }
            acc = na_warp_sum(acc);
            if (lane == 0) z[t * E + e] = acc;
        }
    }

    // the last CTA to finish selects (threadfence + counter; nobody waits)
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // a NaN logit counts as -inf (selection and softmax), as in moe_layer_forward.
    // A row lives in registers (entry lane + 32 j in v[j]); a picked entry is
    // masked out by its bit, so each pick is the largest remaining logit in
    // (value desc, id asc) order and k distinct ids in [0, E) come out.
    constexpr int kNv = kNaMaxE / 32;
    for (int t = warp; t < T; t += nw) {
        const float *zr = z + (size_t)t * E;
        float v[kNv];
        uint32_t avail = 0u;
        float m = -INFINITY;
#pragma unroll
        for (int j = 0; j < kNv; ++j) {
            const int e = lane + 32 * j;
            const float zv = e < E ? __ldcg(zr + e) : -INFINITY;
            v[j] = zv != zv ? -INFINITY : zv;
            if (e < E) avail |= 1u << j;
            m = fmaxf(m, v[j]);
        }
        m = na_warp_max(m);
        float sall = 0.f;
#pragma unroll
        for (int j = 0; j < kNv; ++j)
            if ((avail >> j) & 1u) sall += expf(v[j] - m);
        sall = na_warp_sum(sall);
        int my_idx = 0x7fffffff;
        float my_val = -INFINITY;
        for (int s = 0; s < k; ++s) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < kNv; ++j) {  // ascending ids within the lane: keep the first of equal values
                const int e = lane + 32 * j;
                if (((avail >> j) & 1u) && (v[j] > bv || bi == 0x7fffffff)) { bv = v[j]; bi = e; }
            }
            // the warp's largest value (order-preserving integer key, warp
            // reductions), then the lowest id holding it
            const uint32_t key = na_key(bv);
            const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
            bi = (int)__reduce_min_sync(0xffffffffu, key == kmax ? (uint32_t)bi : 0xffffffffu);
            bv = na_key_value(kmax);
            if (bi != 0x7fffffff && (bi & 31) == lane) avail &= ~(1u << (bi >> 5));
            if (lane == s) { my_idx = bi; my_val = bv; }
        }
        const float top = __shfl_sync(0xffffffffu, my_val, 0);
        float g;
        if (renorm) {
            const float ex = lane < k ? expf(my_val - top) : 0.f;
            g = ex / na_warp_sum(ex);
        } else {
            g = expf(my_val - m) / sall;
        }
        int rank = 0;
        for (int i = 0; i < k; ++i) rank += (__shfl_sync(0xffffffffu, my_idx, i) < my_idx);
        if (lane < k) {
            idx[t * k + rank] = my_idx;
            gates[t * k + rank] = g;
        }
    }
    if (threadIdx.x == 0) *ticket = 0u;
}

// Device address of the scratch array on the current device, looked up once per device.
cudaError_t scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kNaMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_na_mutex);
    if (g_na_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess) return e;
        g_na_ptr[dev] = p;
    }
    *out = g_na_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" MOE_API moe_status moe_route_noalloc(const void *router_w, const void *x, int32_t T,
                                                int32_t E, int32_t d, int32_t k,
                                                int32_t renormalize, int32_t *idx, float *gates,
                                                void *stream) {
    if (!router_w || !x || !idx || !gates || T < 1 || E < 1 || k < 1 || k > E || d < 1)
        return MOE_ERR_ARG;
    // sizes beyond the built-in scratch (and the kernel's shapes) are refused
    if (T > kNaMaxRows || E > kNaMaxE || k > kNaMaxK || d % 64 != 0) return MOE_ERR_UNSUPPORTED;
    // rows are read as 16-byte vectors: both operands must start on a 16-byte boundary
    if (((uintptr_t)router_w | (uintptr_t)x) & 15u) return MOE_ERR_ARG;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the counter must start at zero; the logits are fully rewritten by every call
    if (cudaMemsetAsync(static_cast<unsigned char *>(scratch) + kNaLogitBytes, 0, sizeof(unsigned int), s) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    const int grid = (E + kNaThreads / 32 - 1) / (kNaThreads / 32);
    route_noalloc_kernel<<<grid, kNaThreads, 0, s>>>(
        static_cast<const __nv_bfloat16 *>(router_w), static_cast<const __nv_bfloat16 *>(x), T, E, d, k,
        renormalize, idx, gates, static_cast<unsigned char *>(scratch));
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
