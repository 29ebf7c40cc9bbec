// Router logits, softmax + top-k, and the global LRU cache lookup of one layer
// (decode path, T <= 32 rows), fused into one launch.
//
// Router (FreeToken pages: routers kept in BF16, florigen.ai "NVFP4で約135GBまで縮める";
// k of E routed experts per token: florigen.ai 10 of 512, gaming-st.com 6 of 256,
// pirouter.ai 4 per layer): z = W_r x with bf16 inputs and fp32 accumulation;
// p = softmax(z); the k largest logits (ties to the lower id); gates
// renormalised over the k.  Cache (ai-hardware-zukan "GPUに載らない分をどう間に合わせるか":
// unit = (layer, expert), least-recently-used replacement, contents follow the
// router; gaming-st.com "技術的背景": one global LRU expert cache): the distinct
// selected experts form one lookup batch in ascending id; hits are stamped
// first, then each miss takes the lowest never-used slot or evicts the least
// recently used one.
//
// The step sits on the decode critical path (the next layer's copies cannot
// start before it), so it is built for latency:
//   * one warp per router row issues every load of its row before the first
//     FMA (one HBM round trip for the whole router);
//   * the next layer's router rows are prefetched into L2 (static weights,
//     prefetch.global.L2);
//   * the last CTA to finish (threadfence + atomic ticket; nobody waits)
//     selects the experts, builds the job list and runs the table update with
//     a single warp (deterministic slot assignment), then publishes the miss
//     list to mapped host memory (16-byte records) and raises the flag.
#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kRouteThreads = 256;

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float *f) {
    const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(p[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ uint4 ld_nc16(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Prefetch [p, p + bytes) into L2, one 128-byte line per thread of the CTA.
__device__ __forceinline__ void prefetch_l2_range(const uint8_t *p, uint32_t bytes) {
    for (uint32_t o = threadIdx.x * 128u; o < bytes; o += blockDim.x * 128u)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(p + o));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// z[t][e] for this CTA's experts.  NV = 16-byte vectors per lane per row (d/256 rounded up).
template <int NV>
__device__ void router_logits(const RouteArgs &a) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int nvec = a.d >> 3;
    for (int e = blockIdx.x * nw + warp; e < a.E; e += gridDim.x * nw) {
        const uint4 *wrow = reinterpret_cast<const uint4 *>(a.Wr + (size_t)e * a.d);
        uint4 w[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int v = lane + 32 * i;
            w[i] = v < nvec ? ld_nc16(wrow + v) : make_uint4(0, 0, 0, 0);
        }
        for (int t0 = 0; t0 < a.T; t0 += 4) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int v = lane + 32 * i;
                if (v < nvec) {
                    float wf[8];
                    bf16x8_to_f32(w[i], wf);
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        if (t0 + r < a.T) {
                            float xf[8];
                            bf16x8_to_f32(
                                __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)(t0 + r) * a.d) + v),
                                xf);
#pragma unroll
                            for (int j = 0; j < 8; ++j) acc[r] = fmaf(wf[j], xf[j], acc[r]);
                        }
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float s = warp_sum(acc[r]);
                if (lane == 0 && t0 + r < a.T) a.ws.z[(size_t)(t0 + r) * a.E + e] = s;
            }
        }
    }
}

// x -> (hi, lo) fp16 pair with hi + lo == x for |x| < 65504 (bf16 needs no lo
// in the normal fp16 range; lo keeps what fp16 subnormals would drop).
__device__ void split_x(const RouteArgs &a) {
    const int n = a.T * a.d;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const int t = i / a.d, c = i - t * a.d;
        const float v = __bfloat162float(a.x[i]);
        const __half hi = __float2half_rn(v);
        const __half lo = __float2half_rn(v - __half2float(hi));
        a.ws.xh[(size_t)t * 2 * a.d + c] = hi;
        a.ws.xh[(size_t)t * 2 * a.d + a.d + c] = lo;
    }
}

// Softmax + top-k of row t by one warp; writes idx/gates of the row in ascending id.
__device__ void topk_row(const RouteArgs &a, int t) {
    const int lane = threadIdx.x & 31;
    const float *z = a.ws.z + (size_t)t * a.E;
    const int nv = (a.E + 31) >> 5;
    float v[kMaxE / 32];
#pragma unroll
    for (int j = 0; j < kMaxE / 32; ++j) {
        const int e = lane + 32 * j;
        v[j] = (j < nv && e < a.E) ? z[e] : -INFINITY;
    }
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < kMaxE / 32; ++j) m = fmaxf(m, v[j]);
    m = warp_max(m);
    float sall = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxE / 32; ++j)
        if (lane + 32 * j < a.E) sall += expf(v[j] - m);
    sall = warp_sum(sall);

    int my_idx = 0x7fffffff;
    float my_val = -INFINITY;
    for (int s = 0; s < a.k; ++s) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < kMaxE / 32; ++j) {
            const int e = lane + 32 * j;
            if (e < a.E && v[j] > bv) { bv = v[j]; bi = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if (lane == s) { my_idx = bi; my_val = bv; }
        const int owner = bi & 31, slotj = bi >> 5;
#pragma unroll
        for (int j = 0; j < kMaxE / 32; ++j)
            if (lane == owner && j == slotj) v[j] = -INFINITY;
    }
    const float top = __shfl_sync(0xffffffffu, my_val, 0);
    float g;
    if (a.renorm) {
        const float ex = lane < a.k ? expf(my_val - top) : 0.f;
        g = ex / warp_sum(ex);
    } else {
        g = expf(my_val - m) / sall;
    }
    int rank = 0;
    for (int i = 0; i < a.k; ++i) rank += (__shfl_sync(0xffffffffu, my_idx, i) < my_idx);
    if (lane < a.k) {
        a.ws.idx[t * a.k + rank] = my_idx;
        a.ws.gates[t * a.k + rank] = g;
    }
}

template <int NV>
__global__ void __launch_bounds__(kRouteThreads) route_lookup_kernel(RouteArgs a) {
    if (a.Wr_next != nullptr) {  // next layer's router rows -> L2
        const uint32_t total = (uint32_t)a.E * a.d * 2;
        const uint32_t per = ((total / gridDim.x) + 127u) & ~127u;
        const uint32_t off = per * blockIdx.x;
        if (off < total) prefetch_l2_range(reinterpret_cast<const uint8_t *>(a.Wr_next) + off,
                                           per < total - off ? per : total - off);
    }
    router_logits<NV>(a);
    split_x(a);

    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned int t = atomicAdd(a.ws.ticket, 1u);
        s_last = (t == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int t = warp; t < a.T; t += nw) topk_row(a, t);

    // ---- distinct experts of the batch, ascending: a bitmap over E
    __shared__ uint32_t s_bits[kMaxE / 32];
    __shared__ int s_base[kMaxE / 32];
    __shared__ int s_njobs;
    __shared__ int32_t s_exp[kMaxK * kDecodeMaxRows];
    __shared__ int32_t s_cnt[kMaxK * kDecodeMaxRows];
    __shared__ int32_t s_off[kMaxK * kDecodeMaxRows];
    __shared__ int32_t s_slot[kMaxK * kDecodeMaxRows];
    __shared__ int32_t s_evict[kMaxK * kDecodeMaxRows];
    __shared__ int32_t s_idx[kMaxK * kDecodeMaxRows];
    for (int i = threadIdx.x; i < kMaxE / 32; i += blockDim.x) s_bits[i] = 0u;
    __syncthreads();
    const int nsel = a.T * a.k;
    for (int i = threadIdx.x; i < nsel; i += blockDim.x) {
        const int e = a.ws.idx[i];
        s_idx[i] = e;
        atomicOr(&s_bits[e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    if (warp == 0) {
        const int c = __popc(s_bits[lane]);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        s_base[lane] = incl - c;
        if (lane == 31) s_njobs = incl;
    }
    __syncthreads();
    const int njobs = s_njobs;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        const uint32_t w = s_bits[e >> 5];
        if (w & (1u << (e & 31))) s_exp[s_base[e >> 5] + __popc(w & ((1u << (e & 31)) - 1u))] = e;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < njobs; j += blockDim.x) {
        int c = 0;
        for (int i = 0; i < nsel; ++i) c += (s_idx[i] == s_exp[j]);
        s_cnt[j] = c;
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scan of the counts, 32 at a time
        int carry = 0;
        for (int j0 = 0; j0 < njobs; j0 += 32) {
            const int j = j0 + lane;
            const int c = j < njobs ? s_cnt[j] : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (j < njobs) s_off[j] = carry + incl - c;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    __syncthreads();
    for (int j = threadIdx.x; j < njobs; j += blockDim.x) {
        int pos = s_off[j];
        for (int i = 0; i < nsel; ++i)
            if (s_idx[i] == s_exp[j]) {
                a.ws.rowrefs[pos].t = (int16_t)(i / a.k);
                a.ws.rowrefs[pos].p = (int16_t)(i % a.k);
                ++pos;
            }
    }

    // ---- LRU update by one warp: parallel map reads, then serial list edits
    const int64_t keybase = (int64_t)a.layer * a.E;
    if (warp == 0) {
        for (int j = lane; j < njobs; j += 32) s_slot[j] = a.tab.map[keybase + s_exp[j]];
        __syncwarp();
        if (lane == 0) {
            TableHdr *h = a.tab.hdr;
            unsigned long long clock = h->clock;
            int head = h->head, tail = h->tail, nf = h->next_free;
            const int C = (int)a.tab.C;
            int32_t *prv = a.tab.prev, *nxt = a.tab.next;
            int nmiss = 0;
            for (int j = 0; j < njobs; ++j) {  // hits, ascending id: newest stamps, to the tail
                const int s = s_slot[j];
                s_evict[j] = -1;
                if (s < 0) continue;
                a.tab.stamp[s] = ++clock;
                if (s != tail) {
                    const int p = prv[s], n = nxt[s];
                    if (p >= 0) nxt[p] = n; else head = n;
                    prv[n] = p;  // n >= 0 since s != tail
                    prv[s] = tail; nxt[s] = -1; nxt[tail] = s; tail = s;
                }
            }
            for (int j = 0; j < njobs; ++j) {  // misses, ascending id
                if (s_slot[j] >= 0) continue;
                ++nmiss;
                int s, ev = -1;
                if (nf < C) {
                    s = nf++;  // never-used slots go in index order (the lowest free slot)
                } else {
                    s = head;  // least recently used
                    const int n = nxt[s];
                    const int old = a.tab.owner[s];
                    head = n;
                    if (n >= 0) prv[n] = -1; else tail = -1;
                    a.tab.map[old] = -1;
                    ev = old;
                }
                const int key = (int)(keybase + s_exp[j]);
                a.tab.owner[s] = key;
                a.tab.map[key] = s;
                a.tab.stamp[s] = ++clock;
                prv[s] = tail; nxt[s] = -1;
                if (tail >= 0) nxt[tail] = s; else head = s;
                tail = s;
                s_slot[j] = -2 - s;  // marks a miss, keeps the slot
                s_evict[j] = ev;
            }
            h->clock = clock; h->head = head; h->tail = tail; h->next_free = nf;
            *a.ws.n_misses = nmiss;
            s_base[0] = nmiss;
        }
        __syncwarp();
        // publish: one 16-byte record per entry, then the counts, then the flag
        for (int j = lane; j < njobs; j += 32) {
            const int s = s_slot[j];
            HostEvent he;
            he.expert = s_exp[j];
            he.slot = s >= 0 ? s : -2 - s;
            he.flags = s >= 0 ? 1 : 0;
            he.evicted = s_evict[j];
            *reinterpret_cast<int4 *>(&a.page->ev[j]) = *reinterpret_cast<int4 *>(&he);
        }
        if (lane == 0) {
            a.page->n_events = njobs;
            a.page->n_jobs = njobs;
            a.page->n_misses = s_base[0];
        }
        __threadfence_system();
        __syncwarp();
        if (lane == 0 && a.publish) a.page->seq = a.seq;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < njobs; j += blockDim.x) {
        const int s = s_slot[j];
        Job jb;
        jb.expert = s_exp[j];
        jb.slot = s >= 0 ? s : -2 - s;
        jb.hit = s >= 0;
        jb.nrows = s_cnt[j];
        jb.row_off = s_off[j];
        jb.pad[0] = jb.pad[1] = jb.pad[2] = 0;
        a.ws.jobs[j] = jb;
    }
    if (threadIdx.x == 0) {
        *a.ws.n_jobs = njobs;
        *a.ws.ticket = 0u;
    }
}

__global__ void table_reset_kernel(Table t, int64_t nkeys) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t j = i; j < nkeys; j += stride) t.map[j] = -1;
    for (int64_t j = i; j < t.C; j += stride) {
        t.owner[j] = -1; t.stamp[j] = 0ull; t.prev[j] = -1; t.next[j] = -1;
    }
    if (i == 0) {
        t.hdr->clock = 0ull; t.hdr->next_free = 0; t.hdr->head = -1; t.hdr->tail = -1;
    }
}

}  // namespace

cudaError_t launch_route_lookup(const RouteArgs &a, cudaStream_t s) {
    const int warps = kRouteThreads / 32;
    int grid = (a.E + warps - 1) / warps;
    if (grid < 1) grid = 1;
    const int nv = ((a.d >> 3) + 31) >> 5;  // 16-byte vectors per lane per row
    if (nv <= 1) route_lookup_kernel<1><<<grid, kRouteThreads, 0, s>>>(a);
    else if (nv <= 2) route_lookup_kernel<2><<<grid, kRouteThreads, 0, s>>>(a);
    else if (nv <= 4) route_lookup_kernel<4><<<grid, kRouteThreads, 0, s>>>(a);
    else if (nv <= 8) route_lookup_kernel<8><<<grid, kRouteThreads, 0, s>>>(a);
    else if (nv <= 12) route_lookup_kernel<12><<<grid, kRouteThreads, 0, s>>>(a);
    else if (nv <= 16) route_lookup_kernel<16><<<grid, kRouteThreads, 0, s>>>(a);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

cudaError_t launch_table_reset(Table t, int64_t nkeys, cudaStream_t s) {
    table_reset_kernel<<<256, 256, 0, s>>>(t, nkeys);
    return cudaGetLastError();
}

}  // namespace moe
