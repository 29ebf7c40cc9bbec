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
// Work split: every CTA computes logits for a slice of experts (one warp per
// expert row) and converts x to an fp16 hi/lo pair for the expert GEMVs.  The
// last CTA to finish (threadfence + atomic ticket; nobody waits) selects the
// experts, builds the job list and runs the table update with a single warp,
// so the slot assignment is deterministic, then publishes the miss list to
// mapped host memory and raises the sequence flag.
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

// z[t][e] for this CTA's experts; 8 rows of x per pass.
__device__ void router_logits(const RouteArgs &a) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int nvec = a.d / 8;
    for (int e = blockIdx.x * nw + warp; e < a.E; e += gridDim.x * nw) {
        const uint4 *wrow = reinterpret_cast<const uint4 *>(a.Wr + (size_t)e * a.d);
        for (int t0 = 0; t0 < a.T; t0 += 8) {
            float acc[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) acc[r] = 0.f;
            for (int v = lane; v < nvec; v += 32) {
                float wf[8];
                bf16x8_to_f32(__ldg(wrow + v), wf);
#pragma unroll
                for (int r = 0; r < 8; ++r) {
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
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                float s = warp_sum(acc[r]);
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
        int t = i / a.d, c = i - t * a.d;
        float v = __bfloat162float(a.x[i]);
        __half hi = __float2half_rn(v);
        __half lo = __float2half_rn(v - __half2float(hi));
        a.ws.xh[(size_t)t * 2 * a.d + c] = hi;
        a.ws.xh[(size_t)t * 2 * a.d + a.d + c] = lo;
    }
}

// Softmax + top-k of row t by one warp; writes idx/gates of the row in ascending id.
__device__ void topk_row(const RouteArgs &a, int t) {
    const int lane = threadIdx.x & 31;
    const float *z = a.ws.z + (size_t)t * a.E;
    float v[kMaxE / 32];
#pragma unroll
    for (int j = 0; j < kMaxE / 32; ++j) {
        int e = lane + 32 * j;
        v[j] = e < a.E ? z[e] : -INFINITY;
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
            int e = lane + 32 * j;
            if (e < a.E && v[j] > bv) { bv = v[j]; bi = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if (lane == s) { my_idx = bi; my_val = bv; }
#pragma unroll
        for (int j = 0; j < kMaxE / 32; ++j)
            if (lane == (bi & 31) && j == (bi >> 5)) v[j] = -INFINITY;
    }
    const float top = __shfl_sync(0xffffffffu, my_val, 0);
    float g;
    if (a.renorm) {
        float ex = lane < a.k ? expf(my_val - top) : 0.f;
        float s = warp_sum(ex);
        g = ex / s;
    } else {
        g = expf(my_val - m) / sall;
    }
    int rank = 0;
    for (int i = 0; i < a.k; ++i) {
        int oi = __shfl_sync(0xffffffffu, my_idx, i);
        rank += (oi < my_idx);
    }
    if (lane < a.k) {
        a.ws.idx[t * a.k + rank] = my_idx;
        a.ws.gates[t * a.k + rank] = g;
    }
}

__global__ void __launch_bounds__(kRouteThreads) route_lookup_kernel(RouteArgs a) {
    router_logits(a);
    split_x(a);

    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        unsigned int t = atomicAdd(a.ws.ticket, 1u);
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
    __shared__ int64_t s_evict[kMaxK * kDecodeMaxRows];
    for (int i = threadIdx.x; i < kMaxE / 32; i += blockDim.x) s_bits[i] = 0u;
    __syncthreads();
    const int nsel = a.T * a.k;
    for (int i = threadIdx.x; i < nsel; i += blockDim.x) {
        int e = a.ws.idx[i];
        atomicOr(&s_bits[e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    if (warp == 0) {
        int c = __popc(s_bits[lane]);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        s_base[lane] = incl - c;
        if (lane == 31) s_njobs = incl;
    }
    __syncthreads();
    const int njobs = s_njobs;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        uint32_t w = s_bits[e >> 5];
        if (w & (1u << (e & 31))) s_exp[s_base[e >> 5] + __popc(w & ((1u << (e & 31)) - 1u))] = e;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < njobs; j += blockDim.x) {
        int c = 0;
        for (int i = 0; i < nsel; ++i) c += (a.ws.idx[i] == s_exp[j]);
        s_cnt[j] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int off = 0;
        for (int j = 0; j < njobs; ++j) { s_off[j] = off; off += s_cnt[j]; }
    }
    __syncthreads();
    for (int j = threadIdx.x; j < njobs; j += blockDim.x) {
        int pos = s_off[j];
        for (int i = 0; i < nsel; ++i)
            if (a.ws.idx[i] == s_exp[j]) {
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
            for (int j = 0; j < njobs; ++j) {  // hits, ascending id
                int s = s_slot[j];
                s_evict[j] = -1;
                if (s < 0) continue;
                a.tab.stamp[s] = ++clock;
                if (s != tail) {  // unlink, append at the tail
                    int p = prv[s], n = nxt[s];
                    if (p >= 0) nxt[p] = n; else head = n;
                    prv[n] = p;  // n >= 0 since s != tail
                    prv[s] = tail; nxt[s] = -1; nxt[tail] = s; tail = s;
                }
            }
            for (int j = 0; j < njobs; ++j) {  // misses, ascending id
                if (s_slot[j] >= 0) continue;
                ++nmiss;
                int s;
                int64_t ev = -1;
                if (nf < C) {
                    s = nf++;
                } else {
                    s = head;
                    int n = nxt[s];
                    head = n;
                    if (n >= 0) prv[n] = -1; else tail = -1;
                    int old = a.tab.owner[s];
                    a.tab.map[old] = -1;
                    ev = old;
                }
                int key = (int)(keybase + s_exp[j]);
                a.tab.owner[s] = key;
                a.tab.map[key] = s;
                a.tab.stamp[s] = ++clock;
                prv[s] = tail; nxt[s] = -1;
                if (tail >= 0) nxt[tail] = s; else head = s;
                tail = s;
                s_slot[j] = -2 - s;  // mark as miss, keep the slot
                s_evict[j] = ev;
            }
            h->clock = clock; h->head = head; h->tail = tail; h->next_free = nf;
            a.page->n_misses = nmiss;
        }
    }
    __syncthreads();
    for (int j = threadIdx.x; j < njobs; j += blockDim.x) {
        int s = s_slot[j];
        int hit = s >= 0;
        int slot = hit ? s : -2 - s;
        Job jb;
        jb.expert = s_exp[j]; jb.slot = slot; jb.hit = hit; jb.nrows = s_cnt[j]; jb.row_off = s_off[j];
        jb.pad[0] = jb.pad[1] = jb.pad[2] = 0;
        a.ws.jobs[j] = jb;
        HostEvent he;
        he.expert = s_exp[j]; he.slot = slot; he.hit = hit; he.prefetch = 0; he.evicted = s_evict[j];
        a.page->ev[j] = he;
    }
    if (threadIdx.x == 0) {
        *a.ws.n_jobs = njobs;
        a.page->n_events = njobs;
        a.page->n_jobs = njobs;
        *a.ws.ticket = 0u;
    }
    __threadfence_system();
    __syncthreads();
    if (threadIdx.x == 0 && a.publish) {
        __threadfence_system();
        a.page->seq = a.seq;
    }
}

__global__ void table_reset_kernel(Table t, int64_t nkeys) {
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
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
    route_lookup_kernel<<<grid, kRouteThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_table_reset(Table t, int64_t nkeys, cudaStream_t s) {
    table_reset_kernel<<<256, 256, 0, s>>>(t, nkeys);
    return cudaGetLastError();
}

}  // namespace moe
