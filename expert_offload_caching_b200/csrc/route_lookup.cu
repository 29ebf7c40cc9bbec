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
//     selects the experts and builds the job list;
//   * the table update reads everything it needs in one parallel round (the
//     batch's map entries, the header, every slot's stamp); the victims are
//     the smallest stamps among non-hit slots, found by block-wide argmin
//     rounds, so no list is walked.  The result equals the sequential rule
//     (hits stamped first in ascending id, then each miss in ascending id
//     takes the lowest never-used slot or the least recently used one);
//   * the miss list goes to mapped host memory as 16-byte records, then the
//     flag; the phase times of the tail go with it (diagnostics).
#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kRouteThreads = 256;
constexpr int kStampRegs = 32;           // stamps cached in registers: slots < 256 * 32
constexpr int kMaxSlotBits = 1 << 16;    // hit bitmap covers up to 65536 slots

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

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

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// z[t][e] for this warp's router row e (w: the row, already in registers).
// x rows are staged in shared memory (xs) a chunk at a time, all loads in
// flight together.  NV = 16-byte vectors per lane per row (d/256 rounded up).
template <int NV>
__device__ void router_logits(const RouteArgs &a, const uint4 (&w)[NV], int e, bool has_row,
                              uint4 *xs, int rows_per_chunk) {
    const int lane = threadIdx.x & 31;
    const int nvec = a.d >> 3;
    for (int t0 = 0; t0 < a.T; t0 += rows_per_chunk) {
        const int nr = a.T - t0 < rows_per_chunk ? a.T - t0 : rows_per_chunk;
        const uint4 *xg = reinterpret_cast<const uint4 *>(a.x + (size_t)t0 * a.d);
        for (int i = threadIdx.x; i < nr * nvec; i += blockDim.x) xs[i] = __ldg(xg + i);
        __syncthreads();
        if (has_row) {
            for (int r0 = 0; r0 < nr; r0 += 4) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < NV; ++i) {
                    const int v = lane + 32 * i;
                    if (v < nvec) {
                        float wf[8];
                        bf16x8_to_f32(w[i], wf);
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            if (r0 + r < nr) {
                                float xf[8];
                                bf16x8_to_f32(xs[(r0 + r) * nvec + v], xf);
#pragma unroll
                                for (int j = 0; j < 8; ++j) acc[r] = fmaf(wf[j], xf[j], acc[r]);
                            }
                        }
                    }
                }
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float sum = warp_sum(acc[r]);
                    if (lane == 0 && r0 + r < nr) a.ws.z[(size_t)(t0 + r0 + r) * a.E + e] = sum;
                }
            }
        }
        __syncthreads();
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
__global__ void __launch_bounds__(kRouteThreads) route_lookup_kernel(RouteArgs a, int rows_per_chunk) {
    extern __shared__ __align__(16) uint4 xs[];  // x rows of one chunk (bf16)
    const unsigned long long t_entry = global_ns();  // early: launched before the previous layer ends
    unsigned long long t_logits = 0, t_elect = 0, t_topk = 0, t_jobs = 0, t_read = 0, t_table = 0;
    // static data first: this warp's router row and the next layer's rows (L2)
    const int e_row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const bool has_row = e_row < a.E;
    uint4 w[NV];
    {
        const int lane = threadIdx.x & 31, nvec = a.d >> 3;
        const uint4 *wrow = reinterpret_cast<const uint4 *>(a.Wr + (size_t)(has_row ? e_row : 0) * a.d);
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int v = lane + 32 * i;
            w[i] = (has_row && v < nvec) ? ld_nc16(wrow + v) : make_uint4(0, 0, 0, 0);
        }
    }
    if (a.Wr_next != nullptr) {  // next layer's router rows -> L2
        const uint32_t total = (uint32_t)a.E * a.d * 2;
        const uint32_t per = ((total / gridDim.x) + 127u) & ~127u;
        const uint32_t off = per * blockIdx.x;
        if (off < total) prefetch_l2_range(reinterpret_cast<const uint8_t *>(a.Wr_next) + off,
                                           per < total - off ? per : total - off);
    }
    // the previous layer's kernels are complete past this point: x is final and
    // the shared buffers (logits, jobs, gates, activations) may be rewritten
    pdl_wait();
    pdl_launch_dependents();
    const unsigned long long t_start = global_ns();  // phases are timed from here
    router_logits<NV>(a, w, e_row, has_row, xs, rows_per_chunk);
    split_x(a);

    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        t_logits = global_ns();
        __threadfence();
        const unsigned int t = atomicAdd(a.ws.ticket, 1u);
        s_last = (t == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x == 0) t_elect = global_ns();

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
    if (threadIdx.x == 0) t_topk = global_ns();
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

    __syncthreads();
    if (threadIdx.x == 0) t_jobs = global_ns();

    // ---- cache lookup: one batch, ascending id.  All table reads in one round:
    // the batch's map entries, the header, and every slot's stamp.
    const int64_t keybase = (int64_t)a.layer * a.E;
    const int C = (int)a.tab.C;
    __shared__ unsigned long long s_clock, s_lastv;
    __shared__ int s_nf, s_nhit, s_nmiss, s_pick;
    __shared__ unsigned long long s_redv[kRouteThreads / 32];
    __shared__ int s_reds[kRouteThreads / 32];
    __shared__ uint32_t s_hitmap[kMaxSlotBits / 32];
    __shared__ int32_t s_rank[kMaxK * kDecodeMaxRows];
    __shared__ int32_t s_victim[kMaxK * kDecodeMaxRows];
    __shared__ int32_t s_old[kMaxK * kDecodeMaxRows];
    for (int i = threadIdx.x; i < kMaxSlotBits / 32; i += blockDim.x) s_hitmap[i] = 0u;
    for (int j = threadIdx.x; j < njobs; j += blockDim.x) s_slot[j] = a.tab.map[keybase + s_exp[j]];
    if (threadIdx.x == 0) { s_clock = a.tab.hdr->clock; s_nf = a.tab.hdr->next_free; }
    unsigned long long sv[kStampRegs];  // this thread's slots tid + 256*i
#pragma unroll
    for (int i = 0; i < kStampRegs; ++i) {
        const int sl = threadIdx.x + kRouteThreads * i;
        sv[i] = sl < C ? a.tab.stamp[sl] : ~0ull;
    }
    __syncthreads();
    if (threadIdx.x == 0) t_read = global_ns();
    for (int j = threadIdx.x; j < njobs; j += blockDim.x)
        if (s_slot[j] >= 0) atomicOr(&s_hitmap[s_slot[j] >> 5], 1u << (s_slot[j] & 31));
    if (warp == 0) {  // ranks: hits and misses, each in ascending id
        int hc = 0, mc = 0;
        for (int j0 = 0; j0 < njobs; j0 += 32) {
            const int j = j0 + lane;
            const bool valid = j < njobs, hit = valid && s_slot[j] >= 0;
            const unsigned hm = __ballot_sync(0xffffffffu, hit);
            const unsigned mm = __ballot_sync(0xffffffffu, valid && !hit);
            const unsigned lt = (1u << lane) - 1u;
            if (valid) s_rank[j] = hit ? hc + __popc(hm & lt) : mc + __popc(mm & lt);
            hc += __popc(hm);
            mc += __popc(mm);
        }
        if (lane == 0) { s_nhit = hc; s_nmiss = mc; }
    }
    __syncthreads();
    const int nhit = s_nhit, nmiss = s_nmiss, nf = s_nf;
    const int nfree = C - nf;
    const int nevict = nmiss > nfree ? nmiss - nfree : 0;
    // victims: the nevict non-hit slots with the smallest stamps (stamps are
    // unique, so round r takes the minimum above round r-1's)
    unsigned long long last = 0ull;
    for (int r = 0; r < nevict; ++r) {
        unsigned long long bv = ~0ull;
        int bs = -1;
#pragma unroll
        for (int i = 0; i < kStampRegs; ++i) {
            const int sl = threadIdx.x + kRouteThreads * i;
            if (sl < C && sv[i] > last && sv[i] < bv && !(s_hitmap[sl >> 5] & (1u << (sl & 31)))) {
                bv = sv[i];
                bs = sl;
            }
        }
        for (int sl = threadIdx.x + kRouteThreads * kStampRegs; sl < C; sl += kRouteThreads) {
            const unsigned long long v = a.tab.stamp[sl];  // caches beyond the register tile
            if (v > last && v < bv && !(s_hitmap[sl >> 5] & (1u << (sl & 31)))) { bv = v; bs = sl; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int os = __shfl_xor_sync(0xffffffffu, bs, o);
            if (ov < bv) { bv = ov; bs = os; }
        }
        if (lane == 0) { s_redv[warp] = bv; s_reds[warp] = bs; }
        __syncthreads();
        if (threadIdx.x == 0) {
            unsigned long long mv = s_redv[0];
            int ms = s_reds[0];
            for (int w = 1; w < nw; ++w)
                if (s_redv[w] < mv) { mv = s_redv[w]; ms = s_reds[w]; }
            s_victim[r] = ms;
            s_lastv = mv;
        }
        __syncthreads();
        last = s_lastv;
    }
    for (int r = threadIdx.x; r < nevict; r += blockDim.x) s_old[r] = a.tab.owner[s_victim[r]];
    __syncthreads();
    // slots, stamps and table writes (independent per job)
    const unsigned long long clock = s_clock;
    for (int j = threadIdx.x; j < njobs; j += blockDim.x) {
        const int s0 = s_slot[j];
        if (s0 >= 0) {  // hit: newest stamps in ascending id
            a.tab.stamp[s0] = clock + 1 + s_rank[j];
            s_evict[j] = -1;
        } else {        // miss: a never-used slot, else the next least recently used
            const int m = s_rank[j];
            int sl, ev = -1;
            if (m < nfree) sl = nf + m;
            else { sl = s_victim[m - nfree]; ev = s_old[m - nfree]; }
            const int key = (int)(keybase + s_exp[j]);
            if (ev >= 0) a.tab.map[ev] = -1;
            a.tab.map[key] = sl;
            a.tab.owner[sl] = key;
            a.tab.stamp[sl] = clock + 1 + nhit + m;
            s_slot[j] = -2 - sl;
            s_evict[j] = ev;
        }
    }
    if (threadIdx.x == 0) {
        a.tab.hdr->clock = clock + njobs;
        a.tab.hdr->next_free = nf + (nmiss < nfree ? nmiss : nfree);
        *a.ws.n_misses = nmiss;
    }
    __syncthreads();
    if (threadIdx.x == 0) t_table = global_ns();

    // ---- publish: one 16-byte record per entry, the counts, phase times, then the flag
    if (warp == 0) {
        for (int j = lane; j < njobs; j += 32) {
            const int sj = s_slot[j];
            HostEvent he;
            he.expert = s_exp[j];
            he.slot = sj >= 0 ? sj : -2 - sj;
            he.flags = sj >= 0 ? 1 : 0;
            he.evicted = s_evict[j];
            *reinterpret_cast<int4 *>(&a.page->ev[j]) = *reinterpret_cast<int4 *>(&he);
        }
        if (lane == 0) {
            a.page->n_events = njobs;
            a.page->n_jobs = njobs;
            a.page->n_misses = nmiss;
            a.page->phase_ns[0] = (uint32_t)(t_logits - t_start);
            a.page->phase_ns[1] = (uint32_t)(t_elect - t_logits);
            a.page->phase_ns[2] = (uint32_t)(t_topk - t_elect);
            a.page->phase_ns[3] = (uint32_t)(t_jobs - t_topk);
            a.page->phase_ns[4] = (uint32_t)(t_read - t_jobs);
            a.page->phase_ns[5] = (uint32_t)(t_table - t_read);
        }
        __threadfence_system();
        __syncwarp();
        if (lane == 0) {
            const unsigned long long t_pub = global_ns();
            a.page->phase_ns[6] = (uint32_t)(t_pub - t_table);
            a.page->phase_ns[7] = (uint32_t)(t_start - t_entry);  // launch-to-start: PDL wait
            __threadfence_system();
            if (a.publish) a.page->seq = a.seq;
        }
    }
    __syncthreads();
    for (int j = threadIdx.x; j < njobs; j += blockDim.x) {
        const int sj = s_slot[j];
        Job jb;
        jb.expert = s_exp[j];
        jb.slot = sj >= 0 ? sj : -2 - sj;
        jb.hit = sj >= 0;
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
        t.owner[j] = -1; t.stamp[j] = 0ull;
    }
    if (i == 0) {
        t.hdr->clock = 0ull; t.hdr->next_free = 0;
    }
}

template <int NV>
cudaError_t launch_nv(const RouteArgs &a, int grid, cudaStream_t s) {
    static bool configured = false;  // allow up to 64 KB of dynamic smem for the x chunk
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(route_lookup_kernel<NV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    int rows = (48 * 1024) / (a.d * 2);
    if (rows < 1) rows = 1;
    if (rows > a.T) rows = a.T;
    const size_t smem = (size_t)rows * a.d * 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kRouteThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, route_lookup_kernel<NV>, a, rows);
}

}  // namespace

cudaError_t launch_route_lookup(const RouteArgs &a, cudaStream_t s) {
    const int warps = kRouteThreads / 32;
    const int grid = (a.E + warps - 1) / warps;  // one router row per warp
    const int nv = ((a.d >> 3) + 31) >> 5;      // 16-byte vectors per lane per row
    if (nv <= 1) return launch_nv<1>(a, grid, s);
    if (nv <= 2) return launch_nv<2>(a, grid, s);
    if (nv <= 4) return launch_nv<4>(a, grid, s);
    if (nv <= 8) return launch_nv<8>(a, grid, s);
    if (nv <= 12) return launch_nv<12>(a, grid, s);
    if (nv <= 16) return launch_nv<16>(a, grid, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_table_reset(Table t, int64_t nkeys, cudaStream_t s) {
    table_reset_kernel<<<256, 256, 0, s>>>(t, nkeys);
    return cudaGetLastError();
}

}  // namespace moe
