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

// Order-preserving 32-bit key of a float (larger key <=> larger value, -0 and
// +0 equal, -inf the smallest of the values used here; NaN is mapped to -inf
// before) and back.
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
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

// A selected id outside [0, E) (the selection is total, so this is a broken
// invariant, not an input case): record it in the mapped page; the caller
// skips the access and the host turns the error word into MOE_ERR_CUDA.
constexpr int kCheckExpertRange = 30;
__device__ void route_fail(HostPage *page, int mode, int e, int E) {
    page->diag[1] = mode;
    page->diag[2] = (int)blockIdx.x;
    page->diag[3] = 0;
    page->diag[4] = (int)threadIdx.x;
    page->diag[5] = e;
    page->diag[6] = E;
    __threadfence_system();
    page->error = kCheckExpertRange;
    __threadfence_system();
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// z[t][e] for router row e, split over S consecutive warps of the CTA (warp
// seg holds the seg-th S-th of the row in registers, w); their partial sums
// meet in shared memory and are added in segment order.  x rows are staged in
// shared memory (xs) a chunk at a time, all loads in flight together.  NV =
// 16-byte vectors per lane of a segment (d/(256 S) rounded up).
template <int NV>
__device__ void router_logits(const RouteArgs &a, const uint4 (&w)[NV], int e, bool has_row,
                              uint4 *xs, int rows_per_chunk, int S, int seg) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nvec = a.d >> 3, segv = nvec / S, v0 = seg * segv;
    __shared__ float s_part[kRouteThreads / 32][4];
    for (int t0 = 0; t0 < a.T; t0 += rows_per_chunk) {
        const int nr = a.T - t0 < rows_per_chunk ? a.T - t0 : rows_per_chunk;
        const uint4 *xg = reinterpret_cast<const uint4 *>(a.x + (size_t)t0 * a.d);
        for (int i = threadIdx.x; i < nr * nvec; i += blockDim.x) xs[i] = __ldg(xg + i);
        __syncthreads();
        // the chunk's x as fp16 (hi, lo) pairs for the expert GEMVs (hi + lo == x
        // for |x| < 65504: bf16 needs no lo in the normal fp16 range, lo keeps what
        // fp16 subnormals would drop), each element by one thread of the grid
        // from the staged copy
        const __nv_bfloat16 *xsb = reinterpret_cast<const __nv_bfloat16 *>(xs);
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nr * a.d; i += gridDim.x * blockDim.x) {
            const int t = t0 + i / a.d, c = i - (i / a.d) * a.d;
            const float v = __bfloat162float(xsb[i]);
            const __half hi = __float2half_rn(v);
            const __half lo = __float2half_rn(v - __half2float(hi));
            a.ws.xh[(size_t)t * 2 * a.d + c] = hi;
            a.ws.xh[(size_t)t * 2 * a.d + a.d + c] = lo;
        }
        for (int r0 = 0; r0 < nr; r0 += 4) {  // (the same trip count in every warp of the CTA)
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            if (has_row) {
#pragma unroll
                for (int i = 0; i < NV; ++i) {
                    const int vl = lane + 32 * i;
                    if (vl < segv) {
                        const int v = v0 + vl;
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
            }
            float sum[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) sum[r] = warp_sum(acc[r]);
            if (S == 1) {
                if (has_row && lane == 0)
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        if (r0 + r < nr) a.ws.z[(size_t)(t0 + r0 + r) * a.E + e] = sum[r];
            } else {
                if (lane == 0)
#pragma unroll
                    for (int r = 0; r < 4; ++r) s_part[warp][r] = sum[r];
                __syncthreads();
                if (has_row && seg == 0 && lane < 4 && r0 + lane < nr) {
                    float z = 0.f;
                    for (int q = 0; q < S; ++q) z += s_part[warp + q][lane];
                    a.ws.z[(size_t)(t0 + r0 + lane) * a.E + e] = z;
                }
                __syncthreads();  // s_part is rewritten by the next row group
            }
        }
        __syncthreads();
    }
}

// Softmax + top-k of row t by one warp; writes idx/gates of the row in ascending
// id and returns the expert selected by this lane (lanes < k), else -1.
// NVE: 32-wide chunks of the row held in registers (E <= 32 * NVE).
// The order is total: a NaN logit counts as -inf, equal values go to the lower
// id, and a picked entry is masked out by a bit (not by overwriting its value),
// so k distinct ids in [0, E) come out whatever the logits hold.
template <int NVE>
__device__ int topk_row_n(const RouteArgs &a, int t, int32_t *s_out) {
    const int lane = threadIdx.x & 31;
    const float *z = a.ws.z + (size_t)t * a.E;
    const int nv = (a.E + 31) >> 5;
    float v[NVE];
    uint32_t avail = 0u;  // bit j: entry lane + 32 j is a real expert not yet picked
#pragma unroll
    for (int j = 0; j < NVE; ++j) {
        const int e = lane + 32 * j;
        const bool real = j < nv && e < a.E;
        const float zv = real ? z[e] : -INFINITY;
        v[j] = zv != zv ? -INFINITY : zv;
        if (real) avail |= 1u << j;
    }
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < NVE; ++j) m = fmaxf(m, v[j]);
    m = warp_max(m);
    float sall = 0.f;  // the full softmax denominator (only without renormalisation)
    if (!a.renorm) {
#pragma unroll
        for (int j = 0; j < NVE; ++j)
            if (lane + 32 * j < a.E) sall += expf(v[j] - m);
        sall = warp_sum(sall);
    }

    int my_idx = 0x7fffffff;
    float my_val = -INFINITY;
    for (int s = 0; s < a.k; ++s) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;  // lane-local candidates are visited in ascending id
#pragma unroll
        for (int j = 0; j < NVE; ++j)
            if (((avail >> j) & 1u) && (v[j] > bv || bi == 0x7fffffff)) { bv = v[j]; bi = lane + 32 * j; }
        // the warp's largest value (order-preserving integer key, two
        // single-instruction warp reductions), then the lowest id holding it
        const uint32_t key = order_key(bv);
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
        bi = (int)__reduce_min_sync(0xffffffffu, key == kmax ? (uint32_t)bi : 0xffffffffu);
        bv = key_value(kmax);
        if (lane == s) { my_idx = bi; my_val = bv; }
        if (bi < a.E && lane == (bi & 31)) avail &= ~(1u << (bi >> 5));
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
        if (s_out) s_out[t * a.k + rank] = my_idx;
    }
    return lane < a.k ? my_idx : -1;
}

// s_out: also the row's ids, ascending, in shared memory (or null).
__device__ int topk_row(const RouteArgs &a, int t, int32_t *s_out = nullptr) {
    const int nv = (a.E + 31) >> 5;
    if (nv <= 4) return topk_row_n<4>(a, t, s_out);
    if (nv <= 8) return topk_row_n<8>(a, t, s_out);
    if (nv <= 16) return topk_row_n<16>(a, t, s_out);
    return topk_row_n<kMaxE / 32>(a, t, s_out);
}

constexpr int kLookupMax = kMaxK * kDecodeMaxRows;  // entries of one lookup batch (>= kMaxE)

// Shared memory of one lookup batch.
struct LookupSmem {
    int32_t exp[kLookupMax];    // in: the batch's distinct experts, ascending
    int32_t slot[kLookupMax];   // out: slot of a hit, or -2 - slot for a miss
    int32_t evict[kLookupMax];  // out: key evicted from the slot, or -1
    int32_t rank[kLookupMax];
    int32_t victim[kLookupMax];
    int32_t old[kLookupMax];
    uint32_t hitmap[kMaxSlotBits / 32];
    unsigned long long clock, lastv;
    int nf, nhit, nmiss;
    unsigned long long redv[2][kRouteThreads / 32];  // per warp, by round parity
    int reds[2][kRouteThreads / 32];
};

// One lookup batch of `layer` over sm.exp[0..n), run by all threads of the CTA.
// All table reads happen in one parallel round (the batch's map entries, the
// header, every slot's stamp); hits get the newest stamps in ascending id;
// each miss in ascending id takes the lowest never-used slot, else the next
// least recently used non-hit slot (the smallest stamps, found by block-wide
// argmin rounds: stamps are unique, so round r takes the minimum above round
// r-1's).  Same result as the sequential rule.  *t_read: time after the reads.
// map_pre: this layer's E map entries already in shared memory, and the header
// already in sm.clock / sm.nf (read while the top-k ran); or null.
__device__ void lookup_batch(const Table &tab, int layer, int E, int n, LookupSmem &sm,
                             unsigned long long *t_read, const int32_t *map_pre = nullptr) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int64_t keybase = (int64_t)layer * E;
    const int C = (int)tab.C;
    if (tab.scratch_base >= 0) {  // static split: resident set fixed, misses to scratch slots
        for (int j = threadIdx.x; j < n; j += blockDim.x)
            sm.slot[j] = map_pre ? map_pre[sm.exp[j]] : tab.map[keybase + sm.exp[j]];
        __syncthreads();
        if (threadIdx.x == 0 && t_read) *t_read = global_ns();
        if (warp == 0) {
            int hc = 0, mc = 0;
            for (int j0 = 0; j0 < n; j0 += 32) {
                const int j = j0 + lane;
                const bool valid = j < n, hit = valid && sm.slot[j] >= 0;
                const unsigned hm = __ballot_sync(0xffffffffu, hit);
                const unsigned mm = __ballot_sync(0xffffffffu, valid && !hit);
                if (valid && !hit) {
                    const int m = mc + __popc(mm & ((1u << lane) - 1u));
                    sm.slot[j] = -2 - (tab.scratch_base + m);
                }
                if (valid) sm.evict[j] = -1;
                hc += __popc(hm);
                mc += __popc(mm);
            }
            if (lane == 0) { sm.nhit = hc; sm.nmiss = mc; }
        }
        __syncthreads();
        return;
    }
    for (int i = threadIdx.x; i < kMaxSlotBits / 32; i += blockDim.x) sm.hitmap[i] = 0u;
    for (int j = threadIdx.x; j < n; j += blockDim.x)
        sm.slot[j] = map_pre ? map_pre[sm.exp[j]] : tab.map[keybase + sm.exp[j]];
    if (threadIdx.x == 0 && !map_pre) { sm.clock = tab.hdr->clock; sm.nf = tab.hdr->next_free; }
    // this thread's slots tid + 256 i (past C: slot C - 1's stamp, never used --
    // the candidate test checks the slot; a select on the loaded value here
    // would make every thread wait for its loads before the barrier below)
    unsigned long long sv[kStampRegs];
#pragma unroll
    for (int i = 0; i < kStampRegs; ++i) {
        const int sl = threadIdx.x + kRouteThreads * i;
        sv[i] = tab.stamp[sl < C ? sl : C - 1];
    }
    __syncthreads();
    if (threadIdx.x == 0 && t_read) *t_read = global_ns();
    for (int j = threadIdx.x; j < n; j += blockDim.x)
        if (sm.slot[j] >= 0) atomicOr(&sm.hitmap[sm.slot[j] >> 5], 1u << (sm.slot[j] & 31));
    if (warp == 0) {  // ranks: hits and misses, each in ascending id
        int hc = 0, mc = 0;
        for (int j0 = 0; j0 < n; j0 += 32) {
            const int j = j0 + lane;
            const bool valid = j < n, hit = valid && sm.slot[j] >= 0;
            const unsigned hm = __ballot_sync(0xffffffffu, hit);
            const unsigned mm = __ballot_sync(0xffffffffu, valid && !hit);
            const unsigned lt = (1u << lane) - 1u;
            if (valid) sm.rank[j] = hit ? hc + __popc(hm & lt) : mc + __popc(mm & lt);
            hc += __popc(hm);
            mc += __popc(mm);
        }
        if (lane == 0) { sm.nhit = hc; sm.nmiss = mc; }
    }
    __syncthreads();
    const int nhit = sm.nhit, nmiss = sm.nmiss, nf = sm.nf;
    const int nfree = C - nf;
    const int nevict = nmiss > nfree ? nmiss - nfree : 0;
    // victim candidates of the register tile: stamp << 13 | slot for a used
    // (stamp > 0), non-hit slot, else ~0 (slots of the tile are < 2^13; stamps
    // count lookups, far below 2^51); a chosen one is cleared by its thread
    constexpr int kTileSlots = kRouteThreads * kStampRegs;
    static_assert(kTileSlots <= (1 << 13) && (kStampRegs & (kStampRegs - 1)) == 0, "tile key layout");
    // (built only when the batch evicts: it waits for the stamp loads)
    unsigned long long sk[kStampRegs];
    if (nevict > 0) {
#pragma unroll
        for (int i = 0; i < kStampRegs; ++i) {
            const int sl = threadIdx.x + kRouteThreads * i;
            const bool cand = sl < C && sv[i] != 0ull && !(sm.hitmap[sl >> 5] & (1u << (sl & 31)));
            sk[i] = cand ? (sv[i] << 13) | (unsigned long long)sl : ~0ull;
        }
    }
    unsigned long long last = 0ull;
    for (int r = 0; r < nevict; ++r) {
        // this thread's smallest key: pairwise minima in a tree (depth 5)
        unsigned long long tk[kStampRegs];
#pragma unroll
        for (int i = 0; i < kStampRegs; ++i) tk[i] = sk[i];
#pragma unroll
        for (int w = kStampRegs; w > 1; w >>= 1) {
#pragma unroll
            for (int i = 0; i < w / 2; ++i) tk[i] = tk[2 * i + 1] < tk[2 * i] ? tk[2 * i + 1] : tk[2 * i];
        }
        unsigned long long bv = ~0ull;
        int bs = -1;
        if (tk[0] != ~0ull) {
            bv = tk[0] >> 13;
            bs = (int)(tk[0] & ((1ull << 13) - 1ull));
        }
        for (int sl = threadIdx.x + kTileSlots; sl < C; sl += kRouteThreads) {
            const unsigned long long v = tab.stamp[sl];  // caches beyond the register tile
            if (v > last && v < bv && !(sm.hitmap[sl >> 5] & (1u << (sl & 31)))) { bv = v; bs = sl; }
        }
        // the warp's smallest stamp (stamps are unique: one slot holds it), by
        // 32-bit warp reductions over its halves
        const uint32_t hi = __reduce_min_sync(0xffffffffu, (uint32_t)(bv >> 32));
        const uint32_t lo = __reduce_min_sync(0xffffffffu, (uint32_t)(bv >> 32) == hi ? (uint32_t)bv : ~0u);
        const unsigned long long wv = ((unsigned long long)hi << 32) | lo;
        const uint32_t ws = __reduce_min_sync(0xffffffffu, bv == wv ? (uint32_t)bs : ~0u);
        if (lane == 0) {
            sm.redv[r & 1][warp] = wv;
            sm.reds[r & 1][warp] = (int)ws;
        }
        __syncthreads();
        // every thread takes the block's minimum (buffers alternate by round,
        // so the next round's writes cannot race these reads)
        unsigned long long mv = sm.redv[r & 1][0];
        int ms = sm.reds[r & 1][0];
        for (int w = 1; w < nw; ++w) {
            const unsigned long long ov = sm.redv[r & 1][w];
            if (ov < mv) {
                mv = ov;
                ms = sm.reds[r & 1][w];
            }
        }
        if (threadIdx.x == 0) sm.victim[r] = ms;
        last = mv;
        const int isel = (ms >= 0 && ms < kTileSlots && (ms % kRouteThreads) == (int)threadIdx.x) ? ms / kRouteThreads : -1;
#pragma unroll
        for (int i = 0; i < kStampRegs; ++i)
            if (i == isel) sk[i] = ~0ull;
    }
    __syncthreads();
    for (int r = threadIdx.x; r < nevict; r += blockDim.x) sm.old[r] = tab.owner[sm.victim[r]];
    __syncthreads();
    const unsigned long long clock = sm.clock;
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        const int s0 = sm.slot[j];
        if (s0 >= 0) {  // hit: newest stamps in ascending id
            tab.stamp[s0] = clock + 1 + sm.rank[j];
            sm.evict[j] = -1;
        } else {        // miss: a never-used slot, else the next least recently used
            const int m = sm.rank[j];
            int sl, ev = -1;
            if (m < nfree) sl = nf + m;
            else { sl = sm.victim[m - nfree]; ev = sm.old[m - nfree]; }
            const int key = (int)(keybase + sm.exp[j]);
            if (ev >= 0) tab.map[ev] = -1;
            tab.map[key] = sl;
            tab.owner[sl] = key;
            tab.stamp[sl] = clock + 1 + nhit + m;
            sm.slot[j] = -2 - sl;
            sm.evict[j] = ev;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        tab.hdr->clock = clock + n;
        tab.hdr->next_free = nf + (nmiss < nfree ? nmiss : nfree);
    }
    __syncthreads();
}

// Warp 0: one 16-byte record per batch entry at page->ev[base + j].
__device__ void publish_events(HostPage *page, int base, const LookupSmem &sm, int n, int prefetch) {
    const int lane = threadIdx.x & 31;
    for (int j = lane; j < n; j += 32) {
        const int sj = sm.slot[j];
        HostEvent he;
        he.expert = sm.exp[j];
        he.slot = sj >= 0 ? sj : -2 - sj;
        he.flags = (sj >= 0 ? 1 : 0) | (prefetch << 1);
        he.evicted = sm.evict[j];
        *reinterpret_cast<int4 *>(&page->ev[base + j]) = *reinterpret_cast<int4 *>(&he);
    }
}

template <int NV>
// split: warps per router row (1, 2, 4 or 8; d/8 divisible by it): more CTAs
// pull the router's bytes, and each holds fewer of them in flight.
__global__ void __launch_bounds__(kRouteThreads) route_lookup_kernel(RouteArgs a, int rows_per_chunk, int split) {
    extern __shared__ __align__(16) uint4 xs[];  // x rows of one chunk (bf16)
    const unsigned long long t_entry = global_ns();  // early: launched before the previous layer ends
    unsigned long long t_logits = 0, t_elect = 0, t_topk = 0, t_jobs = 0, t_read = 0, t_table = 0;
    // static data first: this warp's segment of its router row and the next layer's rows (L2)
    const int seg = (int)(threadIdx.x >> 5) % split;
    const int e_row = blockIdx.x * ((blockDim.x >> 5) / split) + (int)(threadIdx.x >> 5) / split;
    const bool has_row = e_row < a.E;
    uint4 w[NV];
    {
        const int lane = threadIdx.x & 31, segv = (a.d >> 3) / split;
        const uint4 *wrow = reinterpret_cast<const uint4 *>(a.Wr + (size_t)(has_row ? e_row : 0) * a.d) + seg * segv;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int v = lane + 32 * i;
            w[i] = (has_row && v < segv) ? ld_nc16(wrow + v) : make_uint4(0, 0, 0, 0);
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
    if (threadIdx.x == 0) span_mark(a.span, 0);
    router_logits<NV>(a, w, e_row, has_row, xs, rows_per_chunk, split, seg);

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
    __shared__ LookupSmem sm;
    // this layer's map entries (behind the x rows in dynamic shared memory) and
    // the table header, loaded by the warps without a top-k row while the top-k
    // runs (only this kernel writes the table, and the previous layer's launch
    // is complete): the lookup then reads them without an L2 round trip
    int32_t *s_map = reinterpret_cast<int32_t *>(xs + ((size_t)rows_per_chunk * a.d * 2 + 15) / 16);
    const int tw = a.T < nw ? a.T : nw;  // warps with top-k rows
    const int64_t keybase = (int64_t)a.layer * a.E;
    auto preload = [&](int first) {
        for (int e = (int)threadIdx.x - first; e < a.E; e += (int)blockDim.x - first) s_map[e] = a.tab.map[keybase + e];
        if ((int)threadIdx.x == first) {
            sm.clock = a.tab.hdr->clock;
            sm.nf = a.tab.hdr->next_free;
        }
    };
    // the selected ids, ascending per row, also go to shared memory (the job
    // list reads them there, not back from global memory)
    __shared__ int32_t s_idx[kMaxK * kDecodeMaxRows];
    if (tw < nw && warp >= tw) preload(32 * tw);
    for (int t = warp; t < a.T; t += nw) topk_row(a, t, s_idx);
    if (tw == nw) preload(0);

    // ---- distinct experts of the batch, ascending: a bitmap over E
    __shared__ uint32_t s_bits[kMaxE / 32];
    __shared__ int s_base[kMaxE / 32];
    __shared__ int s_njobs;
    __shared__ int32_t s_cnt[kMaxK * kDecodeMaxRows];
    __shared__ int32_t s_off[kMaxK * kDecodeMaxRows];
    int32_t *s_exp = sm.exp;
    for (int i = threadIdx.x; i < kMaxE / 32; i += blockDim.x) s_bits[i] = 0u;
    __syncthreads();
    if (threadIdx.x == 0) t_topk = global_ns();
    const int nsel = a.T * a.k;
    if (a.T == 1) {
        // one row: its k ids are already distinct and ascending -- they (the
        // owned ones, with expert parallelism) are the jobs, one row each
        if (warp == 0) {
            int e = lane < a.k ? s_idx[lane] : 0;
            if (lane < a.k && (unsigned)e >= (unsigned)a.E) { route_fail(a.page, 1, e, a.E); e = 0; }
            const bool own = lane < a.k && e % a.ep_size == a.ep_rank;
            const unsigned ob = __ballot_sync(0xffffffffu, own);
            const int pos = __popc(ob & ((1u << lane) - 1u));
            if (own) {
                s_exp[pos] = e;
                s_cnt[pos] = 1;
                s_off[pos] = pos;
                a.ws.rowrefs[pos].t = 0;
                a.ws.rowrefs[pos].p = (int16_t)lane;
            }
            if (lane == 0) s_njobs = __popc(ob);
        }
        __syncthreads();
    } else {
        for (int i = threadIdx.x; i < nsel; i += blockDim.x) {
            const int e = s_idx[i];
            if ((unsigned)e >= (unsigned)a.E) route_fail(a.page, 1, e, a.E);
            else if (e % a.ep_size == a.ep_rank) atomicOr(&s_bits[e >> 5], 1u << (e & 31));
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
        const int nj = s_njobs;
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
            const uint32_t w = s_bits[e >> 5];
            if (w & (1u << (e & 31))) s_exp[s_base[e >> 5] + __popc(w & ((1u << (e & 31)) - 1u))] = e;
        }
        __syncthreads();
        for (int j = threadIdx.x; j < nj; j += blockDim.x) {
            int c = 0;
            for (int i = 0; i < nsel; ++i) c += (s_idx[i] == s_exp[j]);
            s_cnt[j] = c;
        }
        __syncthreads();
        if (warp == 0) {  // exclusive scan of the counts, 32 at a time
            int carry = 0;
            for (int j0 = 0; j0 < nj; j0 += 32) {
                const int j = j0 + lane;
                const int c = j < nj ? s_cnt[j] : 0;
                int incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                if (j < nj) s_off[j] = carry + incl - c;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
        __syncthreads();
        for (int j = threadIdx.x; j < nj; j += blockDim.x) {
            int pos = s_off[j];
            for (int i = 0; i < nsel; ++i)
                if (s_idx[i] == s_exp[j]) {
                    a.ws.rowrefs[pos].t = (int16_t)(i / a.k);
                    a.ws.rowrefs[pos].p = (int16_t)(i % a.k);
                    ++pos;
                }
        }
    }  // T > 1
    const int njobs = s_njobs;

    __syncthreads();
    if (threadIdx.x == 0) t_jobs = global_ns();

    // ---- cache lookup: one batch, ascending id
    lookup_batch(a.tab, a.layer, a.E, njobs, sm, &t_read, s_map);
    const int nmiss = sm.nmiss;
    if (threadIdx.x == 0) {
        *a.ws.n_misses = nmiss;
        t_table = global_ns();
    }

    // ---- publish: one 16-byte record per entry, the counts and phase times,
    // then the flag with one system-scope release store (cumulative: the
    // warp's writes, ordered before it by the warp barrier, land first)
    if (warp == 0) {
        publish_events(a.page, 0, sm, njobs, 0);
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
            a.page->phase_ns[6] = (uint32_t)(global_ns() - t_table);
            a.page->phase_ns[7] = (uint32_t)(t_start - t_entry);  // launch-to-start: PDL wait
        }
        __syncwarp();
        if (lane == 0 && a.publish) {
            const uint32_t v = a.seq;
            asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(&a.page->seq), "r"(v) : "memory");
        }
    }
    __syncthreads();
    for (int j = threadIdx.x; j < njobs; j += blockDim.x) {
        const int sj = sm.slot[j];
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
    if (a.span) {
        __syncthreads();
        if (threadIdx.x == 0) span_mark(a.span, 1);
    }
}

// ------------------------------------------------------------------ prefill --
// Rows of a prefill chunk (T > 32): logits per (8 rows x 64 experts) CTA with
// the rows in shared memory; top-k per row with per-expert counts; one CTA for
// the lookup of the layer's distinct experts and of all experts of the next
// layer (the prefetch batch, holude.com "長いプロンプトとエージェント処理も意識している":
// the next layer's experts stream in while the current layer computes); then
// the rows are scattered into per-expert groups.
constexpr int kPfRows = 8, kPfExperts = 64;

template <int NV>
__global__ void __launch_bounds__(kRouteThreads) prefill_logits_kernel(RouteArgs a) {
    extern __shared__ __align__(16) uint4 xsm[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = blockIdx.x * kPfRows, e0 = blockIdx.y * kPfExperts;
    const int nr = a.T - t0 < kPfRows ? a.T - t0 : kPfRows;
    const int nvec = a.d >> 3;
    const uint4 *xg = reinterpret_cast<const uint4 *>(a.x + (size_t)t0 * a.d);
    for (int i = threadIdx.x; i < nr * nvec; i += blockDim.x) xsm[i] = __ldg(xg + i);
    __syncthreads();
    for (int ee = 0; ee < kPfExperts / (kRouteThreads / 32); ++ee) {
        const int e = e0 + warp * (kPfExperts / (kRouteThreads / 32)) + ee;
        if (e >= a.E) break;
        const uint4 *wrow = reinterpret_cast<const uint4 *>(a.Wr + (size_t)e * a.d);
        uint4 w[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int v = lane + 32 * i;
            w[i] = v < nvec ? __ldg(wrow + v) : make_uint4(0, 0, 0, 0);
        }
        float acc[kPfRows];
#pragma unroll
        for (int r = 0; r < kPfRows; ++r) acc[r] = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int v = lane + 32 * i;
            if (v < nvec) {
                float wf[8];
                bf16x8_to_f32(w[i], wf);
#pragma unroll
                for (int r = 0; r < kPfRows; ++r) {
                    if (r < nr) {
                        float xf[8];
                        bf16x8_to_f32(xsm[r * nvec + v], xf);
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[r] = fmaf(wf[j], xf[j], acc[r]);
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kPfRows; ++r) {
            const float sum = warp_sum(acc[r]);
            if (lane == 0 && r < nr) a.ws.z[(size_t)(t0 + r) * a.E + e] = sum;
        }
    }
}

__global__ void __launch_bounds__(kRouteThreads) prefill_topk_kernel(RouteArgs a) {
    const int t = blockIdx.x * (kRouteThreads / 32) + (threadIdx.x >> 5);
    if (t >= a.T) return;
    const int e = topk_row(a, t);
    if ((unsigned)e < (unsigned)a.E) {
        if (e % a.ep_size == a.ep_rank) atomicAdd(&a.ws.cnt[e], 1);  // (this rank's experts)
    } else if ((threadIdx.x & 31) < a.k) {
        route_fail(a.page, 2, e, a.E);
    }
}

__global__ void __launch_bounds__(kRouteThreads) prefill_lookup_kernel(RouteArgs a) {
    __shared__ LookupSmem sm;
    __shared__ int32_t s_cnt[kMaxE], s_off[kMaxE];
    __shared__ int s_n, s_nmiss;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp == 0) {  // the layer's distinct experts, ascending, with their row counts
        int nj = 0;
        for (int e0 = 0; e0 < a.E; e0 += 32) {
            const int e = e0 + lane;
            const int c = e < a.E ? a.ws.cnt[e] : 0;
            const unsigned m = __ballot_sync(0xffffffffu, c > 0);
            const int pos = nj + __popc(m & ((1u << lane) - 1u));
            if (c > 0) { sm.exp[pos] = e; s_cnt[pos] = c; a.ws.jobidx[e] = pos; }
            else if (e < a.E) a.ws.jobidx[e] = -1;
            if (e < a.E) a.ws.fill[e] = 0;
            nj += __popc(m);
        }
        int carry = 0;  // exclusive scan of the counts: each group's first row
        for (int j0 = 0; j0 < nj; j0 += 32) {
            const int j = j0 + lane;
            const int c = j < nj ? s_cnt[j] : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (j < nj) s_off[j] = carry + incl - c;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            s_n = nj;
            *a.ws.n_grouped = nj > 0 ? carry : 0;  // routed grouped rows (carry: their total)
        }
    }
    __syncthreads();
    const int n = s_n;
    lookup_batch(a.tab, a.layer, a.E, n, sm, nullptr);
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        const int sj = sm.slot[j];
        Job jb;
        jb.expert = sm.exp[j];
        jb.slot = sj >= 0 ? sj : -2 - sj;
        jb.hit = sj >= 0;
        jb.nrows = s_cnt[j];
        jb.row_off = s_off[j];
        jb.pad[0] = jb.pad[1] = jb.pad[2] = 0;
        a.ws.jobs[j] = jb;
    }
    if (warp == 0) publish_events(a.page, 0, sm, n, 0);
    if (threadIdx.x == 0) {
        s_nmiss = sm.nmiss;
        *a.ws.n_jobs = n;
        *a.ws.n_misses = sm.nmiss;
    }
    __syncthreads();  // the routed batch is consumed before the prefetch batch reuses sm
    int npf = 0, pf_miss = 0;
    if (a.prefetch && a.layer + 1 < a.L) {  // all of the next layer's experts (this rank's)
        if (warp == 0) {
            int c = 0;
            for (int e0 = 0; e0 < a.E; e0 += 32) {
                const int e = e0 + lane;
                const bool own = e < a.E && e % a.ep_size == a.ep_rank;
                const unsigned ob = __ballot_sync(0xffffffffu, own);
                if (own) sm.exp[c + __popc(ob & ((1u << lane) - 1u))] = e;
                c += __popc(ob);
            }
            if (lane == 0) s_n = c;
        }
        __syncthreads();
        npf = s_n;
        lookup_batch(a.tab, a.layer + 1, a.E, npf, sm, nullptr);
        if (warp == 0) publish_events(a.page, n, sm, npf, 1);
        pf_miss = sm.nmiss;
    }
    if (warp == 0) {
        if (lane == 0) {
            a.page->n_events = n + npf;
            a.page->n_jobs = n;
            a.page->n_misses = s_nmiss;
            a.page->n_prefetch_misses = pf_miss;
        }
        __threadfence_system();
        __syncwarp();
        if (lane == 0 && a.publish) {
            __threadfence_system();
            a.page->seq = a.seq;
        }
    }
}

__global__ void prefill_scatter_kernel(RouteArgs a) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.T * a.k) return;
    const int e = a.ws.idx[i];
    if ((unsigned)e >= (unsigned)a.E) { route_fail(a.page, 3, e, a.E); return; }
    if (e % a.ep_size != a.ep_rank) return;  // another rank's expert
    const int j = a.ws.jobidx[e];
    if (j < 0) { route_fail(a.page, 4, e, a.E); return; }
    const int pos = a.ws.jobs[j].row_off + atomicAdd(&a.ws.fill[e], 1);
    a.ws.rowrefs[pos].t = (int16_t)(i / a.k);
    a.ws.rowrefs[pos].p = (int16_t)(i % a.k);
}

template <int NV>
cudaError_t launch_prefill_nv(const RouteArgs &a, cudaStream_t s) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(prefill_logits_kernel<NV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const dim3 grid((a.T + kPfRows - 1) / kPfRows, (a.E + kPfExperts - 1) / kPfExperts);
    prefill_logits_kernel<NV><<<grid, kRouteThreads, (size_t)kPfRows * a.d * 2, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prefill_topk_kernel<<<(a.T + kRouteThreads / 32 - 1) / (kRouteThreads / 32), kRouteThreads, 0, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prefill_lookup_kernel<<<1, kRouteThreads, 0, s>>>(a);
    return cudaGetLastError();
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

// Static per-layer split: expert e < per_layer of layer l resident in slot
// l*per_layer + e; every other key absent; the scratch slots unowned.
__global__ void table_static_kernel(Table t, int L, int E, int per_layer) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t nkeys = (int64_t)L * E;
    for (int64_t j = i; j < nkeys; j += stride) {
        const int l = (int)(j / E), e = (int)(j - (int64_t)l * E);
        t.map[j] = e < per_layer ? l * per_layer + e : -1;
    }
    for (int64_t j = i; j < t.C; j += stride) {
        const bool resident = j < (int64_t)L * per_layer;
        t.owner[j] = resident ? (int)((j / per_layer) * E + j % per_layer) : -1;
        t.stamp[j] = 0ull;
    }
    if (i == 0) {
        t.hdr->clock = 0ull;
        t.hdr->next_free = L * per_layer;
    }
}

template <int NV>
cudaError_t launch_nv(const RouteArgs &a, int grid, int split, cudaStream_t s) {
    static bool configured = false;  // allow up to 64 KB of dynamic smem (x chunk + map entries)
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(route_lookup_kernel<NV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    int rows = (48 * 1024) / (a.d * 2);
    if (rows < 1) rows = 1;
    if (rows > a.T) rows = a.T;
    // the x chunk, then (16-byte aligned) the layer's E map entries
    const size_t smem = (((size_t)rows * a.d * 2 + 15) & ~(size_t)15) + (size_t)a.E * 4;
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
    return cudaLaunchKernelEx(&cfg, route_lookup_kernel<NV>, a, rows, split);
}

}  // namespace

cudaError_t launch_route_lookup(const RouteArgs &a, cudaStream_t s) {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    const int warps = kRouteThreads / 32;
    const int nvec = a.d >> 3;
    // warps per router row: split while the grid stays within one CTA per SM
    // and every lane keeps at least one 16-byte vector of its segment
    int split = 1;
    while (split < 8 && (int64_t)a.E * 2 * split <= (int64_t)warps * sms && nvec % (2 * split) == 0 &&
           nvec / (2 * split) >= 32)
        split *= 2;
    const int grid = (a.E + warps / split - 1) / (warps / split);
    const int nv = (nvec / split + 31) >> 5;  // 16-byte vectors per lane per segment
    if (nv <= 1) return launch_nv<1>(a, grid, split, s);
    if (nv <= 2) return launch_nv<2>(a, grid, split, s);
    if (nv <= 4) return launch_nv<4>(a, grid, split, s);
    if (nv <= 8) return launch_nv<8>(a, grid, split, s);
    if (nv <= 12) return launch_nv<12>(a, grid, split, s);
    if (nv <= 16) return launch_nv<16>(a, grid, split, s);
    return cudaErrorInvalidValue;
}

// Prefill selection on logits already in ws.z: top-k + counts, then the
// lookup CTA.  The caller zeroes ws.cnt first.
cudaError_t launch_prefill_select(const RouteArgs &a, cudaStream_t s) {
    prefill_topk_kernel<<<(a.T + kRouteThreads / 32 - 1) / (kRouteThreads / 32), kRouteThreads, 0, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prefill_lookup_kernel<<<1, kRouteThreads, 0, s>>>(a);
    return cudaGetLastError();
}

// Prefill routing: logits, top-k + counts, then the lookup CTA (which
// publishes the miss and prefetch lists).  The caller zeroes ws.cnt first.
cudaError_t launch_prefill_route(const RouteArgs &a, cudaStream_t s) {
    const int nv = ((a.d >> 3) + 31) >> 5;
    if (nv <= 1) return launch_prefill_nv<1>(a, s);
    if (nv <= 2) return launch_prefill_nv<2>(a, s);
    if (nv <= 4) return launch_prefill_nv<4>(a, s);
    if (nv <= 8) return launch_prefill_nv<8>(a, s);
    if (nv <= 12) return launch_prefill_nv<12>(a, s);
    if (nv <= 16) return launch_prefill_nv<16>(a, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_prefill_scatter(const RouteArgs &a, cudaStream_t s) {
    const int n = a.T * a.k;
    prefill_scatter_kernel<<<(n + 255) / 256, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_table_reset(Table t, int64_t nkeys, cudaStream_t s) {
    table_reset_kernel<<<256, 256, 0, s>>>(t, nkeys);
    return cudaGetLastError();
}

cudaError_t launch_table_static(Table t, int L, int E, int per_layer, cudaStream_t s) {
    table_static_kernel<<<256, 256, 0, s>>>(t, L, E, per_layer);
    return cudaGetLastError();
}

}  // namespace moe
