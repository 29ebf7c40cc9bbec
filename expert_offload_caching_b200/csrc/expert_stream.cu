// Streaming expert GEMVs for decode (W4A16 over NVFP4 / MXFP4 records):
// gate/up with fused SwiGLU, down, and the gate-weighted combine.
//
// The arithmetic is the routed expert of the FreeToken pages (florigen.ai
// "NVFP4で約135GBまで縮める": NVFP4 routed experts; ai-hardware-zukan
// "GPUに載らない分をどう間に合わせるか": MXFP4 checkpoints):
//   h_j = silu(g_j) * u_j,  g = W1 x, u = W3 x;   y_e = W2 h;
//   y = sum over selected e (ascending id) of gate_e * y_e + y_shared.
//
// Decode reads each weight once for 1-32 activation rows, so the launch is
// bound by how many weight bytes are in flight, not by math.  Design:
//   * one CTA per SM; warp 0's lane 0 is the producer: it walks the CTA's
//     work items (a few consecutive 16-row weight tiles of one expert, whose
//     codes and scales are contiguous in the record) and moves each with two
//     1-D bulk copies (cp.async.bulk, completion counted on the stage's
//     mbarrier, L2 evict-first) into a ring of shared-memory stages; it waits
//     for a stage's previous item to be released before reusing it;
//   * consumer warps (warps 1..C) take the CTA's items in turn (item l: warp
//     1 + l mod C, stage l mod S, with S a multiple of C, so each stage serves
//     one warp and its uses are waited on in order); a warp
//     computes every tile of its item over the whole K by itself, so there is
//     no cross-warp reduction and no CTA barrier per item: it waits on the
//     stage's full barrier, runs the K-steps (E2M1 decoded in registers,
//     block scales applied in fp16, mma.sync m16n8k16 with fp32 accumulation:
//     the K-step code of gemv_inner.cuh), releases the stage, and writes its
//     outputs;
//   * phase 3 launches run an expert's down tiles in the same launch as its
//     gate/up tiles: every CTA's items are gate/up items first, so a down item
//     waits (bounded) only for gate/up items that never wait -- deadlock-free
//     with every CTA resident (one per SM);
//   * combine: a down launch with combine set has the warp that completes the
//     last expert of a 16-row output tile (per-tile ticket) sum the tile's rows
//     over the layer's selected experts in ascending id, plus the shared
//     expert's partial.
// Every wait is bounded (globaltimer, the launch's wait_ns); a wait that runs
// out writes the mapped page's error word, the CTA stops, and no bulk copy
// outlives it.
#include "gemv_inner.cuh"

namespace moe {

namespace {

using namespace gemv;

constexpr int kStMaxStages = 8;
constexpr int kStMaxGroups = 5;                // consumer warp groups (P warps each) + the producer warp
// (with the producer, 16 or 11 warps: at most four per SM sub-partition, so
// up to 128 registers per thread for groups of three)
__host__ __device__ constexpr int st_max_groups(int P) { return kStMaxGroups; }
constexpr int kErrStreamFull = 42;             // a stage's copy did not land in time
constexpr int kErrStreamEmpty = 43;            // a stage was not released in time
constexpr int kErrStreamDep = 44;              // a down item's gate/up tiles did not complete in time
constexpr int kErrStreamSize = 45;             // more experts than the metadata area holds

struct ExpMeta {            // one expert of the launch (dynamic shared memory)
    const uint8_t *rec;     // its record (slot in the arena, or the shared record)
    int nrows, row_off;     // rows using it, first row ref
    float ts[3];            // NVFP4 tensor scales (gate, up, down)
    int job;                // job index, -1: the shared expert
    int cnt;                // phase 3: gate/up tiles of it this CTA completed
    int pad;
};
static_assert(sizeof(ExpMeta) == 40, "metadata stride");

__device__ __forceinline__ unsigned long long st_now() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ uint32_t st_ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void st_mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void st_mbar_expect(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool st_mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}
// Wait for the phase of the given parity; false when the deadline passes or
// the CTA is stopping.
__device__ __forceinline__ bool st_mbar_wait(uint64_t *bar, uint32_t parity, unsigned long long deadline,
                                             volatile int *stop) {
    for (uint32_t i = 0;; ++i) {
        if (st_mbar_test(bar, parity)) return true;
        if ((i & 31u) == 31u && (*stop || st_now() > deadline)) return false;
    }
}
// 1-D bulk copy global -> this CTA's shared memory (16-byte aligned, size a
// multiple of 16), completion counted on bar; L2 evict-first (read once).
__device__ __forceinline__ void st_bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ void st_fail(const GemvArgs &a, int code, int item, int what) {
    HostPage *pg = a.page;
    pg->diag[1] = 31;  // kernel: expert_stream
    pg->diag[2] = (int)blockIdx.x;
    pg->diag[3] = item;
    pg->diag[4] = what;
    pg->diag[5] = a.phase;
    __threadfence_system();
    pg->error = code;
    __threadfence_system();
}

// A work item: expert e (launch-local), gate/up (else down), tiles
// [tile0, tile0 + nt).  Items are numbered gate/up first (expert-major), then
// down (phase 3).
struct StItem {
    int e, gate_up, tile0, nt;
};
__device__ __forceinline__ StItem st_item(int g, int phase, int nexp, int nA, int nB, int iA, int iB, int tpa,
                                          int tpb) {
    StItem it;
    const int gA = (phase & 1) ? nexp * iA : 0;
    if (g < gA) {
        it.e = g / iA;
        it.tile0 = (g - it.e * iA) * tpa;
        it.nt = min(tpa, nA - it.tile0);
        it.gate_up = 1;
    } else {
        g -= gA;
        it.e = g / iB;
        it.tile0 = (g - it.e * iB) * tpb;
        it.nt = min(tpb, nB - it.tile0);
        it.gate_up = 0;
    }
    return it;
}

// kFull: d and F are multiples of 256, so every K-step chunk is in range.
// kSA: activations from shared memory -- x staged once per CTA, and a down
// item's h rows copied into its stage by the group after h is complete
// (T <= 2); else they are read from global memory.
template <int NG, int FMT, int P, bool kFull, bool kSA>
__global__ void __launch_bounds__(32 * (P * st_max_groups(P) + 1), 1) expert_stream_kernel(GemvArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t s_full[kStMaxStages], s_empty[kStMaxStages];
    __shared__ __align__(8) uint64_t s_xbar, s_hbar[kStMaxGroups];
    __shared__ int s_nexp, s_last, s_combine;
    __shared__ int s_head_exp, s_head_slot;  // phase 3 with head_bytes: the layer's first miss
    __shared__ int s_pair_ok[st_max_groups(P)];
    __shared__ float s_red[st_max_groups(P) * 2 * (P - 1) * NG * 4 * 32];  // [group][buffer][member 1..P-1][NG][4][32]
    __shared__ volatile int s_stop;
    constexpr bool kMx = FMT == kFmtMxfp4;
    constexpr int kActA = kSA ? 2 : 0, kActB = kSA ? 2 : 1;  // activation loads: gate/up (x), down (h)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NS = a.ns, C = a.nc;
    ExpMeta *meta = reinterpret_cast<ExpMeta *>(smem + a.meta_off);
    RowRef *rrs = reinterpret_cast<RowRef *>(smem + a.rr_off);
    __half *xs = reinterpret_cast<__half *>(smem + a.x_off);  // kSA: [T][2][d] fp16 (hi, lo)

    pdl_wait();  // the job list, x and the row refs come from the route kernel; h from gate/up
    const unsigned long long deadline = st_now() + a.wait_ns;
    // diagnostic trace: slot 0 start, 1 set-up done, 2 gate/up counts published, 3 end;
    // group 0 / member 0's first 8 items: 4 + 3k stage wait begins, 5 + 3k data in, 6 + 3k sums in
    unsigned long long *tr = (a.trace && blockIdx.x < kTraceCtas) ? a.trace + (size_t)blockIdx.x * kTraceSlots : nullptr;
    auto stamp = [&](int slot) { if (tr) tr[slot] = st_now(); };
    if (threadIdx.x == 0) {
        stamp(0);
        span_mark(a.span, 0);
        s_stop = 0;
        for (int s = 0; s < NS; ++s) {
            st_mbar_init(&s_full[s], 1);   // the producer's expect-tx arrive (+ the bytes)
            st_mbar_init(&s_empty[s], 1);  // the group that used the stage
        }
        st_mbar_init(&s_xbar, 1);
        for (int g = 0; g < C; ++g) st_mbar_init(&s_hbar[g], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (kSA && (a.phase & 1)) {  // x as fp16 (hi, lo) rows, one bulk copy (written by the route kernel, complete)
            const uint32_t xb = (uint32_t)a.T * 4u * (uint32_t)a.d;
            st_mbar_expect(&s_xbar, xb);
            st_bulk_g2s(xs, a.act, xb, &s_xbar, evict_first_policy());
        }
    }
    pdl_launch_dependents();

    // ---- the launch's experts: hit jobs in ascending job index, then the
    // shared expert; or the one job only_job.  Each lane reads whole job
    // records (one L2 round trip after the count).
    if (warp == 0) {
        int cnt = 0;
        auto put = [&](int pos, int j, const Job &jb) {
            ExpMeta &m = meta[pos];
            m.job = j;
            m.rec = a.arena + (int64_t)jb.slot * a.rec_bytes;
            m.nrows = jb.nrows;
            m.row_off = jb.row_off;
            m.cnt = 0;
        };
        auto load_job = [&](int j) {
            union {
                Job jb;
                uint4 v[2];
            } u;
            const uint4 *src = reinterpret_cast<const uint4 *>(a.jobs + j);  // 32-byte records
            u.v[0] = __ldcg(src);
            u.v[1] = __ldcg(src + 1);
            return u.jb;
        };
        int head = -1;  // the first miss (lowest job index): its expert and slot
        if (a.only_job >= 0) {
            if (lane == 0) put(0, a.only_job, load_job(a.only_job));
            cnt = 1;
        } else {
            const int nj = __ldcg(a.n_jobs);
            for (int b = 0; b < nj; b += 32) {
                const int j = b + lane;
                Job jb;
                bool hit = false, miss = false;
                if (j < nj) {
                    jb = load_job(j);
                    hit = jb.hit != 0;
                    miss = !hit;
                }
                const unsigned ball = __ballot_sync(0xffffffffu, hit);
                const int pos = cnt + __popc(ball & ((1u << lane) - 1u));
                if (hit && pos < a.exp_cap) put(pos, j, jb);
                cnt += __popc(ball);
                const unsigned mb = __ballot_sync(0xffffffffu, miss);
                if (head < 0 && mb) {
                    const int src = __ffs(mb) - 1;
                    const int ex = __shfl_sync(0xffffffffu, jb.expert, src);
                    const int sl = __shfl_sync(0xffffffffu, jb.slot, src);
                    if (lane == 0) {
                        s_head_exp = ex;
                        s_head_slot = sl;
                    }
                    head = 1;
                }
            }
            if (a.shared_item) {
                if (lane == 0 && cnt < a.exp_cap) {
                    ExpMeta &m = meta[cnt];
                    m.job = -1;
                    m.rec = a.shared_rec;
                    m.nrows = a.T;
                    m.row_off = 0;
                    m.cnt = 0;
                }
                ++cnt;
            }
        }
        if (lane == 0 && head < 0) s_head_exp = -1;
        if (lane == 0) {
            if (cnt > a.exp_cap) {  // cannot happen with the host's sizing; refuse rather than overrun
                st_fail(a, kErrStreamSize, cnt, a.exp_cap);
                s_stop = 1;
                cnt = 0;
            }
            s_nexp = cnt;
        }
    } else if (warp == 1 && lane == 0) {
        // combine here: always (1), or (2) only if the lookup had no miss (the
        // route kernel, complete, wrote the count)
        s_combine = a.combine == 1 || (a.combine == 2 && __ldcg(a.n_misses) == 0);
    }
    for (int i = threadIdx.x; i < a.T * a.k; i += blockDim.x) rrs[i] = a.rowrefs[i];
    __syncthreads();
    if (threadIdx.x == 0) stamp(1);
    const int nexp = s_nexp;
    const bool combine = s_combine != 0;

    // ---- item geometry
    const int nA = a.F >> 3, nB = a.d >> 4;  // tiles per expert: 8 gate/up row pairs, 16 down rows
    const int iA = (nA + a.tpa - 1) / a.tpa, iB = (nB + a.tpb - 1) / a.tpb;
    const int total = nexp * (((a.phase & 1) ? iA : 0) + ((a.phase & 2) ? iB : 0));
    const int G = (int)gridDim.x;
    const int n_my = (int)blockIdx.x < total ? (total - 1 - (int)blockIdx.x) / G + 1 : 0;
    const uint32_t cbA = 8u * (uint32_t)a.d, sbA = kMx ? (uint32_t)(a.d >> 1) : (uint32_t)a.d;
    const uint32_t cbB = 8u * (uint32_t)a.F, sbB = kMx ? (uint32_t)(a.F >> 1) : (uint32_t)a.F;
    // stage layout: codes of the item's nt tiles, their scales, 16 bytes of
    // tensor scales (NVFP4), then (kSA, down items) the expert's h rows
    auto ts_off = [&](const StItem &it) { return (uint32_t)it.nt * (it.gate_up ? cbA + sbA : cbB + sbB); };

    if (nexp == 0 && combine && blockIdx.x == 0) {
        // nothing of this layer is computed here (an expert-parallel shard that
        // owns none of the selected experts): its partial output is the shared
        // expert's (computed by earlier launches) or zero
        for (int i = threadIdx.x; i < a.T * a.d; i += blockDim.x) {
            const int t = i / a.d, o = i - t * a.d;
            a.y[i] = a.shared_part ? __ldcg(a.part_out + ((size_t)t * (a.k + 1) + a.k) * a.d + o) : 0.f;
        }
    }

    if (a.phase == 3 && a.head_bytes && s_head_exp >= 0) {
        // every thread of every CTA, before its own work: the head of the
        // layer's first miss, from the page-locked pool over PCIe straight into
        // its slot (16-byte loads, four in flight per thread: megabytes in
        // flight over the grid, enough to keep the link busy) while the copy
        // engine is still starting on the rest of the record.  The launch's own
        // items wait meanwhile; they are not on the layer's critical path.
        const int64_t rec_idx = ((int64_t)a.layer * a.E + s_head_exp) % a.pool_P;
        const uint4 *src = reinterpret_cast<const uint4 *>(a.pool_d + rec_idx * a.rec_bytes);
        uint4 *dst = reinterpret_cast<uint4 *>(const_cast<uint8_t *>(a.arena) + (int64_t)s_head_slot * a.rec_bytes);
        const int64_t n16 = a.head_bytes >> 4, step = (int64_t)gridDim.x * blockDim.x;
        int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
        for (; i + 3 * step < n16; i += 4 * step) {
            const uint4 v0 = __ldcv(src + i), v1 = __ldcv(src + i + step), v2 = __ldcv(src + i + 2 * step),
                        v3 = __ldcv(src + i + 3 * step);
            dst[i] = v0;
            dst[i + step] = v1;
            dst[i + 2 * step] = v2;
            dst[i + 3 * step] = v3;
        }
        for (; i < n16; i += step) dst[i] = __ldcv(src + i);
    }

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol = evict_first_policy();
            int issued = 0, skipped = -1;
            for (int l = 0; l < n_my; ++l) {
                const int s = l % NS, n = l / NS;
                if (n > 0 && !st_mbar_wait(&s_empty[s], (n - 1) & 1, deadline, &s_stop)) {
                    if (!s_stop) st_fail(a, kErrStreamEmpty, l, s);
                    s_stop = 1;
                    break;
                }
                const StItem it = st_item((int)blockIdx.x + l * G, a.phase, nexp, nA, nB, iA, iB, a.tpa, a.tpb);
                const uint32_t cb = it.gate_up ? cbA : cbB, sb = it.gate_up ? sbA : sbB;
                const uint8_t *rec = meta[it.e].rec;
                const uint8_t *codes = rec + (it.gate_up ? a.lay.w13_codes : a.lay.w2_codes) + (int64_t)it.tile0 * cb;
                const uint8_t *scales = rec + (it.gate_up ? a.lay.w13_scales : a.lay.w2_scales) + (int64_t)it.tile0 * sb;
                uint8_t *dst = smem + (size_t)s * a.stage_bytes;
                issued = l + 1;
                if (a.inj_skip && blockIdx.x == 0 && l == 0) {  // test injection: this stage never fills
                    skipped = 0;
                    continue;
                }
                st_mbar_expect(&s_full[s], (uint32_t)it.nt * (cb + sb) + (kMx ? 0u : 16u));
                st_bulk_g2s(dst, codes, (uint32_t)it.nt * cb, &s_full[s], pol);
                st_bulk_g2s(dst + (size_t)it.nt * cb, scales, (uint32_t)it.nt * sb, &s_full[s], pol);
                if (!kMx)  // the record's tensor scales (gate, up, down; 12 of 16 bytes)
                    st_bulk_g2s(dst + (size_t)it.nt * (cb + sb), rec + a.lay.tscales, 16u, &s_full[s], pol);
            }
            // no copy outlives the CTA: the last item issued into each stage has landed
            const unsigned long long drain = st_now() + 1000000000ull;
            volatile int never = 0;
            for (int l = issued > NS ? issued - NS : 0; l < issued; ++l)
                if (l != skipped) st_mbar_wait(&s_full[l % NS], (l / NS) & 1, drain, &never);
        }
    } else if (warp <= P * C) {
        // ---------------------------------------------------------- consumers
        // warp groups of P: group gq takes the CTA's items gq, gq + C, ... (stage
        // l mod S, S a multiple of C); member mp takes the mp-th P-th of each
        // tile's K-steps; members 1..P-1 leave their partial sums in shared memory
        // for member 0 at the group's named barrier (2 + gq, 32 P threads)
        const int cw = warp - 1, gq = cw / P, mp = cw % P;
        const int g = lane >> 2, q = lane & 3;
        const uint32_t pair_bar = 2u + (uint32_t)gq;
        auto pair_sync = [&]() { asm volatile("barrier.sync %0, %1;" ::"r"(pair_bar), "r"(32 * P) : "memory"); };
        int rbuf = 0;         // partials double buffer, flipped per row group
        int hcount = 0;       // kSA: down items of this group so far (the h barrier's phases)
        bool x_seen = !kSA;   // kSA: this warp has observed x in shared memory
        // phase 3: gate/up tiles this CTA completed, per launch expert, published
        // once, when every consumer warp has passed its last gate/up item
        bool published = a.phase != 3;
        auto publish = [&]() {
            // (named barrier 1: every consumer warp; it orders their h writes
            // before the fence of the warp that publishes)
            asm volatile("barrier.sync 1, %0;" ::"r"(32 * P * C) : "memory");
            if (cw == 0) {
                __threadfence();
                for (int e = lane; e < nexp; e += 32)
                    if (meta[e].cnt) atomicAdd(a.done + e, (unsigned)meta[e].cnt);
                if (lane == 0) stamp(2);
            }
            published = true;
        };
        for (int l = gq; l < n_my; l += C) {
            const int s = l % NS, n = l / NS;
            const int gi = (int)blockIdx.x + l * G;
            const StItem it = st_item(gi, a.phase, nexp, nA, nB, iA, iB, a.tpa, a.tpb);
            const bool gate_up = it.gate_up;
            if (!gate_up && !published) publish();
            const ExpMeta m = meta[it.e];
            const bool shared = m.job < 0;
            uint8_t *stage = smem + (size_t)s * a.stage_bytes;
            const uint32_t toff = ts_off(it);
            const int tk = (gq == 0 && mp == 0 && lane == 0) ? (l / C) : 99;  // traced item ordinal
            if (tk < 8) stamp(4 + 3 * tk);
            const bool need_x = kSA && gate_up && !x_seen;
            const bool need_h = kSA && !gate_up;
            // member 0 takes the waits (bounded) and hands the verdict to the
            // other members at the group barrier, so the group breaks or proceeds as one
            if (mp == 0) {
                int ok = 1;
                if (lane == 0) {
                    ok = st_mbar_wait(&s_full[s], n & 1, deadline, &s_stop);
                    if (!ok && !s_stop) st_fail(a, kErrStreamFull, l, s);
                    if (tk < 8) stamp(5 + 3 * tk);
                    if (ok && need_x) {
                        ok = st_mbar_wait(&s_xbar, 0, deadline, &s_stop);
                        if (!ok && !s_stop) st_fail(a, kErrStreamFull, l, -1);
                    }
                    if (ok && !gate_up && a.phase == 3) {  // h: every gate/up tile of this expert
                        unsigned ns_ = 32;
                        for (uint32_t i = 0;; ++i) {
                            if (st_ld_acquire(a.done + it.e) >= (uint32_t)nA) break;
                            if ((i & 7u) == 7u && (s_stop || st_now() > deadline)) {
                                if (!s_stop) st_fail(a, kErrStreamDep, gi, it.e);
                                ok = 0;
                                break;
                            }
                            __nanosleep(ns_);
                            if (ns_ < 512) ns_ <<= 1;
                        }
                        __threadfence();
                    }
                    if (ok && need_h) {
                        // the expert's h rows (complete: the launch before, or the
                        // counts above) into the stage, behind the tensor scales;
                        // the generic-proxy writes of other CTAs are ordered before
                        // this thread's async-proxy reads
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                        const uint32_t hb = 4u * (uint32_t)a.F;
                        st_mbar_expect(&s_hbar[gq], (uint32_t)m.nrows * hb);
                        for (int r = 0; r < m.nrows; ++r) {
                            int tr, p;
                            if (shared) { tr = r; p = a.k; }
                            else { const RowRef rf = rrs[m.row_off + r]; tr = rf.t; p = rf.p; }
                            const size_t sel = (size_t)tr * (a.k + 1) + p;
                            st_bulk_g2s(stage + toff + 16 + (size_t)r * hb, a.hh_out + sel * 2 * a.F, hb, &s_hbar[gq],
                                        evict_first_policy());
                        }
                        ok = st_mbar_wait(&s_hbar[gq], hcount & 1, deadline, &s_stop);
                        if (!ok && !s_stop) st_fail(a, kErrStreamFull, l, -2);
                    }
                    if (!ok) s_stop = 1;
                    s_pair_ok[gq] = ok;
                }
            }
            pair_sync();
            const int ok = s_pair_ok[gq];
            if (!ok) break;
            // every lane observes the completed phases (member 0 saw them complete)
            for (uint32_t i = 0; i < (1u << 20) && !st_mbar_test(&s_full[s], n & 1); ++i) {
            }
            if (need_x) {
                for (uint32_t i = 0; i < (1u << 20) && !st_mbar_test(&s_xbar, 0); ++i) {
                }
                x_seen = true;
            }
            if (need_h) {
                for (uint32_t i = 0; i < (1u << 20) && !st_mbar_test(&s_hbar[gq], hcount & 1); ++i) {
                }
                ++hcount;
            }
            float ts0 = 1.f, ts1 = 1.f, ts2 = 1.f;
            if (!kMx && mp == 0) {  // read before the stage is released
                const float *tsv = reinterpret_cast<const float *>(stage + toff);
                ts0 = tsv[0];
                ts1 = tsv[1];
                ts2 = tsv[2];
            }
            const int K = gate_up ? a.d : a.F;
            const int NCH = K >> 6, nsteps = (NCH + 3) >> 2;
            const int st0 = mp * nsteps / P, st1 = (mp + 1) * nsteps / P;
            const uint32_t cb = gate_up ? cbA : cbB, sb = gate_up ? sbA : sbB;
            const int rA = gate_up ? 2 * g : g, rB = gate_up ? 2 * g + 1 : g + 8;
            const __half *hs = reinterpret_cast<const __half *>(stage + toff + 16);  // kSA: h rows [r][2][F]
            for (int t = 0; t < it.nt; ++t) {
                const int tile = it.tile0 + t;
                const uint8_t *s_codes = stage + (size_t)t * cb;
                const uint8_t *s_scales = stage + (size_t)it.nt * cb + (size_t)t * sb;
                for (int r0 = 0; r0 < m.nrows; r0 += 4 * NG) {
                    // mma column n = g carries activation row r0 + 4*grp + g/2, its
                    // hi (g even) or lo (g odd) fp16 part
                    const __half *col[NG];
                    bool colv[NG];
                    int ngrp = 0;
#pragma unroll
                    for (int grp = 0; grp < NG; ++grp) {
                        const int r = r0 + 4 * grp + (g >> 1);
                        colv[grp] = r < m.nrows;
                        col[grp] = gate_up ? (kSA ? xs : a.act) : (kSA ? hs : a.hh_out);
                        if (r0 + 4 * grp < m.nrows) ngrp = grp + 1;
                        if (colv[grp]) {
                            int tr, p;
                            if (shared) { tr = r; p = a.k; }
                            else { const RowRef rf = rrs[m.row_off + r]; tr = rf.t; p = rf.p; }
                            if (gate_up)
                                col[grp] = (kSA ? xs : a.act) + (size_t)tr * 2 * a.d + (g & 1) * a.d;
                            else if (kSA)
                                col[grp] = hs + (size_t)r * 2 * a.F + (g & 1) * a.F;
                            else
                                col[grp] = a.hh_out + (size_t)(tr * (a.k + 1) + p) * 2 * a.F + (g & 1) * a.F;
                        }
                    }
                    // accumulator sets: chunk half (x step parity with pairs, whose
                    // members run more steps each): short mma dependency chains
                    constexpr int kChains = P >= 3 ? 2 : 4;
                    float acc[kChains][NG][4];
#pragma unroll
                    for (int z = 0; z < kChains; ++z)
#pragma unroll
                        for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                            for (int u = 0; u < 4; ++u) acc[z][grp][u] = 0.f;
                    auto kstep = [&](int st, float(&a0)[NG][4], float(&a1)[NG][4]) {
                        const int c = 4 * st + q;
                        const bool cv = kFull || c < NCH;  // ragged K tail: this lane feeds zeros
                        const int cc = cv ? c : 0;
                        if constexpr (kMx) {
                            const uint32_t sa = cv ? *reinterpret_cast<const uint16_t *>(s_scales + rA * (K >> 5) + 2 * c) : 0u;
                            const uint32_t sbv = cv ? *reinterpret_cast<const uint16_t *>(s_scales + rB * (K >> 5) + 2 * c) : 0u;
                            if (gate_up)
                                step_mma_mx_x2<NG, kActA>(s_codes + rA * (K >> 1) + 32 * cc, s_codes + rB * (K >> 1) + 32 * cc,
                                                          sa, sbv, cc, cv, col, colv, ngrp, a0, a1);
                            else
                                step_mma_mx_x2<NG, kActB>(s_codes + rA * (K >> 1) + 32 * cc, s_codes + rB * (K >> 1) + 32 * cc,
                                                          sa, sbv, cc, cv, col, colv, ngrp, a0, a1);
                        } else {
                            const uint32_t sa = cv ? *reinterpret_cast<const uint32_t *>(s_scales + rA * (K >> 4) + 4 * c) : 0u;
                            const uint32_t sbv = cv ? *reinterpret_cast<const uint32_t *>(s_scales + rB * (K >> 4) + 4 * c) : 0u;
                            if (gate_up)
                                step_mma_x2<NG, kActA>(s_codes + rA * (K >> 1) + 32 * cc, s_codes + rB * (K >> 1) + 32 * cc,
                                                       sa, sbv, cc, cv, col, colv, ngrp, a0, a1);
                            else
                                step_mma_x2<NG, kActB>(s_codes + rA * (K >> 1) + 32 * cc, s_codes + rB * (K >> 1) + 32 * cc,
                                                       sa, sbv, cc, cv, col, colv, ngrp, a0, a1);
                        }
                    };
                    if constexpr (kChains == 4) {
                        for (int st = st0; st < st1; st += 2) {
                            kstep(st, acc[0], acc[1]);
                            if (st + 1 < st1) kstep(st + 1, acc[kChains - 2], acc[kChains - 1]);
                        }
                    } else {
                        for (int st = st0; st < st1; ++st) kstep(st, acc[0], acc[1]);
                    }
                    float d4[NG][4];
#pragma unroll
                    for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            float v = acc[0][grp][u] + acc[1][grp][u];
                            if constexpr (kChains == 4) v += acc[kChains - 2][grp][u] + acc[kChains - 1][grp][u];
                            d4[grp][u] = v;
                        }
                    float *rbase = s_red + (size_t)(gq * 2 + rbuf) * (P - 1) * NG * 128;  // this row group's buffer
                    rbuf ^= 1;
                    if (mp > 0) {
                        float(*rb)[4][32] = reinterpret_cast<float(*)[4][32]>(rbase + (mp - 1) * NG * 128);
#pragma unroll
                        for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                            for (int u = 0; u < 4; ++u) rb[grp][u][lane] = d4[grp][u];
                    }
                    pair_sync();  // the members' partials are in shared memory; all are done with the stage's rows
                    if (tk < 8) stamp(6 + 3 * tk);
                    if (t == it.nt - 1 && r0 + 4 * NG >= m.nrows && mp == 0 && lane == 0)
                        st_mbar_arrive(&s_empty[s]);  // the group's last read of the stage: hand it back
                    if (mp > 0) continue;
                    // member 0: each lane's results -- activation row r0 + 4*grp + q; tile
                    // rows rA (d0, d1), rB (d2, d3)
#pragma unroll
                    for (int grp = 0; grp < NG; ++grp) {
                        for (int j = 1; j < P; ++j) {  // members in order: a fixed summation order
                            const float(*rb)[4][32] = reinterpret_cast<const float(*)[4][32]>(rbase + (j - 1) * NG * 128);
#pragma unroll
                            for (int u = 0; u < 4; ++u) d4[grp][u] += rb[grp][u][lane];
                        }
                        const int r = r0 + 4 * grp + q;
                        if (r >= m.nrows) continue;
                        int tr, p;
                        if (shared) { tr = r; p = a.k; }
                        else { const RowRef rf = rrs[m.row_off + r]; tr = rf.t; p = rf.p; }
                        const float v0 = d4[grp][0] + d4[grp][1];
                        const float v1 = d4[grp][2] + d4[grp][3];
                        const size_t sel = (size_t)tr * (a.k + 1) + p;
                        if (gate_up) {
                            const float gt = kMx ? v0 : ts0 * v0, up = kMx ? v1 : ts1 * v1;
                            const float h = gt / (1.0f + expf(-gt)) * up;
                            const int o = 8 * tile + g;
                            const __half hi = __float2half_rn(h);
                            const __half lo = __float2half_rn(h - __half2float(hi));
                            a.hh_out[sel * 2 * a.F + o] = hi;
                            a.hh_out[sel * 2 * a.F + a.F + o] = lo;
                        } else {
                            const int o = 16 * tile + g;
                            const float sd = kMx ? 1.0f : ts2;
                            a.part_out[sel * a.d + o] = sd * v0;
                            a.part_out[sel * a.d + o + 8] = sd * v1;
                        }
                    }
                }
            }
            if (m.nrows <= 0 && mp == 0 && lane == 0) st_mbar_arrive(&s_empty[s]);  // (an expert without rows)
            if (mp > 0) continue;  // member 0 publishes and combines
            if (gate_up && a.phase == 3 && lane == 0) atomicAdd(&meta[it.e].cnt, it.nt);  // (shared memory)
            if (!gate_up && combine) {
                // the item's tiles whose last expert this is: their rows are combined here.
                // One expert in the launch: every tile (earlier launches completed the rest).
                uint32_t last = it.nt >= 32 ? 0xffffffffu : ((1u << it.nt) - 1u);
                __syncwarp();
                if (nexp > 1) {
                    uint32_t mine = 0u;
                    if (lane == 0) {
                        __threadfence();
                        for (int t = 0; t < it.nt; ++t)
                            if (atomicAdd(&a.tile_ticket[it.tile0 + t], 1u) == (unsigned)(nexp - 1)) mine |= 1u << t;
                    }
                    last = __shfl_sync(0xffffffffu, mine, 0);
                    if (last) __threadfence();
                }
                for (int t = 0; t < it.nt; ++t) {
                    if (!((last >> t) & 1u)) continue;
                    const int tile = it.tile0 + t;
                    for (int i = lane; i < 16 * a.T; i += 32) {
                        const int tr = i >> 4, o = 16 * tile + (i & 15);
                        const float *pr = a.part_out + (size_t)tr * (a.k + 1) * a.d + o;
                        float sum = 0.f;
                        for (int p = 0; p < a.k; ++p)  // (with expert parallelism: the owned experts)
                            if (a.ep_size == 1 || a.idx[tr * a.k + p] % a.ep_size == a.ep_rank)
                                sum = fmaf(a.gates[tr * a.k + p], __ldcg(pr + (size_t)p * a.d), sum);
                        if (a.shared_part) sum += __ldcg(pr + (size_t)a.k * a.d);
                        a.y[(size_t)tr * a.d + o] = sum;
                    }
                    if (nexp > 1 && lane == 0) a.tile_ticket[tile] = 0u;
                }
            }
        }
        // every consumer warp passes the barrier exactly once, on error paths too
        // (a consumer without down items, or one that stopped, arrives here)
        if (!published) publish();
    }

    if (threadIdx.x == 32) stamp(3);  // (warp 1: the first consumer warp)
    __syncthreads();
    if (kSA && (a.phase & 1) && threadIdx.x == 0) {  // no copy outlives the CTA: x has landed
        volatile int never = 0;
        st_mbar_wait(&s_xbar, 0, st_now() + 1000000000ull, &never);
    }
    if (a.phase == 3) {  // the last CTA out resets the launch's gate/up counters
        if (threadIdx.x == 0) {
            __threadfence();
            s_last = atomicAdd(a.exit_ticket, 1u) == gridDim.x - 1;
        }
        __syncthreads();
        if (s_last) {
            __threadfence();
            for (int e = threadIdx.x; e < nexp; e += blockDim.x) a.done[e] = 0u;
            if (threadIdx.x == 0) *a.exit_ticket = 0u;
        }
    }
    if (threadIdx.x == 0) span_mark(a.span, 1);
}

template <int NG, int FMT, int P, bool kFull, bool kSA>
cudaError_t launch_st(const GemvArgs &a, int grid, size_t smem, cudaStream_t s) {
    static bool configured = false;  // per instantiation: allow the large dynamic shared memory
    if (!configured) {
        const cudaError_t e = cudaFuncSetAttribute(expert_stream_kernel<NG, FMT, P, kFull, kSA>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, 210 * 1024);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(32 * (P * a.nc + 1));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, expert_stream_kernel<NG, FMT, P, kFull, kSA>, a);
}

template <int NG, int FMT, int P>
cudaError_t launch_st_fs(const GemvArgs &a, int grid, size_t smem, bool full, bool sa, cudaStream_t s) {
    if (full) return sa ? launch_st<NG, FMT, P, true, true>(a, grid, smem, s) : launch_st<NG, FMT, P, true, false>(a, grid, smem, s);
    return sa ? launch_st<NG, FMT, P, false, true>(a, grid, smem, s) : launch_st<NG, FMT, P, false, false>(a, grid, smem, s);
}

}  // namespace

cudaError_t launch_stream(const GemvArgs &a_in, int max_exp, cudaStream_t s) {
    GemvArgs a = a_in;
    const bool mx = a.lay.fmt == kFmtMxfp4;
    if (!mx && a.lay.fmt != kFmtNvfp4) return cudaErrorInvalidValue;
    if (a.phase < 1 || a.phase > 3 || max_exp < 1 || max_exp > kMaxSlots) return cudaErrorInvalidValue;
    if (a.d % 64 || a.F % 64 || a.d < 64 || a.F < 64 || a.d / 64 > 4 * kMaxSteps || a.F / 64 > 4 * kMaxSteps)
        return cudaErrorInvalidValue;
    if (a.phase == 3 && (a.done == nullptr || a.exit_ticket == nullptr)) return cudaErrorInvalidValue;
    // bulk copies start on 16-byte boundaries: record bases and section offsets
    const uintptr_t al = reinterpret_cast<uintptr_t>(a.arena) | reinterpret_cast<uintptr_t>(a.shared_rec) |
                         (uintptr_t)a.rec_bytes | (uintptr_t)a.lay.w13_codes | (uintptr_t)a.lay.w13_scales |
                         (uintptr_t)a.lay.w2_codes | (uintptr_t)a.lay.w2_scales;
    if (al & 15) return cudaErrorInvalidValue;
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    // activations in shared memory for up to 2 rows: x once per CTA, and a
    // down item's h rows in its stage
    const int ng = a.T <= 4 ? 1 : 2;  // more rows: passes over the staged tile
    const bool sa = a.T <= 2;
    const size_t xbytes = sa ? (size_t)a.T * 4 * a.d : 0, hbytes = sa ? (size_t)a.T * 4 * a.F : 0;
    // stage = the larger item: a tile's codes + scales, 16 bytes of tensor
    // scales, and for a down item its h rows; at least 16 KB; several
    // consecutive tiles of one expert per item where they fit
    const size_t tA = 8 * (size_t)a.d + (mx ? a.d / 2 : a.d), tB = 8 * (size_t)a.F + (mx ? a.F / 2 : a.F);
    size_t sb = tA + 16 > tB + 16 + hbytes ? tA + 16 : tB + 16 + hbytes;
    if (sb < 16 * 1024) sb = 16 * 1024;
    sb = (sb + 127) & ~(size_t)127;
    const int nA = a.F / 8, nB = a.d / 16;
    // items: enough of them that every SM's consumers get a few
    const int64_t want = 3 * (int64_t)sms;
    auto per_item = [&](size_t room, size_t tile_bytes, int tiles_per_exp, int phases_exp) {
        int tp = (int)(room / tile_bytes);
        const int64_t tiles = (int64_t)tiles_per_exp * phases_exp;
        while (tp > 1 && tiles / tp < want) --tp;
        return tp < 1 ? 1 : tp;
    };
    a.tpa = per_item(sb - 16, tA, nA, max_exp);
    a.tpb = per_item(sb - 16 - hbytes, tB, nB, max_exp);
    // (areas rounded to 16 bytes: x is a bulk-copy destination)
    const size_t meta = ((size_t)max_exp * sizeof(ExpMeta) + 15) & ~(size_t)15;
    const size_t rr = (((size_t)a.T * a.k * sizeof(RowRef)) + 15) & ~(size_t)15;
    const size_t budget = 200 * 1024;
    if (meta + rr + xbytes + 2 * sb > budget) return cudaErrorInvalidValue;
    int ns = (int)((budget - meta - rr - xbytes) / sb);
    if (ns > kStMaxStages) ns = kStMaxStages;
    // consumer warp groups: P = 3 warps each for up to 4 activation rows per
    // pass (NG 1), 2 otherwise; a group serves two stages (one loads while the
    // other is computed) where the stages allow, else one.  The stage count is
    // a multiple of the group count, so a stage always serves the same group
    // and its phases are consumed in order (a parity wait can then not see an
    // older phase).
    const int gmax = kStMaxGroups;
    int nc = ns >= 2 * gmax ? gmax : (ns >= 6 ? ns / 2 : (ns < gmax ? ns : gmax));
    a.nc = nc;
    a.ns = ns = (ns >= 2 * nc ? 2 : 1) * nc;
    a.stage_bytes = (uint32_t)sb;
    a.meta_off = (uint32_t)(ns * sb);
    a.rr_off = (uint32_t)(ns * sb + meta);
    a.x_off = (uint32_t)(ns * sb + meta + rr);
    a.exp_cap = max_exp;
    const size_t smem = ns * sb + meta + rr + xbytes;
    const int iA = (nA + a.tpa - 1) / a.tpa, iB = (nB + a.tpb - 1) / a.tpb;
    const int64_t items = (int64_t)max_exp * (((a.phase & 1) ? iA : 0) + ((a.phase & 2) ? iB : 0));
    const int grid = (int)(items < sms ? items : sms);
    const bool full = a.d % 256 == 0 && a.F % 256 == 0;
    if (mx) {
        if (ng == 1) return launch_st_fs<1, kFmtMxfp4, 3>(a, grid, smem, full, sa, s);
        return launch_st_fs<2, kFmtMxfp4, 2>(a, grid, smem, full, false, s);
    }
    if (ng == 1) return launch_st_fs<1, kFmtNvfp4, 3>(a, grid, smem, full, sa, s);
    return launch_st_fs<2, kFmtNvfp4, 2>(a, grid, smem, full, false, s);
}

}  // namespace moe
