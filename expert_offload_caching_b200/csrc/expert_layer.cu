// Persistent decode layer kernel: every expert GEMV of one layer -- gate/up
// with SwiGLU, down, and the gate-weighted combine -- in ONE launch, the hit
// experts (and the shared expert) at once and each missed expert as soon as
// its record lands in HBM.
//
// The FreeToken offload step computes the experts that are resident in GPU
// memory while the missing ones stream in over PCIe (florigen.ai
// "FreeTokenは何をしているのか"; pirouter.ai "32 GB に 65 GB が載る仕組み").  A
// launch per miss puts a kernel launch, a grid ramp and an event wait on the
// critical path of every miss; here the copy stream instead writes a per-miss
// flag after each half of a record (the gate/up prefix, then W2; a stream
// memory write, ordered after the copy), and the CTAs that hold a miss's items
// wait for that flag.
//
// Work items (the same 16-row weight tiles as the per-launch GEMV) form one
// queue in dependency order:
//   hit and shared experts: all gate/up tiles, then all down tiles;
//   then per miss, in the order the host copies them (ascending expert id):
//   its gate/up tiles, then its down tiles.
// CTAs claim items with an atomic counter and stage the next ones while they
// compute the current one (3-deep cp.async ring).  A down tile needs all of its
// expert's gate/up tiles (h): those come earlier in the queue, so they are
// already held by running CTAs, which wait on nothing but copy flags -- the
// smallest unfinished item can always proceed, so the schedule cannot
// deadlock.  Every wait (flag, gate/up completion) is bounded by a time limit;
// when it runs out the CTA records the error in the mapped page and stops,
// and so do the CTAs that then wait on it.  The host can also release all
// waits of a call (an error on its side: the copies will never come).
//
// The combine is as in the per-launch kernel: the CTA that completes the last
// expert of a 16-row output tile (per-tile ticket over all of the layer's
// experts) sums that tile's rows in ascending expert id, plus the shared
// expert.
#include "gemv_inner.cuh"

namespace moe {

namespace {

using namespace gemv;

constexpr int kSharedJob = kMaxSlots - 1;  // done_a slot of the shared expert

// Error codes written to HostPage::error by this kernel.
constexpr int kErrFlagWait = 40;   // a miss's copy flag did not arrive in time
constexpr int kErrDepWait = 41;    // a down tile's gate/up tiles did not complete in time

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned long long now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ void layer_fail(const LayerArgs &a, int code, int item, int job, uint32_t seen) {
    a.page->diag[1] = 30;
    a.page->diag[2] = (int)blockIdx.x;
    a.page->diag[3] = item;
    a.page->diag[4] = job;
    a.page->diag[5] = (int)seen;
    a.page->diag[6] = (int)a.seq;
    __threadfence_system();
    a.page->error = code;
    __threadfence_system();
}

// Thread 0: wait until *p >= want (as a 32-bit sequence), the host releases
// this call, or the deadline passes.  Returns 0 on success, 1 if released, 2
// on timeout.
__device__ int wait_geq(const uint32_t *p, uint32_t want, const LayerArgs &a, unsigned long long deadline) {
    unsigned ns = 32;
    for (uint32_t it = 0;; ++it) {
        if ((int32_t)(ld_acquire(p) - want) >= 0) return 0;
        if ((int32_t)(ld_acquire(a.release) - a.seq) >= 0) return 1;
        if ((it & 15u) == 15u && now_ns() > deadline) return 2;
        __nanosleep(ns);
        if (ns < 1024) ns <<= 1;
    }
}

// One queue entry: the job (index into the job list, kSharedJob for the
// shared expert), the phase, the tile and, for a miss, its ordinal.
struct Item {
    int job, gate_up, tile, miss;
};

// S: tiles in flight per CTA (the shared-memory ring); 2 where 3 would keep
// two CTAs from sharing an SM.
template <int NG, int FMT, int S>
__global__ void __launch_bounds__(kMaxSteps * 32) expert_layer_kernel(LayerArgs a) {
    constexpr int kRing = S + 1;  // claimed-item slots: one more than the tiles in flight
    extern __shared__ __align__(128) uint8_t smem[];
    // the launch's experts: hits (ascending job index, then the shared expert)
    // from the front, misses (ascending) from the back: miss m at kMaxSlots - 1 - m
    __shared__ int s_list[kMaxSlots];
    __shared__ int s_nhit, s_nmiss;
    __shared__ int s_item[kRing], s_def[kRing];
    __shared__ int s_stop, s_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    constexpr bool kMx = FMT == kFmtMxfp4;

    pdl_wait();  // the job list and x come from the route kernel
    const unsigned long long t0 = now_ns();
    if (threadIdx.x == 0) {
        span_mark(a.span, 0);
        span_mark(a.span_hit, 0);
        s_stop = 0;
    }
    pdl_launch_dependents();
    const unsigned long long deadline = t0 + a.wait_ns;

    // ---- hit list (ascending job index, then the shared expert) and miss list
    if (warp == 0) {
        const int nj = __ldcg(a.n_jobs);
        int nh = 0, nm = 0;
        for (int b = 0; b < nj; b += 32) {
            const int j = b + lane;
            const bool valid = j < nj;
            const bool hit = valid && __ldcg(&a.jobs[j].hit);
            const unsigned hb = __ballot_sync(0xffffffffu, hit);
            const unsigned mb = __ballot_sync(0xffffffffu, valid && !hit);
            const unsigned lt = (1u << lane) - 1u;
            if (hit) s_list[nh + __popc(hb & lt)] = j;
            else if (valid) s_list[kMaxSlots - 1 - (nm + __popc(mb & lt))] = j;
            nh += __popc(hb);
            nm += __popc(mb);
        }
        if (lane == 0) {
            if (a.shared_item) s_list[nh++] = kSharedJob;
            s_nhit = nh;
            s_nmiss = nm;
        }
    }
    __syncthreads();
    const int H = s_nhit, M = s_nmiss;
    const int nA = a.F >> 3, nB = a.d >> 4, per = nA + nB;
    if (H + M == 0 && blockIdx.x == 0) {
        // a shard of an expert-parallel layer that owns none of the selected
        // experts (and no resident shared expert): its partial output is the
        // shared expert's (computed by earlier launches) or zero
        for (int e = threadIdx.x; e < a.T * a.d; e += blockDim.x) {
            const int t = e / a.d, o = e - t * a.d;
            a.y[e] = a.shared_rec ? __ldcg(a.part + ((size_t)t * (a.k + 1) + a.k) * a.d + o) : 0.f;
        }
    }
    const int total = (H + M) * per, hit_items = H * per;
    auto decode = [&](int i) -> Item {
        Item it;
        if (i < H * nA) { it.job = s_list[i / nA]; it.gate_up = 1; it.tile = i % nA; it.miss = -1; }
        else if (i < hit_items) {
            const int j = i - H * nA;
            it.job = s_list[j / nB]; it.gate_up = 0; it.tile = j % nB; it.miss = -1;
        } else {
            const int j = i - hit_items, m = j / per, r = j - m * per;
            it.job = s_list[kMaxSlots - 1 - m]; it.miss = m;
            it.gate_up = r < nA;
            it.tile = r < nA ? r : r - nA;
        }
        return it;
    };
    auto record = [&](int job) -> const uint8_t * {
        return job == kSharedJob ? a.shared_rec : a.arena + (int64_t)__ldcg(&a.jobs[job].slot) * a.rec_bytes;
    };
    auto flag_of = [&](const Item &it) -> const uint32_t * {  // null: resident, nothing to wait for
        return it.miss < 0 ? nullptr : a.miss_flag + 2 * it.job + (it.gate_up ? 0 : 1);
    };

    // shared-memory ring, sized for the longer of the two K (d for gate/up, F for down)
    const int Kmax = a.d > a.F ? a.d : a.F;
    const uint32_t buf_bytes = 16u * (uint32_t)(Kmax >> 1) + (kMx ? (uint32_t)(Kmax >> 1) : (uint32_t)Kmax);
    const int nwarps = (int)(blockDim.x >> 5);
    float(*red)[NG][4][32] = reinterpret_cast<float(*)[NG][4][32]>(smem + S * buf_bytes);

    // issue the copies of the j-th claimed item into buffer j % S (no commit);
    // weights are read once per layer: evict-first in L2
    const uint64_t ef = evict_first_policy();
    auto issue = [&](int i, int j) {
        const Item it = decode(i);
        const int K = it.gate_up ? a.d : a.F;
        const uint32_t code_bytes = 16u * (uint32_t)(K >> 1), scale_bytes = kMx ? (uint32_t)(K >> 1) : (uint32_t)K;
        const uint8_t *rec = record(it.job);
        uint8_t *dst = smem + (j % S) * buf_bytes;
        const uint8_t *codes = rec + (it.gate_up ? a.lay.w13_codes : a.lay.w2_codes) + (int64_t)it.tile * code_bytes;
        const uint8_t *scales = rec + (it.gate_up ? a.lay.w13_scales : a.lay.w2_scales) + (int64_t)it.tile * scale_bytes;
        for (uint32_t o = threadIdx.x; o < (code_bytes >> 4); o += blockDim.x)
            cp_async16_ef(dst + 16 * o, codes + 16 * o, ef);
        for (uint32_t o = threadIdx.x; o < (scale_bytes >> 4); o += blockDim.x)
            cp_async16_ef(dst + code_bytes + 16 * o, scales + 16 * o, ef);
        if (it.gate_up && it.miss < 0) {  // a resident expert's down projection -> L2 (a 1/nA slice)
            const uint32_t tot = (uint32_t)(a.lay.bytes - a.lay.w2_codes);
            const uint32_t sl = ((tot / nA) + 127u) & ~127u;
            const uint32_t off = sl * it.tile;
            if (off < tot) prefetch_l2_range(rec + a.lay.w2_codes + off, sl < tot - off ? sl : tot - off);
        }
    };
    // claim (thread 0): the next queue item into ring slot j % kRing, and
    // whether its record is already resident (else its copies wait for compute time)
    auto claim = [&](int j) {
        const int i = (int)atomicAdd(a.queue, 1u);
        s_item[j % kRing] = i;
        int def = 0;
        if (i < total) {
            const uint32_t *f = flag_of(decode(i));
            def = f != nullptr && (int32_t)(ld_acquire(f) - a.seq) < 0;
        }
        s_def[j % kRing] = def;
    };
    auto stage = [&](int j) {  // all threads; always one commit group
        const int i = s_item[j % kRing];
        if (i < total && !s_def[j % kRing]) issue(i, j);
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    if (threadIdx.x == 0)
        for (int j = 0; j < S - 1; ++j) claim(j);
    __syncthreads();
    for (int j = 0; j < S - 1; ++j) stage(j);

    int rr = 0;
    for (int j = 0;; ++j) {
        asm volatile("cp.async.wait_group %0;" ::"n"(S - 2) : "memory");
        if (threadIdx.x == 0) claim(j + S - 1);
        __syncthreads();  // item j landed for every thread; every thread is done with item j - 1
        const int i = s_item[j % kRing];
        if (i >= total || s_stop) break;
        stage(j + S - 1);
        const Item it = decode(i);
        // a miss whose record had not landed at claim time: wait for its flag now
        if (s_def[j % kRing]) {
            if (threadIdx.x == 0) {
                const int w = wait_geq(flag_of(it), a.seq, a, deadline);
                if (w == 2) layer_fail(a, kErrFlagWait, i, it.job, ld_acquire(flag_of(it)));
                if (w) s_stop = 1;
                __threadfence();
            }
            __syncthreads();
            if (s_stop) break;
            issue(i, j);
            asm volatile("cp.async.commit_group;" ::: "memory");
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            __syncthreads();
        }
        // a down tile reads h: wait until the expert's gate/up tiles are done
        if (!it.gate_up) {
            if (threadIdx.x == 0) {
                const int w = wait_geq(a.done_a + it.job, (uint32_t)nA, a, deadline);
                if (w == 2) layer_fail(a, kErrDepWait, i, it.job, ld_acquire(a.done_a + it.job));
                if (w) s_stop = 1;
                __threadfence();
            }
            __syncthreads();
            if (s_stop) break;
        }

        const bool gate_up = it.gate_up, shared = it.job == kSharedJob;
        const int K = gate_up ? a.d : a.F;
        const int NCH = K >> 6, nsteps = (NCH + 3) >> 2, spw = (nsteps + nwarps - 1) / nwarps;
        const uint32_t code_bytes = 16u * (uint32_t)(K >> 1);
        const uint8_t *rec = record(it.job);
        const int nrows = shared ? a.T : __ldcg(&a.jobs[it.job].nrows);
        const int row_off = shared ? 0 : __ldcg(&a.jobs[it.job].row_off);
        const uint8_t *s_codes = smem + (j % S) * buf_bytes, *s_scales = s_codes + code_bytes;
        const float *ts = kMx ? nullptr : reinterpret_cast<const float *>(rec + a.lay.tscales);
        const int rA = gate_up ? 2 * g : g, rB = gate_up ? 2 * g + 1 : g + 8;
        const __half *act = gate_up ? a.xh : a.hh;
        for (int r0 = 0; r0 < nrows; r0 += 4 * NG) {
            const __half *col[NG];
            bool colv[NG];
            int ngrp = 0;
#pragma unroll
            for (int grp = 0; grp < NG; ++grp) {
                const int r = r0 + 4 * grp + (g >> 1);
                colv[grp] = r < nrows;
                col[grp] = act;
                if (r0 + 4 * grp < nrows) ngrp = grp + 1;
                if (colv[grp]) {
                    int t, p;
                    if (shared) { t = r; p = a.k; }
                    else { const RowRef rf = a.rowrefs[row_off + r]; t = rf.t; p = rf.p; }
                    col[grp] = gate_up ? act + (size_t)t * 2 * a.d + (g & 1) * a.d
                                       : act + (size_t)(t * (a.k + 1) + p) * 2 * a.F + (g & 1) * a.F;
                }
            }
            float acc[NG][4];
#pragma unroll
            for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                for (int u = 0; u < 4; ++u) acc[grp][u] = 0.f;
            for (int st = 0; st < spw; ++st) {
                const int c = 4 * (warp * spw + st) + q;
                const bool cv = c < NCH;
                const int cc = cv ? c : 0;
                if constexpr (kMx) {
                    const uint32_t sa = cv ? *reinterpret_cast<const uint16_t *>(s_scales + rA * (K >> 5) + 2 * c) : 0u;
                    const uint32_t sb = cv ? *reinterpret_cast<const uint16_t *>(s_scales + rB * (K >> 5) + 2 * c) : 0u;
                    if (gate_up)
                        step_mma_mx<NG, false>(s_codes + rA * (K >> 1) + 32 * cc, s_codes + rB * (K >> 1) + 32 * cc, sa,
                                               sb, cc, cv, col, colv, ngrp, acc);
                    else
                        step_mma_mx<NG, true>(s_codes + rA * (K >> 1) + 32 * cc, s_codes + rB * (K >> 1) + 32 * cc, sa,
                                              sb, cc, cv, col, colv, ngrp, acc);
                } else {
                    const uint32_t sa = cv ? *reinterpret_cast<const uint32_t *>(s_scales + rA * (K >> 4) + 4 * c) : 0u;
                    const uint32_t sb = cv ? *reinterpret_cast<const uint32_t *>(s_scales + rB * (K >> 4) + 4 * c) : 0u;
                    if (gate_up)
                        step_mma<NG, false>(s_codes + rA * (K >> 1) + 32 * cc, s_codes + rB * (K >> 1) + 32 * cc, sa, sb,
                                            cc, cv, col, colv, ngrp, acc);
                    else
                        step_mma<NG, true>(s_codes + rA * (K >> 1) + 32 * cc, s_codes + rB * (K >> 1) + 32 * cc, sa, sb,
                                           cc, cv, col, colv, ngrp, acc);
                }
            }
            float(*rb)[NG][4][32] = red + (rr & 1) * nwarps;
            ++rr;
#pragma unroll
            for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                for (int u = 0; u < 4; ++u) rb[warp][grp][u][lane] = acc[grp][u];
            __syncthreads();
            if (warp == 0) {
                for (int w = 1; w < nwarps; ++w)
#pragma unroll
                    for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                        for (int u = 0; u < 4; ++u) acc[grp][u] += rb[w][grp][u][lane];
#pragma unroll
                for (int grp = 0; grp < NG; ++grp) {
                    const int r = r0 + 4 * grp + q;
                    if (r >= nrows) continue;
                    int t, p;
                    if (shared) { t = r; p = a.k; }
                    else { const RowRef rf = a.rowrefs[row_off + r]; t = rf.t; p = rf.p; }
                    const float v0 = acc[grp][0] + acc[grp][1];
                    const float v1 = acc[grp][2] + acc[grp][3];
                    const size_t sel = (size_t)t * (a.k + 1) + p;
                    if (gate_up) {
                        const float gt = kMx ? v0 : ts[0] * v0, up = kMx ? v1 : ts[1] * v1;
                        const float h = gt / (1.0f + expf(-gt)) * up;
                        const int o = 8 * it.tile + g;
                        const __half hi = __float2half_rn(h);
                        const __half lo = __float2half_rn(h - __half2float(hi));
                        a.hh[sel * 2 * a.F + o] = hi;
                        a.hh[sel * 2 * a.F + a.F + o] = lo;
                    } else {
                        const int o = 16 * it.tile + g;
                        const float sd = kMx ? 1.0f : ts[2];
                        a.part[sel * a.d + o] = sd * v0;
                        a.part[sel * a.d + o + 8] = sd * v1;
                    }
                }
            }
        }
        __syncthreads();  // warp 0's outputs of this item are written
        if (gate_up) {
            if (threadIdx.x == 0) {
                __threadfence();
                atomicAdd(a.done_a + it.job, 1u);
            }
        } else {  // the tile's last expert combines its rows
            if (threadIdx.x == 0) {
                __threadfence();
                s_last = atomicAdd(&a.tile_ticket[it.tile], 1u) == (unsigned)(H + M - 1);
            }
            __syncthreads();
            if (s_last) {
                __threadfence();
                for (int e = threadIdx.x; e < 16 * a.T; e += blockDim.x) {
                    const int t = e >> 4, o = 16 * it.tile + (e & 15);
                    const float *pr = a.part + (size_t)t * (a.k + 1) * a.d + o;
                    float sum = 0.f;
                    for (int p = 0; p < a.k; ++p)  // (with expert parallelism: the owned experts)
                        if (a.ep_size == 1 || a.idx[t * a.k + p] % a.ep_size == a.ep_rank)
                            sum = fmaf(a.gates[t * a.k + p], __ldcg(pr + (size_t)p * a.d), sum);
                    if (a.shared_rec) sum += __ldcg(pr + (size_t)a.k * a.d);
                    a.y[(size_t)t * a.d + o] = sum;
                }
                if (threadIdx.x == 0) a.tile_ticket[it.tile] = 0u;
            }
        }
        if (threadIdx.x == 0 && i < hit_items) span_mark(a.span_hit, 1);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");  // no copy outlives the CTA
    // the last CTA out resets the launch's counters for the next layer
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = atomicAdd(a.queue + 1, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (s_last) {
        __threadfence();
        for (int j = threadIdx.x; j < kMaxSlots; j += blockDim.x) a.done_a[j] = 0u;
        for (int t = threadIdx.x; t < nB; t += blockDim.x) a.tile_ticket[t] = 0u;  // after a stop, too
        if (threadIdx.x == 0) {
            a.queue[0] = 0u;
            a.queue[1] = 0u;
        }
    }
    if (threadIdx.x == 0) span_mark(a.span, 1);
}

template <int NG, int FMT, int S>
cudaError_t launch_layer_ng(const LayerArgs &a, int threads, size_t smem, cudaStream_t st) {
    static bool configured = false;
    static int sms = 0;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(expert_layer_kernel<NG, FMT, S>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return e;
        int dev = 0;
        e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, expert_layer_kernel<NG, FMT, S>, threads,
                                                                  smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    if (per_sm > 4) per_sm = 4;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms * per_sm);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, expert_layer_kernel<NG, FMT, S>, a);
}

template <int NG, int FMT>
cudaError_t launch_layer_fmt(const LayerArgs &a, int threads, size_t buf, size_t red, cudaStream_t st) {
    // 3 tiles in flight unless that keeps a second CTA off the SM (227 KB of
    // shared memory per SM, of which ~5 KB static per CTA)
    const size_t smem3 = 3 * buf + red;
    if (2 * (smem3 + 6 * 1024) <= 227 * 1024) return launch_layer_ng<NG, FMT, 3>(a, threads, smem3, st);
    return launch_layer_ng<NG, FMT, 2>(a, threads, 2 * buf + red, st);
}

}  // namespace

cudaError_t launch_expert_layer(const LayerArgs &a, cudaStream_t s) {
    const int Kmax = a.d > a.F ? a.d : a.F;
    const int nsteps = (Kmax / 64 + 3) / 4;
    if (nsteps < 1 || nsteps > kMaxSteps || a.F / 8 > kMaxTiles || a.d / 16 > kMaxTiles) return cudaErrorInvalidValue;
    const int spw = nsteps >= 8 ? 2 : 1;
    const int warps = (nsteps + spw - 1) / spw;
    const int ng = a.T <= 4 ? 1 : 2;
    const bool mx = a.lay.fmt == kFmtMxfp4;
    if (!mx && a.lay.fmt != kFmtNvfp4) return cudaErrorInvalidValue;
    const size_t buf = 16 * (size_t)(Kmax / 2) + (size_t)(mx ? Kmax / 2 : Kmax);
    const size_t red = 2 * (size_t)warps * ng * 4 * 32 * sizeof(float);
    if (2 * buf + red > 200 * 1024) return cudaErrorInvalidValue;
    const int threads = warps * 32;
    if (mx) {
        if (ng == 1) return launch_layer_fmt<1, kFmtMxfp4>(a, threads, buf, red, s);
        return launch_layer_fmt<2, kFmtMxfp4>(a, threads, buf, red, s);
    }
    if (ng == 1) return launch_layer_fmt<1, kFmtNvfp4>(a, threads, buf, red, s);
    return launch_layer_fmt<2, kFmtNvfp4>(a, threads, buf, red, s);
}

}  // namespace moe
