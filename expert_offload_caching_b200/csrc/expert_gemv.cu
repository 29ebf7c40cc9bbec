// NVFP4 expert GEMV for decode (W4A16): gate/up projection with fused SwiGLU,
// down projection, and the gate-weighted combine.
//
// The routed expert is a SwiGLU FFN over NVFP4 weights (FreeToken pages: routed
// expert MLPs in NVFP4, florigen.ai "NVFP4で約135GBまで縮める"): w = e2m1 * e4m3
// block scale (one per 16 consecutive K) * fp32 tensor scale.
//   h_j = silu(g_j) * u_j,  g = W1 x, u = W3 x;   y_e = W2 h.
//   y = sum over selected e (ascending id) of gate_e * y_e + y_shared.
//
// Decode is HBM-bound (a few rows, weights read once) and latency-bound when
// one expert is processed alone.  So:
//   * a persistent grid walks the launch's (expert, 16-row weight tile) items;
//     a tile's rows are contiguous in the record, so a CTA stages whole tiles
//     into a 3-deep ring of shared-memory buffers with 16-byte asynchronous
//     copies (cp.async.cg, L1 bypassed), the next two tiles in flight while it
//     computes the current one.  No registers hold data in flight;
//   * the warps split the tile's K-steps of 256 elements;
//   * E2M1 codes are decoded in registers with cvt.rn.f16x2.e2m1x2 (2 per op),
//     then multiplied by the E4M3 block scale (cvt.rn.f16x2.e4m3x2); the
//     product of an E2M1 and an E4M3 value is exact in fp16;
//   * the dot products run on the tensor cores (mma.sync m16n8k16, fp16 in,
//     fp32 accumulate): the 8 mma columns carry up to 4 activation rows as fp16
//     (hi, lo) pairs, hi + lo == the fp32 (or bf16) value, so nothing is lost
//     against fp32 FMAs.  The dot product is order-free: the mma's logical k
//     positions are mapped onto each thread's own 64-element chunk, and the
//     activations are loaded at the same positions;
//   * MXFP4 records (E8M0 scale 2^(c-127) per 32 elements, no tensor scale):
//     the scale spans far more than fp16 does, so per K-step and row the
//     quad's largest scale code c_max is factored out: the mma sees
//     e2m1 * 2^(c - c_max + 12) (exact in fp16 while c >= c_max - 35; the
//     +12 keeps those weights normal and below 6 * 2^12), and the step's
//     fp32 result is multiplied by 2^(c_max - 139) before it is accumulated;
//   * K-split partial sums are reduced in shared memory in a fixed order;
//   * the gate/up launch prefetches the expert's down-projection bytes into
//     L2 (prefetch.global.L2), so the down launch reads L2;
//   * the last down launch of a layer also does the combine, per 16-row tile:
//     the tile's last CTA (threadfence + per-tile ticket, no waiting) sums its
//     rows' partials in ascending id.
#include "gemv_inner.cuh"

namespace moe {

namespace {

using namespace gemv;

// Persistent schedule: the launch's work items are (expert, 16-row weight
// tile) pairs -- the valid experts of the launch in ascending id (hit jobs, or
// the one job only_job), then the shared expert -- numbered expert-major; CTA b
// takes items b, b + G, b + 2G, ... (G = gridDim.x, a few CTAs per SM).  Each
// CTA streams its items through a kGStages-deep ring of shared-memory buffers
// (16-byte cp.async copies of the whole tile, one group per item), so the
// loads of the next items are in flight while it computes the current one.
// Each warp owns spw consecutive K-steps of 256 elements; warp 0 sums the
// warps' partials in a fixed order.  Dynamic shared memory: kGStages x (16*K/2
// code bytes + K scale bytes) + two buffers of partials (warps x NG x 512
// bytes each), used in turn, so two barriers per item suffice.
//
// Launched with programmatic stream serialization: gate/up waits for the
// route kernel before reading anything (job list, activations); the down
// projection reads the job list (complete, two launches back), stages its
// first W2 tiles, and only then waits for gate/up's h.  Every CTA executes the
// wait, so a launch completes only after its predecessor.
//
// Combine (down launches with a.combine): the CTA that completes the last
// expert of a tile (per-tile ticket counting the launch's experts) sums that
// tile's 16 output rows over the layer's experts in ascending id, plus the
// shared expert, for every row t.
template <int NG, int FMT>
__global__ void __launch_bounds__(kMaxSteps * 32) expert_gemv_kernel(GemvArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_valid[kMaxSlots];  // job index per valid expert, -1: the shared expert
    __shared__ int s_nvalid, s_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const bool gate_up = a.mode == kGateUp;

    if (gate_up) {
        pdl_wait();  // job list and x come from the previous launch
        if (threadIdx.x == 0) span_mark(a.span, 0);
    }
    pdl_launch_dependents();

    // ---- the launch's valid experts.  L2 reads (ld.global.cg): the down launch
    // reads the job list before its PDL wait, and an SM's L1 may still hold
    // lines of an older launch.
    if (warp == 0) {
        int cnt = 0;
        if (a.only_job >= 0) {
            if (lane == 0) s_valid[0] = a.only_job;
            cnt = 1;
        } else {
            const int nj = __ldcg(a.n_jobs);
            for (int b = 0; b < a.slots; b += 32) {
                const int slot = b + lane;
                int v = -2;
                if (slot < a.slots) {
                    if (slot == a.shared_slot) v = -1;
                    else if (slot < nj && __ldcg(&a.jobs[slot].hit)) v = slot;
                }
                const unsigned ball = __ballot_sync(0xffffffffu, v != -2);
                if (v != -2) s_valid[cnt + __popc(ball & ((1u << lane) - 1u))] = v;
                cnt += __popc(ball);
            }
        }
        if (lane == 0) s_nvalid = cnt;
    }
    __syncthreads();
    const int nvalid = s_nvalid;

    const int K = gate_up ? a.d : a.F;
    const int tiles = gate_up ? (a.F >> 3) : (a.d >> 4);
    const int nitems = nvalid * tiles;
    const int G = (int)gridDim.x;
    const int n_my = (int)blockIdx.x < nitems ? (nitems - 1 - (int)blockIdx.x) / G + 1 : 0;
    const int NCH = K >> 6;
    const int nwarps = (int)(blockDim.x >> 5);
    const int nsteps = (NCH + 3) >> 2;
    const int spw = (nsteps + nwarps - 1) / nwarps;
    constexpr bool kMx = FMT == kFmtMxfp4;
    const uint32_t code_bytes = 16u * (uint32_t)(K >> 1), scale_bytes = kMx ? (uint32_t)(K >> 1) : (uint32_t)K;
    const uint32_t buf_bytes = code_bytes + scale_bytes;
    float(*red)[NG][4][32] = reinterpret_cast<float(*)[NG][4][32]>(smem + kGStages * buf_bytes);

    auto record = [&](int jid) -> const uint8_t * {
        return jid < 0 ? a.shared_rec : a.arena + (int64_t)__ldcg(&a.jobs[jid].slot) * a.rec_bytes;
    };
    // stage this CTA's j-th item into buffer j % kGStages; always one cp.async group
    auto stage = [&](int j) {
        if (j < n_my) {
            const int item = (int)blockIdx.x + j * G;
            const int jid = s_valid[item / tiles], tile = item - (item / tiles) * tiles;
            const uint8_t *rec = record(jid);
            uint8_t *dst = smem + (j % kGStages) * buf_bytes;
            const uint8_t *codes = rec + (gate_up ? a.lay.w13_codes : a.lay.w2_codes) + (int64_t)tile * code_bytes;
            const uint8_t *scales =
                rec + (gate_up ? a.lay.w13_scales : a.lay.w2_scales) + (int64_t)tile * scale_bytes;
            for (uint32_t o = threadIdx.x; o < (code_bytes >> 4); o += blockDim.x)
                cp_async16(dst + 16 * o, codes + 16 * o);
            for (uint32_t o = threadIdx.x; o < (scale_bytes >> 4); o += blockDim.x)
                cp_async16(dst + code_bytes + 16 * o, scales + 16 * o);
            if (gate_up) {  // this expert's down projection -> L2 for the down launch (a 1/tiles slice)
                const uint32_t total = (uint32_t)(a.lay.bytes - a.lay.w2_codes);
                const uint32_t per = ((total / tiles) + 127u) & ~127u;
                const uint32_t off = per * tile;
                if (off < total)
                    prefetch_l2_range(rec + a.lay.w2_codes + off, per < total - off ? per : total - off);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    for (int j = 0; j < kGStages - 1; ++j) stage(j);
    if (!gate_up) {
        pdl_wait();  // h comes from the gate/up launch; W2 tiles already in flight
        if (threadIdx.x == 0) span_mark(a.span, 0);
    }
    // tile-local rows of this thread: gate_up 2g (gate) / 2g+1 (up); down g / g+8
    const int rA = gate_up ? 2 * g : g, rB = gate_up ? 2 * g + 1 : g + 8;
    int rr = 0;  // row-group counter: the partials buffer alternates, so warp 0's
                 // epilogue of one group overlaps the other warps' next group
    for (int j = 0; j < n_my; ++j) {
        asm volatile("cp.async.wait_group %0;" ::"n"(kGStages - 2) : "memory");  // item j landed
        __syncthreads();  // ... for every thread; and every thread is done with item j - 1
        stage(j + kGStages - 1);  // into item j - 1's buffer
        const int item = (int)blockIdx.x + j * G;
        const int jid = s_valid[item / tiles], tile = item - (item / tiles) * tiles;
        const bool shared = jid < 0;
        const uint8_t *rec = record(jid);
        const int nrows = shared ? a.T : __ldcg(&a.jobs[jid].nrows);
        const int row_off = shared ? 0 : __ldcg(&a.jobs[jid].row_off);
        const uint8_t *s_codes = smem + (j % kGStages) * buf_bytes, *s_scales = s_codes + code_bytes;
        // tensor scales (gate, up, down): NVFP4 only
        const float *ts = kMx ? nullptr : reinterpret_cast<const float *>(rec + a.lay.tscales);
        for (int r0 = 0; r0 < nrows; r0 += 4 * NG) {
            // mma column n = g carries activation row r0 + 4*grp + g/2, the hi (g
            // even) or lo (g odd) fp16 part.
            const __half *col[NG];
            bool colv[NG];
            int ngrp = 0;
#pragma unroll
            for (int grp = 0; grp < NG; ++grp) {
                const int r = r0 + 4 * grp + (g >> 1);
                colv[grp] = r < nrows;
                col[grp] = a.act;
                if (r0 + 4 * grp < nrows) ngrp = grp + 1;
                if (colv[grp]) {
                    int t, p;
                    if (shared) { t = r; p = a.k; }
                    else { const RowRef rr = a.rowrefs[row_off + r]; t = rr.t; p = rr.p; }
                    col[grp] = gate_up ? a.act + (size_t)t * 2 * a.d + (g & 1) * a.d
                                       : a.act + (size_t)(t * (a.k + 1) + p) * 2 * a.F + (g & 1) * a.F;
                }
            }
            float acc[NG][4];
#pragma unroll
            for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[grp][i] = 0.f;
            for (int st = 0; st < spw; ++st) {  // this warp's K-steps (uniform across the warp)
                const int c = 4 * (warp * spw + st) + q;
                const bool cv = c < NCH;  // ragged K tail: some lanes of the quad feed zeros
                const int cc = cv ? c : 0;
                if constexpr (kMx) {  // two E8M0 codes per row and chunk
                    const uint32_t sa = cv ? *reinterpret_cast<const uint16_t *>(s_scales + rA * (K >> 5) + 2 * c) : 0u;
                    const uint32_t sb = cv ? *reinterpret_cast<const uint16_t *>(s_scales + rB * (K >> 5) + 2 * c) : 0u;
                    step_mma_mx<NG>(s_codes + rA * (K >> 1) + 32 * cc, s_codes + rB * (K >> 1) + 32 * cc, sa, sb, cc,
                                    cv, col, colv, ngrp, acc);
                } else {
                    const uint32_t sa = cv ? *reinterpret_cast<const uint32_t *>(s_scales + rA * (K >> 4) + 4 * c) : 0u;
                    const uint32_t sb = cv ? *reinterpret_cast<const uint32_t *>(s_scales + rB * (K >> 4) + 4 * c) : 0u;
                    step_mma<NG>(s_codes + rA * (K >> 1) + 32 * cc, s_codes + rB * (K >> 1) + 32 * cc, sa, sb, cc,
                                 cv, col, colv, ngrp, acc);
                }
            }
            // ---- reduce the warps' partial sums (fixed order), then the epilogue
            float(*rb)[NG][4][32] = red + (rr & 1) * nwarps;
            ++rr;
#pragma unroll
            for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                for (int i = 0; i < 4; ++i) rb[warp][grp][i][lane] = acc[grp][i];
            __syncthreads();
            if (warp == 0) {
                for (int w = 1; w < nwarps; ++w)
#pragma unroll
                    for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                        for (int i = 0; i < 4; ++i) acc[grp][i] += rb[w][grp][i][lane];
#pragma unroll
                for (int grp = 0; grp < NG; ++grp) {
                    const int r = r0 + 4 * grp + q;  // this thread's results: activation row q
                    if (r >= nrows) continue;
                    int t, p;
                    if (shared) { t = r; p = a.k; }
                    else { const RowRef rr = a.rowrefs[row_off + r]; t = rr.t; p = rr.p; }
                    const float v0 = acc[grp][0] + acc[grp][1];  // tile row rA
                    const float v1 = acc[grp][2] + acc[grp][3];  // tile row rB
                    const size_t sel = (size_t)t * (a.k + 1) + p;
                    if (gate_up) {
                        const float gt = kMx ? v0 : ts[0] * v0, up = kMx ? v1 : ts[1] * v1;
                        const float h = gt / (1.0f + expf(-gt)) * up;
                        const int o = 8 * tile + g;
                        const __half hi = __float2half_rn(h);
                        const __half lo = __float2half_rn(h - __half2float(hi));
                        a.hh_out[sel * 2 * a.F + o] = hi;
                        a.hh_out[sel * 2 * a.F + a.F + o] = lo;
                    } else {
                        const int o = 16 * tile + g;
                        const float sd = kMx ? 1.0f : ts[2];
                        a.part_out[sel * a.d + o] = sd * v0;
                        a.part_out[sel * a.d + o + 8] = sd * v1;
                    }
                }
            }
        }

        if (a.combine && !gate_up) {  // the tile's last expert: combine its rows
            __syncthreads();  // warp 0's partials of this item are written
            if (threadIdx.x == 0) {
                __threadfence();
                s_last = atomicAdd(&a.tile_ticket[tile], 1u) == (unsigned)(nvalid - 1);
            }
            __syncthreads();
            if (s_last) {
                __threadfence();
                if (a.combine == 1 || __ldcg(a.n_misses) == 0) {
                    for (int e = threadIdx.x; e < 16 * a.T; e += blockDim.x) {
                        const int t = e >> 4, o = 16 * tile + (e & 15);
                        const float *pr = a.part_out + (size_t)t * (a.k + 1) * a.d + o;
                        float sum = 0.f;
                        for (int p = 0; p < a.k; ++p)
                            if (a.ep_size == 1 || a.idx[t * a.k + p] % a.ep_size == a.ep_rank)
                                sum = fmaf(a.gates[t * a.k + p], __ldcg(pr + (size_t)p * a.d), sum);
                        if (a.shared_rec) sum += __ldcg(pr + (size_t)a.k * a.d);
                        a.y[(size_t)t * a.d + o] = sum;
                    }
                }
                if (threadIdx.x == 0) a.tile_ticket[tile] = 0u;
            }
            __syncthreads();
        }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");  // no copy outlives the CTA
    if (a.span) {
        __syncthreads();
        if (threadIdx.x == 0) span_mark(a.span, 1);
    }
}

template <int NG, int FMT>
cudaError_t launch_ng(const GemvArgs &a, int tiles, int threads, size_t smem, cudaStream_t s) {
    static bool configured = false;  // per instantiation: allow > 48 KB of dynamic smem
    static int sms = 0;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(expert_gemv_kernel<NG, FMT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
        if (e != cudaSuccess) return e;
        int dev = 0;
        e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    // persistent grid: as many CTAs as fit at once (at most 4 per SM), no more than the items
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, expert_gemv_kernel<NG, FMT>, threads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    if (per_sm > 4) per_sm = 4;
    int grid = sms * per_sm;
    if (grid > a.slots * tiles) grid = a.slots * tiles;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, expert_gemv_kernel<NG, FMT>, a);
}

}  // namespace

cudaError_t launch_gemv(const GemvArgs &a_in, int slots, cudaStream_t s) {
    GemvArgs a = a_in;
    const int K = a.mode == kGateUp ? a.d : a.F;
    const int tiles = a.mode == kGateUp ? a.F / 8 : a.d / 16;
    const int nsteps = (K / 64 + 3) / 4;
    if (nsteps < 1 || nsteps > kMaxSteps || slots < 1 || slots > kMaxSlots || tiles > kMaxTiles)
        return cudaErrorInvalidValue;
    a.slots = a.only_job >= 0 ? 1 : slots;
    const int spw = nsteps >= 8 ? 2 : 1;  // 2 K-steps per warp for long rows: smaller CTAs, more per SM
    const int warps = (nsteps + spw - 1) / spw;
    const int ng = a.T <= 4 ? 1 : 2;  // more rows: passes over the staged tile
    const bool mx = a.lay.fmt == kFmtMxfp4;
    if (!mx && a.lay.fmt != kFmtNvfp4) return cudaErrorInvalidValue;
    const size_t buf = 16 * (size_t)(K / 2) + (size_t)(mx ? K / 2 : K);  // one tile: codes + scales
    const size_t smem = kGStages * buf + 2 * (size_t)warps * ng * 4 * 32 * sizeof(float);
    if (smem > 160 * 1024) return cudaErrorInvalidValue;
    if (mx) {
        if (ng == 1) return launch_ng<1, kFmtMxfp4>(a, tiles, warps * 32, smem, s);
        return launch_ng<2, kFmtMxfp4>(a, tiles, warps * 32, smem, s);
    }
    if (ng == 1) return launch_ng<1, kFmtNvfp4>(a, tiles, warps * 32, smem, s);
    return launch_ng<2, kFmtNvfp4>(a, tiles, warps * 32, smem, s);
}

}  // namespace moe
