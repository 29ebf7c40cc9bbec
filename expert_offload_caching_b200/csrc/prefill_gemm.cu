// Grouped NVFP4 x NVFP4 expert GEMMs of a prefill chunk on the 5th-generation
// tensor cores: tcgen05.mma kind::mxf4nvf4 with one E4M3 scale per 16 values
// (block16), operands staged by TMA, fp32 accumulators in tensor memory.
//
// What is computed is the W4A4 expert of the checkpoint (florigen.ai, "NVFP4で
// 約135GBまで縮める": routed experts in NVFP4 for weights and activations): for
// every distinct expert e of the layer and every row r routed to it,
//   gate/up:  [g; u](r) = (Wq_e . xq_r) * ts_w * st_x(r)      (ts_w: gate or up scale)
//             h(r) = silu(g) * u
//   down:     y_e(r) = (W2q_e . hq_r) * ts_down * st_h(r)
// where Wq, xq, hq are the E2M1 values times their E4M3 block scales (the
// products are exact; the sum is accumulated in fp32 by the tensor core) and
// ts, st are the fp32 per-matrix and per-row scales, applied in the epilogue.
//
// Orientation ("weights as M"): a CTA computes one 128-row tile of an expert's
// weight matrix against up to 128 rows of that expert's activations (the MMA's
// N, 16..128), since the rows per expert are few (k*T/E, about 80 for a
// 4096-row chunk of 512 experts, top-10) while the weight rows are many.
// Activation rows sit in expert-grouped order (the scatter of the routing
// step), so an expert's rows are one contiguous TMA box.
//
// Per CTA: warp 0 stages K in steps of 256 values (128 bytes: one row of the
// 128-byte swizzle) -- one TMA box of the weight tile, one of the activation
// tile, and the two scale-factor atoms of each 64-value MMA step, written by
// the warp's lanes -- into a 3-deep ring; warp 1 copies the scale factors into
// tensor memory (tcgen05.cp) and issues the MMAs from one thread; warps 2-5
// read the accumulator (tcgen05.ld) and apply the epilogue.  Every mbarrier
// wait is bounded in time; a wait that runs out records an error in the mapped
// page and the CTA winds down and frees its tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kBM = 128;                 // weight rows per tile (MMA M)
constexpr int kBN = 128;                 // activation rows per tile (largest MMA N used)
constexpr int kStageKBytes = 128;        // K bytes per stage: 256 E2M1 values
constexpr int kStepsPerStage = 4;        // MMA K = 64 values = 32 bytes
constexpr int kStages = 3;
constexpr int kGemmThreads = 192;        // 6 warps
constexpr uint32_t kTileBytes = kBM * kStageKBytes;  // 16 KB, weight and activation tiles alike
constexpr uint32_t kSfAtom = 512;        // 128 rows x 4 E4M3 scales
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kTileBytes;
constexpr uint32_t kOffSfA = kOffB + kStages * kTileBytes;
constexpr uint32_t kOffSfB = kOffSfA + kStages * kStepsPerStage * kSfAtom;
constexpr uint32_t kOffBar = kOffSfB + kStages * kStepsPerStage * kSfAtom;
constexpr uint32_t kSmemUsed = kOffBar + 128;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // + alignment of the base to 1024
// Tensor memory: accumulator columns [0, 128), then per (stage, step) 4
// columns of A scales and 4 of B scales.
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemSf = 128;

static_assert(kTmemSf + kStages * kStepsPerStage * 8 <= kTmemCols, "tensor memory columns");
static_assert(kSmemBytes <= 113 * 1024, "two CTAs per SM");

__device__ __forceinline__ uint64_t gtimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ uint32_t saddr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarriers
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
// Wait for the phase of the given parity to complete; false after limit_ns.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
        if (i == 0) {
            t0 = gtimer();
        } else if ((i & 15) == 0 && gtimer() - t0 > limit_ns) {
            return false;
        }
    }
}

// ---- TMA (tiled, 128-byte swizzle, completion counted on an mbarrier)
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// ---- tcgen05
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
// 32 rows x 16 bytes of shared memory -> 4 columns of every lane quarter
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}
// MXFP4 x MXFP4: E2M1 with one UE8M0 scale per 32 values on each side (OCP
// microscaling); per MMA (K = 64) each row has two scales, in the low two bytes
// of its 32-bit scale-factor column (scale-factor id 0).
__device__ __forceinline__ void tc_mma_mxf4(uint32_t d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}
// arrive on the mbarrier once every tcgen05 operation issued so far by this thread is done
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}
// lanes [32q, 32q + 32) x 16 consecutive 32-bit columns; thread i gets lane 32q + i
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor of a K-major tile in the 128-byte swizzle
// layout that TMA writes: 128-byte rows, 8-row groups 1024 bytes apart (the
// tile base 1024-aligned; a K step inside the 128-byte row moves the start).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
    uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;             // leading byte offset (16 B; unused by this layout)
    d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;             // descriptor version of sm_100
    d |= (uint64_t)2 << 61;             // 128-byte swizzle
    return d;
}
// Descriptor of one scale-factor atom (32 rows of 16 bytes, no swizzle) for tcgen05.cp.
__device__ __forceinline__ uint64_t desc_sf(uint32_t addr) {
    uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;             // leading byte offset (one 16-byte column: unused)
    d |= (uint64_t)(128 >> 4) << 32;    // stride byte offset: 8 rows x 16 B
    d |= (uint64_t)1 << 46;
    return d;
}
// Instruction descriptor: E2M1 x E2M1, UE4M3 scales, K-major A and B, M = 128, N.
__device__ __forceinline__ uint32_t idesc_nvf4(int N) {
    return (1u << 7)                          // A format E2M1
           | (1u << 10)                       // B format E2M1
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(kBM >> 4) << 24);    // M / 16; scale format bit 23 = 0: UE4M3
}

// A bounded wait ran out: record where in the mapped page (plain stores; when
// several CTAs fail, one of them is reported).
__device__ void gemm_fail(const GroupedGemmArgs &a, int code, int stage) {
    a.page->diag[1] = 10 + a.mode;
    a.page->diag[2] = (int)blockIdx.x;
    a.page->diag[3] = stage;
    a.page->diag[4] = (int)threadIdx.x;
    a.page->diag[5] = a.d;
    a.page->diag[6] = a.F;
    __threadfence_system();
    a.page->error = code;
    __threadfence_system();
}

// FMT: the records' format.  NVFP4: E4M3 scales per 16 (kind::mxf4nvf4
// block16), per-matrix and per-row fp32 scales in the epilogue.  MXFP4: E8M0
// scales per 32 (kind::mxf4 block32), nothing else to apply.
template <int FMT>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_ws,
                        const __grid_constant__ CUtensorMap tm_act, const GroupedGemmArgs a) {
    constexpr bool kMx = FMT == kFmtMxfp4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = (int)blockIdx.x / a.m_tiles, mt = (int)blockIdx.x % a.m_tiles;
    if (pair >= *a.n_pairs) return;  // grid sized for the worst case
    const int2 pr = a.pairs[pair];   // (job, n tile); job == n_jobs: the shared expert
    const int nj = *a.n_jobs;
    const bool shared = pr.x >= nj;
    int nrows, row_off, zc;
    const uint8_t *rec;
    if (shared) {
        nrows = a.T;
        row_off = a.T * a.k;
        zc = a.layer;
        rec = a.shared_rec + (int64_t)a.layer * a.rec_bytes;
    } else {
        const Job jb = a.jobs[pr.x];
        nrows = jb.nrows;
        row_off = jb.row_off;
        zc = jb.slot;
        rec = a.arena + (int64_t)jb.slot * a.rec_bytes;
    }
    const int n0 = pr.y * kBN;
    const int nvalid = min(kBN, nrows - n0);
    const int N = (nvalid + 15) & ~15;
    const bool gate_up = a.mode == kGateUp;
    const int K = gate_up ? a.d : a.F;
    const int rows_w = gate_up ? 2 * a.F : a.d;
    const int ksteps = K >> 6;
    const int nkb = (ksteps + kStepsPerStage - 1) / kStepsPerStage;
    const int sf_pitch = kMx ? K >> 5 : K >> 4;  // scale bytes per row, weights and activations alike
    const uint8_t *wsf = rec + (gate_up ? a.lay.w13_scales : a.lay.w2_scales);
    const float *tsc = kMx ? nullptr : reinterpret_cast<const float *>(rec + a.lay.tscales);

    extern __shared__ uint8_t dsm_raw[];
    const uint32_t raw = saddr(dsm_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sm = dsm_raw + (base - raw);
    const uint32_t bar_full = base + kOffBar, bar_empty = bar_full + 8 * kStages,
                   bar_done = bar_empty + 8 * kStages;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sm + kOffBar + 8 * (2 * kStages + 1));
    volatile int32_t *s_fail = reinterpret_cast<volatile int32_t *>(sm + kOffBar + 8 * (2 * kStages + 1) + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 33);  // lane 0's tx-count arrive + all 32 lanes after their scales
            mbar_init(bar_empty + 8 * s, 1);  // tcgen05.commit of the MMA thread
        }
        mbar_init(bar_done, 1);
        *s_fail = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        tmem_alloc(base + kOffBar + 8 * (2 * kStages + 1), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 0) span_mark(a.span, 0);

    if (warp == 0) {
        // ---- producer: operand tiles by TMA, scale factors by the lanes.  The
        // scale words of stage it + 1 are loaded into registers while stage it
        // is handed over, so their latency overlaps the wait for a free stage.
        uint32_t wa[4][kStepsPerStage], wb[4][kStepsPerStage];
        auto load_sf = [&](int itl) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                // row m = lane + 32c of the tile; its 4 scales of a K step are one word
                const int wrow = mt * kBM + lane + 32 * c;
                const int n = n0 + lane + 32 * c;
                const uint8_t *pw = wsf + (int64_t)wrow * sf_pitch;
                const uint8_t *pb = a.act_scales + (int64_t)(row_off + n) * sf_pitch;
#pragma unroll
                for (int i = 0; i < kStepsPerStage; ++i) {
                    const int ks = itl * kStepsPerStage + i;
                    if constexpr (kMx) {  // two E8M0 bytes, as bytes 0-1 (and again 2-3) of the word
                        const uint32_t va = (wrow < rows_w && ks < ksteps)
                                                ? __ldg(reinterpret_cast<const uint16_t *>(pw) + ks) : 0u;
                        const uint32_t vb = (n < nrows && ks < ksteps)
                                                ? __ldg(reinterpret_cast<const uint16_t *>(pb) + ks) : 0u;
                        wa[c][i] = va | (va << 16);
                        wb[c][i] = vb | (vb << 16);
                    } else {
                        wa[c][i] = (wrow < rows_w && ks < ksteps) ? __ldg(reinterpret_cast<const uint32_t *>(pw) + ks) : 0u;
                        wb[c][i] = (n < nrows && ks < ksteps) ? __ldg(reinterpret_cast<const uint32_t *>(pb) + ks) : 0u;
                    }
                }
            }
        };
        load_sf(0);
        int it = 0;
        for (; it < nkb; ++it) {
            const int s = it % kStages, r = it / kStages;
            bool ok = r == 0 || mbar_wait(bar_empty + 8 * s, (r - 1) & 1, a.wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
                if (lane == 0) { gemm_fail(a, 41, it); *s_fail = 1; }
                break;
            }
            if (lane == 0) {
                mbar_arrive_tx(bar_full + 8 * s, 2 * kTileBytes);
                const uint32_t da = base + kOffA + s * kTileBytes, db = base + kOffB + s * kTileBytes;
                // test injection: block 0 never issues its first stage's copies, so
                // that stage's wait runs out (the wind-down path below is exercised)
                if (!(a.inj_skip && blockIdx.x == 0 && it == 0)) {
                    tma_load_3d(da, shared ? &tm_ws : &tm_w, bar_full + 8 * s, it * kStageKBytes, mt * kBM, zc);
                    tma_load_2d(db, &tm_act, bar_full + 8 * s, it * kStageKBytes, row_off + n0);
                }
            }
            // scale-factor atoms: lane row holds rows lane, lane + 32, lane + 64, lane + 96
#pragma unroll
            for (int i = 0; i < kStepsPerStage; ++i) {
                uint4 *sfa = reinterpret_cast<uint4 *>(sm + kOffSfA + (s * kStepsPerStage + i) * kSfAtom);
                uint4 *sfb = reinterpret_cast<uint4 *>(sm + kOffSfB + (s * kStepsPerStage + i) * kSfAtom);
                sfa[lane] = make_uint4(wa[0][i], wa[1][i], wa[2][i], wa[3][i]);
                sfb[lane] = make_uint4(wb[0][i], wb[1][i], wb[2][i], wb[3][i]);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(bar_full + 8 * s);
            if (it + 1 < nkb) load_sf(it + 1);
        }
        // on failure: let the stages already issued land before the CTA exits
        if (it < nkb && lane == 0) {
            for (int j = it - 1; j >= 0 && j >= it - kStages; --j)
                mbar_wait(bar_full + 8 * (j % kStages), (j / kStages) & 1, a.wait_ns);
        }
    } else if (warp == 1) {
        // ---- MMA issue, one thread
        if (lane == 0) {
            const uint32_t idesc = idesc_nvf4(N) | (kMx ? (1u << 23) : 0u);  // bit 23: UE8M0 scales
            for (int it = 0; it < nkb; ++it) {
                const int s = it % kStages, r = it / kStages;
                if (!mbar_wait(bar_full + 8 * s, r & 1, a.wait_ns)) {
                    gemm_fail(a, 42, it);
                    *s_fail = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t da = base + kOffA + s * kTileBytes, db = base + kOffB + s * kTileBytes;
                for (int i = 0; i < kStepsPerStage; ++i) {
                    const int ks = it * kStepsPerStage + i;
                    if (ks >= ksteps) break;
                    const uint32_t t_sfa = tmem + kTmemSf + (uint32_t)((s * kStepsPerStage + i) * 8);
                    const uint32_t t_sfb = t_sfa + 4;
                    tc_cp_sf(t_sfa, desc_sf(base + kOffSfA + (s * kStepsPerStage + i) * kSfAtom));
                    tc_cp_sf(t_sfb, desc_sf(base + kOffSfB + (s * kStepsPerStage + i) * kSfAtom));
                    if constexpr (kMx)
                        tc_mma_mxf4(tmem, desc_sw128(da + 32 * i), desc_sw128(db + 32 * i), idesc, t_sfa, t_sfb,
                                    (it | i) != 0 ? 1u : 0u);
                    else
                        tc_mma_nvf4(tmem, desc_sw128(da + 32 * i), desc_sw128(db + 32 * i), idesc, t_sfa, t_sfb,
                                    (it | i) != 0 ? 1u : 0u);
                }
                tc_commit(bar_empty + 8 * s);
            }
            tc_commit(bar_done);
        }
        __syncwarp();
    } else {
        // ---- epilogue: warp w reads lanes [32 (w % 4), +32) of the accumulator
        bool ok = mbar_wait(bar_done, 0, a.wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && lane == 0) { gemm_fail(a, 43, nkb); *s_fail = 1; }
        tc_fence_after();
        if (ok && !*s_fail) {
            const int q = warp & 3;
            const int m = q * 32 + lane;
            const int wrow = mt * kBM + m;
            const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
            if (gate_up) {
                const float ts_g = kMx ? 1.0f : tsc[0], ts_u = kMx ? 1.0f : tsc[1];
                for (int c0 = 0; c0 < N; c0 += 16) {
                    float v[16];
                    tmem_ld16(trow + (uint32_t)c0, v);
#pragma unroll
                    for (int cc = 0; cc < 16; ++cc) {
                        const float other = __shfl_xor_sync(0xffffffffu, v[cc], 1);
                        const int n = c0 + cc;
                        if ((lane & 1) == 0 && n < nvalid && wrow < rows_w) {
                            const int g = row_off + n0 + n;
                            const float st = kMx ? 1.0f : a.act_st[g];
                            const float gt = v[cc] * ts_g * st;   // row 2j: gate_j
                            const float up = other * ts_u * st;   // row 2j + 1: up_j
                            a.h32[(int64_t)g * a.F + (wrow >> 1)] = gt / (1.0f + expf(-gt)) * up;
                        }
                    }
                }
            } else {
                const float ts_d = kMx ? 1.0f : tsc[2];
                const int tk = a.T * a.k;
                for (int c0 = 0; c0 < N; c0 += 16) {
                    float v[16];
                    tmem_ld16(trow + (uint32_t)c0, v);
#pragma unroll
                    for (int cc = 0; cc < 16; ++cc) {
                        const int n = c0 + cc;
                        if (n < nvalid && wrow < rows_w) {
                            const int g = row_off + n0 + n;
                            int t, p;
                            if (g < tk) {
                                const RowRef rr = a.rowrefs[g];
                                t = rr.t;
                                p = rr.p;
                            } else {
                                t = g - tk;
                                p = a.k;
                            }
                            a.part[((int64_t)t * (a.k + 1) + p) * a.d + wrow] =
                                v[cc] * ts_d * (kMx ? 1.0f : a.act_st[g]);
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0) span_mark(a.span, 1);
}

// (job, n tile) pairs of the layer: a block-wide exclusive scan over the jobs
// of ceil(rows / kBN), then the shared expert's tiles (job index n_jobs).
__global__ void __launch_bounds__(1024) tile_plan_kernel(const Job *jobs, const int32_t *n_jobs, int T,
                                                         int has_shared, int2 *pairs, int32_t *n_pairs) {
    __shared__ int s_warp[32];
    __shared__ int s_total;
    const int nj = *n_jobs;
    const int j = threadIdx.x;
    const int cnt = j < nj ? (jobs[j].nrows + kBN - 1) / kBN : 0;
    const int lane = j & 31, w = j >> 5;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[w] = incl;
    __syncthreads();
    if (w == 0) {
        int v = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        s_warp[lane] = v;  // inclusive over warps
        if (lane == 31) s_total = v;
    }
    __syncthreads();
    const int excl = incl - cnt + (w > 0 ? s_warp[w - 1] : 0);
    for (int i = 0; i < cnt; ++i) pairs[excl + i] = make_int2(j, i);
    const int nsh = has_shared ? (T + kBN - 1) / kBN : 0;
    for (int i = j; i < nsh; i += blockDim.x) pairs[s_total + i] = make_int2(nj, i);
    if (j == 0) *n_pairs = s_total + nsh;
}

// ---- bf16 x bf16 -> fp32 GEMM on the tensor cores (tcgen05.mma kind::f16,
// accumulators in tensor memory): out[t][n] = sum_K A[t][K] B[n][K], A and B
// K-major bf16 (TMA boxes of 128 bytes = 64 values of K, 128-byte swizzle,
// 4 MMAs of K = 16 per box, a 4-deep ring).  One CTA per 128 rows of A x 128
// rows of B.  The products are exact in fp32; only the summation order
// differs from an fp32 FMA chain.  Uses: the router logits of a prefill chunk
// (A = x, B = W_r of the layer) and a BF16 shared expert (A = x, B = W13; then
// A = h as bf16 (hi, lo) halves, B = W2 with K wrapped: K positions j and F + j
// both read W2's column j, so hi and lo meet W2 in one accumulation).
constexpr int kRStages = 4;
constexpr uint64_t kRWaitNs = 4000000000ull;  // 4 s per wait
constexpr uint32_t kROffBar = 2 * kRStages * kTileBytes;
constexpr uint32_t kRSmemBytes = kROffBar + 128 + 1024;

__device__ __forceinline__ void tc_mma_bf16(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t"
        "}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}
// Instruction descriptor: bf16 x bf16 -> fp32, K-major A and B, M = 128, N.
__device__ __forceinline__ uint32_t idesc_bf16(int N) {
    return (1u << 4)                          // D format fp32
           | (1u << 7)                        // A format bf16
           | (1u << 10)                       // B format bf16
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(kBM >> 4) << 24);    // M / 16
}

__device__ void router_fail(HostPage *page, int code, int stage) {
    page->diag[1] = 20;
    page->diag[2] = (int)(blockIdx.x + 1000 * blockIdx.y);
    page->diag[3] = stage;
    page->diag[4] = (int)threadIdx.x;
    __threadfence_system();
    page->error = code;
    __threadfence_system();
}

// kbytes: bytes of K per row of A; wrap: B's K coordinate is taken modulo wrap
// bytes (0: no wrap); zb: B's matrix index (layer) in its 3D map.
__global__ void __launch_bounds__(kGemmThreads, 1)
    bf16_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     float *z, int64_t z_stride, int T, int E, int kbytes, int wrap, int layer, HostPage *page) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * kBM, e0 = blockIdx.y * kBM;
    const int nkb = (kbytes + kStageKBytes - 1) / kStageKBytes;
    extern __shared__ uint8_t dsm_raw[];
    const uint32_t raw = saddr(dsm_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sm = dsm_raw + (base - raw);
    const uint32_t bar_full = base + kROffBar, bar_empty = bar_full + 8 * kRStages,
                   bar_done = bar_empty + 8 * kRStages;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sm + kROffBar + 8 * (2 * kRStages + 1));
    volatile int32_t *s_fail = reinterpret_cast<volatile int32_t *>(sm + kROffBar + 8 * (2 * kRStages + 1) + 4);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kRStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(bar_done, 1);
        *s_fail = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        tmem_alloc(base + kROffBar + 8 * (2 * kRStages + 1), 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {  // TMA producer
            int it = 0;
            for (; it < nkb; ++it) {
                const int s = it % kRStages, r = it / kRStages;
                if (r > 0 && !mbar_wait(bar_empty + 8 * s, (r - 1) & 1, kRWaitNs)) {
                    router_fail(page, 51, it);
                    *s_fail = 1;
                    break;
                }
                mbar_arrive_tx(bar_full + 8 * s, 2 * kTileBytes);
                tma_load_2d(base + s * kTileBytes, &tm_x, bar_full + 8 * s, it * kStageKBytes, t0);
                const int kb = it * kStageKBytes;
                tma_load_3d(base + (kRStages + s) * kTileBytes, &tm_w, bar_full + 8 * s, wrap ? kb % wrap : kb, e0,
                            layer);
            }
            if (it < nkb)  // let the stages already issued land before the CTA exits
                for (int j = it - 1; j >= 0 && j >= it - kRStages; --j)
                    mbar_wait(bar_full + 8 * (j % kRStages), (j / kRStages) & 1, kRWaitNs);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {  // MMA issue
            const uint32_t idesc = idesc_bf16(kBM);
            for (int it = 0; it < nkb; ++it) {
                const int s = it % kRStages, r = it / kRStages;
                if (!mbar_wait(bar_full + 8 * s, r & 1, kRWaitNs)) {
                    router_fail(page, 52, it);
                    *s_fail = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t da = base + s * kTileBytes, db = base + (kRStages + s) * kTileBytes;
                const int steps = min(4, (kbytes - it * kStageKBytes) / 32);  // K = 16 bf16 = 32 bytes each
                for (int i = 0; i < steps; ++i)
                    tc_mma_bf16(tmem, desc_sw128(da + 32 * i), desc_sw128(db + 32 * i), idesc, (it | i) != 0);
                tc_commit(bar_empty + 8 * s);
            }
            tc_commit(bar_done);
        }
        __syncwarp();
    } else {  // epilogue: lane = row of x, columns = experts
        bool ok = mbar_wait(bar_done, 0, kRWaitNs);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && lane == 0) { router_fail(page, 53, nkb); *s_fail = 1; }
        tc_fence_after();
        if (ok && !*s_fail) {
            const int q = warp & 3;
            const int t = t0 + q * 32 + lane;
            const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
            for (int c0 = 0; c0 < kBM && e0 + c0 < E; c0 += 16) {
                float v[16];
                tmem_ld16(trow + (uint32_t)c0, v);
                if (t < T) {
                    float *zr = z + (size_t)t * z_stride + e0 + c0;
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (e0 + c0 + i < E) zr[i] = v[i];
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

}  // namespace

cudaError_t launch_bf16_gemm(const CUtensorMap &tm_a, const CUtensorMap &tm_b, float *out, int64_t out_stride,
                             int M, int N, int kbytes, int wrap, int zb, HostPage *page, cudaStream_t s) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(bf16_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kRSmemBytes);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    if ((kbytes % kStageKBytes) || (wrap % kStageKBytes)) return cudaErrorInvalidValue;  // whole TMA boxes
    const dim3 grid((M + kBM - 1) / kBM, (N + kBM - 1) / kBM);
    bf16_gemm_kernel<<<grid, kGemmThreads, kRSmemBytes, s>>>(tm_a, tm_b, out, out_stride, M, N, kbytes, wrap, zb,
                                                             page);
    return cudaGetLastError();
}

cudaError_t launch_router_gemm(const CUtensorMap &tm_x, const CUtensorMap &tm_w, float *z, int T, int E, int d,
                               int layer, HostPage *page, cudaStream_t s) {
    return launch_bf16_gemm(tm_x, tm_w, z, E, T, E, 2 * d, 0, layer, page, s);
}



int grouped_pairs_cap(int n_jobs, int T, int k, int has_shared) {
    return n_jobs + (T * k + kBN - 1) / kBN + (has_shared ? (T + kBN - 1) / kBN : 0);
}

cudaError_t launch_tile_plan(const Job *jobs, const int32_t *n_jobs, int T, int has_shared, int2 *pairs,
                             int32_t *n_pairs, cudaStream_t s) {
    tile_plan_kernel<<<1, 1024, 0, s>>>(jobs, n_jobs, T, has_shared, pairs, n_pairs);
    return cudaGetLastError();
}

cudaError_t launch_grouped_gemm(const GroupedGemmMaps &maps, const GroupedGemmArgs &a, int pairs_cap,
                                cudaStream_t s) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<kFmtNvfp4>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(grouped_gemm_kernel<kFmtMxfp4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const CUtensorMap &w = a.mode == kGateUp ? maps.w13 : maps.w2;
    const CUtensorMap &ws = a.mode == kGateUp ? maps.w13_shared : maps.w2_shared;
    const CUtensorMap &act = a.mode == kGateUp ? maps.xq : maps.hq;
    const unsigned grid = (unsigned)pairs_cap * (unsigned)a.m_tiles;
    if (grid == 0) return cudaSuccess;
    if (a.lay.fmt == kFmtMxfp4)
        grouped_gemm_kernel<kFmtMxfp4><<<grid, kGemmThreads, kSmemBytes, s>>>(w, ws, act, a);
    else if (a.lay.fmt == kFmtNvfp4)
        grouped_gemm_kernel<kFmtNvfp4><<<grid, kGemmThreads, kSmemBytes, s>>>(w, ws, act, a);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

// ---- tensor maps (host)
namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}
}  // namespace

// rows x row_bytes bytes per matrix, `count` matrices `matrix_stride` bytes
// apart (count 0: a single 2D matrix); boxes of 128 bytes x 128 rows.
bool make_operand_map(CUtensorMap *out, const void *base, int64_t row_bytes, int64_t rows, int64_t count,
                      int64_t matrix_stride) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn || !base) return false;
    if ((reinterpret_cast<uintptr_t>(base) & 15) || (row_bytes & 15) || (matrix_stride & 15)) return false;
    cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)rows, (cuuint64_t)(count > 0 ? count : 1)};
    cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)matrix_stride};
    cuuint32_t box[3] = {(cuuint32_t)kStageKBytes, (cuuint32_t)kBM, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const cuuint32_t rank = count > 0 ? 3 : 2;
    const CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace moe
