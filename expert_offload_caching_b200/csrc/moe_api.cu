// C ABI of the per-layer routed-expert step (declared in include/moe_offload.h).
//
// One layer (FreeToken offload backend, florigen.ai "FreeTokenは何をしているのか": experts
// in host RAM, an LRU cache of expert slots on the GPU, misses sent over PCIe):
//   compute stream:  route+top-k+lookup kernel -> gate/up and down GEMVs of the
//                    hit experts and the shared expert (they run while the host
//                    reads the miss list) -> per miss: wait for its copy event,
//                    gate/up + down of that expert -> combine.
//   host:            waits (bounded) for the device's miss list in mapped pinned
//                    memory, then issues one cudaMemcpyAsync per miss on the copy
//                    stream (pinned pool -> slot) with an event after each.
//   copy stream:     the miss records, back to back.
// A slot is only overwritten after the lookup that evicted it has run, i.e.
// after every earlier kernel on the compute stream; copies of one slot are
// ordered on the copy stream.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>
#include <immintrin.h>

#include "../../include/moe_offload.h"
#include "moe_internal.cuh"

using namespace moe;
static_assert(kFmtNvfp4 == MOE_FMT_NVFP4 && kFmtMxfp4 == MOE_FMT_MXFP4 && kFmtBf16 == MOE_FMT_BF16,
              "record format values");

namespace {

inline int64_t up256(int64_t x) { return (x + 255) / 256 * 256; }

bool dims_valid(const moe_dims *d) {
    return d && d->L > 0 && d->E > 0 && d->k > 0 && d->k <= d->E && d->d > 0 && d->F > 0 &&
           d->max_rows > 0 && d->pool_records >= 0 &&
           (d->weight_format == MOE_FMT_NVFP4 || d->weight_format == MOE_FMT_MXFP4) &&
           (!d->has_shared || d->shared_format == d->weight_format || d->shared_format == MOE_FMT_BF16);
}
// The shared experts' format (the routed one when there are none).
int shared_fmt(const moe_dims *d) { return d->has_shared ? d->shared_format : d->weight_format; }
bool dims_supported(const moe_dims *d) {
    return d->d % 64 == 0 && d->F % 64 == 0 && d->d <= 4096 && d->F <= 4096 && d->k <= kMaxK &&
           d->E <= kMaxE &&
           d->max_rows <= 4096 && (int64_t)d->L * d->E < (1ll << 31) &&
           // prefill GEMM operands: TMA boxes of 128 bytes of a row
           (d->max_rows <= kDecodeMaxRows || (d->d >= 256 && d->F >= 256));
}

// Section offsets of a record of format fmt (the header's MOE_FMT_* layouts).
RecordLayout layout_fmt(const moe_dims *d, int fmt) {
    RecordLayout r;
    const int64_t dd = d->d, ff = d->F;
    r.fmt = fmt;
    if (fmt == MOE_FMT_BF16) {  // W13 then W2, bf16, unpadded
        r.tscales = r.w13_scales = r.w2_scales = -1;
        r.w13_codes = 0;
        r.w2_codes = 2 * (2 * ff * dd);
        r.bytes = r.w2_codes + 2 * (dd * ff);
    } else if (fmt == MOE_FMT_MXFP4) {  // E8M0 scale per 32, no tensor scales
        r.tscales = -1;
        r.w13_codes = 0;
        r.w13_scales = r.w13_codes + up256(2 * ff * dd / 2);
        r.w2_codes = r.w13_scales + up256(2 * ff * dd / 32);
        r.w2_scales = r.w2_codes + up256(dd * ff / 2);
        r.bytes = r.w2_scales + up256(dd * ff / 32);
    } else {
        r.tscales = 0;  // head: the gate/up half (tensor scales + W13) is a contiguous prefix
        r.w13_codes = up256(12);
        r.w13_scales = r.w13_codes + up256(2 * ff * dd / 2);
        r.w2_codes = r.w13_scales + up256(2 * ff * dd / 16);
        r.w2_scales = r.w2_codes + up256(dd * ff / 2);
        r.bytes = r.w2_scales + up256(dd * ff / 16);
    }
    return r;
}
RecordLayout layout_of(const moe_dims *d) { return layout_fmt(d, d->weight_format); }
RecordLayout shared_layout_of(const moe_dims *d) { return layout_fmt(d, shared_fmt(d)); }

int max_jobs(const moe_dims *d, int T) {
    int64_t n = (int64_t)T * d->k;
    return (int)(n < d->E ? n : d->E);
}

// Workspace carve-up (offsets from the caller's base).  Row buffers are sized
// for the largest call (max_rows); the prefill buffers exist when max_rows > 32.
constexpr int64_t kLkWords = 4 + 4 * (int64_t)kMaxSlots + 4;
struct WsLayout {
    int64_t z, idx, gates, jobs, n_jobs, n_misses, ticket, ticket2, lk, rowrefs, xh, hh, part, cnt, fill,
        jobidx, h32, xq, xq_scales, xq_st, hq, hq_scales, hq_st, pairs, n_pairs, n_grouped, sg, hs, xstage, ystage,
        total;
};
int pairs_capacity(const moe_dims *d) {
    return grouped_pairs_cap(d->E, d->max_rows, d->k, d->has_shared ? 1 : 0);
}
WsLayout ws_layout(const moe_dims *d) {
    WsLayout w;
    const int64_t T = d->max_rows, k = d->k, E = d->E, dd = d->d, F = d->F;
    const bool prefill = T > kDecodeMaxRows;
    const int64_t Td = prefill ? kDecodeMaxRows : T;  // rows of the decode-only buffers
    const int64_t R = T * (k + 1);                     // grouped prefill rows (routed + shared)
    int64_t o = 0;
    auto take = [&](int64_t bytes) { int64_t r = o; o += up256(bytes); return r; };
    w.z = take(T * E * 4);
    w.idx = take(T * k * 4);
    w.gates = take(T * k * 4);
    const int64_t nj = prefill ? E : max_jobs(d, (int)T);
    w.jobs = take(nj * (int64_t)sizeof(Job));
    w.n_jobs = take(4);
    w.n_misses = take(4);
    w.ticket = take(4);
    w.ticket2 = take(4 * kMaxTiles);
    // layer kernel: queue[2], release, pad, done_a, flags; streaming kernel: done, exit (+3 pad)
    w.lk = take(4 * (kLkWords));
    w.rowrefs = take(T * k * (int64_t)sizeof(RowRef));
    w.xh = take(Td * 2 * dd * 2);
    w.hh = take(Td * (k + 1) * 2 * F * 2);
    w.part = take(T * (k + 1) * dd * 4);
    w.cnt = prefill ? take(E * 4) : -1;
    w.fill = prefill ? take(E * 4) : -1;
    w.jobidx = prefill ? take(E * 4) : -1;
    w.h32 = prefill ? take(R * F * 4) : -1;
    w.xq = prefill ? take(R * dd / 2) : -1;
    w.xq_scales = prefill ? take(R * dd / 16) : -1;
    w.xq_st = prefill ? take(R * 4) : -1;
    w.hq = prefill ? take(R * F / 2) : -1;
    w.hq_scales = prefill ? take(R * F / 16) : -1;
    w.hq_st = prefill ? take(R * 4) : -1;
    w.pairs = prefill ? take((int64_t)pairs_capacity(d) * 8) : -1;
    w.n_pairs = prefill ? take(4) : -1;
    w.n_grouped = prefill ? take(4) : -1;
    // a BF16 shared expert on the prefill path: its gate/up outputs [T][2F] fp32
    // and h as bf16 (hi, lo) halves [T][2F]
    const bool sbf = prefill && d->has_shared && d->shared_format == MOE_FMT_BF16;
    w.sg = sbf ? take(T * 2 * F * 4) : -1;
    w.hs = sbf ? take(T * 2 * F * 2) : -1;
    w.xstage = take(T * dd * 2);
    w.ystage = take(T * dd * 4);
    w.total = o;
    return w;
}

struct TableLayout {
    int64_t hdr, map, owner, stamp, total;
};
TableLayout table_layout(const moe_dims *d, int64_t C) {
    TableLayout t;
    int64_t o = 0;
    auto take = [&](int64_t bytes) { int64_t r = o; o += up256(bytes); return r; };
    t.hdr = take(sizeof(TableHdr));
    t.map = take((int64_t)d->L * d->E * 4);
    t.owner = take(C * 4);
    t.stamp = take(C * 8);
    t.total = o;
    return t;
}

struct TimedLaunch {
    int cls;
    cudaEvent_t a, b;
    double bytes;
    int64_t slot;  // device span slot, -1 if the kernel is not instrumented
};

}  // namespace

struct moe_ctx {
    moe_dims dims;
    RecordLayout lay;   // routed records
    RecordLayout slay;  // shared-expert records
    int64_t P = 0;
    const uint8_t *pool = nullptr;
    const __nv_bfloat16 *router_w = nullptr;
    const uint8_t *shared_recs = nullptr;
    uint8_t *ws = nullptr;
    WsLayout wl;
    DecodeWs dws;
    cudaStream_t cs = nullptr, xs = nullptr;
    // decode misses alternate between the caller's copy stream and one of the
    // library's own (copy_streams = 2), so one copy's start-up overlaps the
    // other's transfer; xs2 starts after xs's earlier work (ev_xs_tail) and xs
    // waits for xs2 at the end of each call, so the caller's copy stream still
    // covers every copy
    cudaStream_t xs2 = nullptr;
    cudaEvent_t ev_xs_tail = nullptr, ev_xs2_tail = nullptr;
    int copy_streams = 1;
    // decode expert kernels of the per-miss path: 1 = streaming (bulk-copy ring,
    // a warp per tile; the hit experts' gate/up and down in one launch), 0 = the
    // split-K kernel (expert_gemv.cu)
    int gemv_kind = 1;
    // decode: the hit launch's SMs copy the first head_bytes of the layer's first
    // miss from the pool (pool_d: its device address) while the copy engine
    // starts on the rest (moe_debug_inject what = 10; 0: off)
    const uint8_t *pool_d = nullptr;
    uint32_t head_bytes = 0;
    // decode misses: the whole record as one copy (the default: fewer copy
    // start-ups; measured faster or equal), or the gate/up prefix and W2 as two,
    // so a miss's gate/up runs while its W2 streams (what = 11)
    bool split_copies = false;
    // diagnostic trace of the next streaming hit launches (moe_debug_inject what = 9)
    unsigned long long *trace_d = nullptr;
    int64_t trace_arm = 0;
    // cache
    uint8_t *arena = nullptr;
    int64_t C = 0;
    Table tab;
    uint32_t flags = 0;
    bool configured = false;
    // miss list page
    HostPage *page_h = nullptr, *page_d = nullptr;
    int page_cap = 0;
    uint32_t seq = 0;
    std::vector<cudaEvent_t> miss_ev;   // [2 * page_cap]: W13 part, W2 part of miss j
    cudaEvent_t ev_routed = nullptr;    // prefill: this layer's routed misses copied
    std::vector<cudaEvent_t> ev_pf;     // [L]: prefetch copies for a layer issued
    std::vector<char> pf_pending;       // [L]: a prefetch for the layer is not yet waited on
    // prefill GEMM operand descriptors (activation and shared maps at init,
    // arena maps at cache_configure)
    GroupedGemmMaps maps;
    // state
    moe_status state = MOE_OK;
    std::string err;
    moe_stats stats;
    int last_T = 0;
    // timing
    bool timing = false;
    std::vector<cudaEvent_t> ev_pool;
    std::vector<TimedLaunch> pending;
    // injection and limits
    int64_t inj_copy_fail_at = 0, inj_drop_publish = 0, inj_drop_flags = 0, inj_gemm_skip = 0, inj_stream_skip = 0;
    // decode: a launch for the hit experts and a gate/up and a down launch per
    // miss, gated by copy events (the default; measured faster: a stream memory
    // write between copies idles the copy engine longer than an event record),
    // or the persistent layer kernel (one launch per layer, misses gated by
    // flags the copy stream writes; where stream memory writes work: fused_ok)
    bool fused = false, fused_ok = false;
    // expert parallelism: the routed experts e with e % ep_size == ep_rank; the
    // shared expert on rank 0; y is this rank's partial sum
    int32_t ep_rank = 0, ep_size = 1;
    double wait_limit = 60.0;
    std::chrono::steady_clock::time_point issue_t0;  // end of the last miss-list wait
    // prefill with a BF16 shared expert: its gate/up outputs and bf16 (hi, lo) h
    float *dws_sg = nullptr;
    uint16_t *dws_hs = nullptr;
    // device spans of timed launches: [slot][2] = {min start, min ~end}, all ones when free
    unsigned long long *kspan = nullptr;
    int64_t kspan_cap = 0, kspan_used = 0;
};

namespace {

moe_status cuda_fail(moe_ctx *c, cudaError_t e, const char *what) {
    if (c) {
        c->err = std::string(what) + ": " + cudaGetErrorString(e);
    }
    return MOE_ERR_CUDA;
}
#define CK(call)                                                    \
    do {                                                            \
        cudaError_t e_ = (call);                                    \
        if (e_ != cudaSuccess) return cuda_fail(ctx, e_, #call);    \
    } while (0)

// cuStreamWriteValue32 (driver API, through the runtime's entry-point query):
// a 32-bit store to device memory executed in stream order, after the
// stream's earlier work (the default flags include a memory barrier, so the
// bytes of an earlier copy are visible before the value).
typedef CUresult (*StreamWriteFn)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);
StreamWriteFn stream_write_fn() {
    static const StreamWriteFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuStreamWriteValue32", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<StreamWriteFn>(p);
        cudaGetLastError();
        return static_cast<StreamWriteFn>(nullptr);
    }();
    return fn;
}
cudaError_t stream_write(cudaStream_t s, uint32_t *addr, uint32_t value) {
    const StreamWriteFn fn = stream_write_fn();
    if (!fn) return cudaErrorNotSupported;
    return fn(reinterpret_cast<CUstream>(s), reinterpret_cast<CUdeviceptr>(addr), value, 0) == CUDA_SUCCESS
               ? cudaSuccess
               : cudaErrorNotSupported;
}
// The copy stream of a call's m-th miss (0-based): every other one on the
// library's second copy stream when two are enabled; xs2's first copy of the
// call is ordered after xs's work of earlier calls.
cudaError_t miss_stream(moe_ctx *ctx, int m, bool *used2, cudaStream_t *out) {
    *out = ctx->xs;
    if (ctx->copy_streams < 2 || !(m & 1)) return cudaSuccess;
    *out = ctx->xs2;
    if (*used2) return cudaSuccess;
    *used2 = true;
    return cudaStreamWaitEvent(ctx->xs2, ctx->ev_xs_tail, 0);
}
// End of a call's copies: the caller's copy stream waits for xs2's, and marks
// where the next call's xs2 copies may start.
cudaError_t copy_tail(moe_ctx *ctx, bool used2) {
    cudaError_t e = cudaSuccess;
    if (used2) {
        e = cudaEventRecord(ctx->ev_xs2_tail, ctx->xs2);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(ctx->xs, ctx->ev_xs2_tail, 0);
    }
    if (e == cudaSuccess) e = cudaEventRecord(ctx->ev_xs_tail, ctx->xs);
    return e;
}

cudaEvent_t pool_event(moe_ctx *ctx) {
    if (!ctx->ev_pool.empty()) {
        cudaEvent_t e = ctx->ev_pool.back();
        ctx->ev_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

void time_begin(moe_ctx *ctx, TimedLaunch &tl, int cls) {
    tl.cls = cls;
    tl.a = tl.b = nullptr;
    tl.bytes = 0;
    tl.slot = -1;
    if (!ctx->timing) return;
    tl.a = pool_event(ctx);
    cudaEventRecord(tl.a, ctx->cs);
}
// A span slot for an instrumented launch (null when timing is off or the
// slots cannot be had); the kernel records into it.
unsigned long long *time_span(moe_ctx *ctx, TimedLaunch &tl) {
    if (!ctx->timing || !tl.a) return nullptr;
    if (!ctx->kspan) {
        const int64_t cap = 1 << 18;
        if (cudaMalloc(&ctx->kspan, cap * 2 * sizeof(unsigned long long)) != cudaSuccess ||
            cudaMemset(ctx->kspan, 0xff, cap * 2 * sizeof(unsigned long long)) != cudaSuccess) {
            cudaGetLastError();
            ctx->kspan = nullptr;
            return nullptr;
        }
        ctx->kspan_cap = cap;
    }
    if (ctx->kspan_used == ctx->kspan_cap) return nullptr;  // full until the next resolve
    tl.slot = ctx->kspan_used++;
    return ctx->kspan + 2 * tl.slot;
}
// Returns the index of the pending record, or -1 when timing is off.
long time_end(moe_ctx *ctx, TimedLaunch &tl, double bytes) {
    if (!ctx->timing || !tl.a) return -1;
    tl.b = pool_event(ctx);
    cudaEventRecord(tl.b, ctx->cs);
    tl.bytes = bytes;
    ctx->pending.push_back(tl);
    return (long)ctx->pending.size() - 1;
}
moe_status resolve_timing(moe_ctx *ctx) {
    if (ctx->pending.empty()) return MOE_OK;
    CK(cudaStreamSynchronize(ctx->cs));
    std::vector<unsigned long long> sp;
    if (ctx->kspan && ctx->kspan_used > 0) {
        sp.resize(2 * ctx->kspan_used);
        CK(cudaMemcpy(sp.data(), ctx->kspan, sp.size() * sizeof(unsigned long long), cudaMemcpyDeviceToHost));
        CK(cudaMemset(ctx->kspan, 0xff, sp.size() * sizeof(unsigned long long)));
        ctx->kspan_used = 0;
    }
    for (auto &t : ctx->pending) {
        float ms = 0.f;
        CK(cudaEventElapsedTime(&ms, t.a, t.b));
        ctx->stats.kernel_ms[t.cls] += ms;
        ctx->stats.kernel_launches[t.cls] += 1;
        ctx->stats.kernel_bytes[t.cls] += t.bytes;
        if (t.slot >= 0 && 2 * t.slot + 1 < (int64_t)sp.size()) {
            const unsigned long long start = sp[2 * t.slot], end = ~sp[2 * t.slot + 1];
            if (start != ~0ull && sp[2 * t.slot + 1] != ~0ull && end >= start)
                ctx->stats.kernel_span_ms[t.cls] += (double)(end - start) * 1e-6;
        }
        ctx->ev_pool.push_back(t.a);
        ctx->ev_pool.push_back(t.b);
    }
    ctx->pending.clear();
    return MOE_OK;
}

bool shared_separate(const moe_ctx *ctx) {
    return ctx->dims.has_shared && ctx->slay.fmt != ctx->lay.fmt;
}
// This context computes the shared expert (with expert parallelism: rank 0 only).
bool shared_here(const moe_ctx *ctx) { return ctx->dims.has_shared && ctx->ep_rank == 0; }

GemvArgs gemv_args(moe_ctx *ctx, int layer, int T, int mode, int only_job, int combine = 0) {
    const moe_dims &D = ctx->dims;
    GemvArgs g{};
    g.mode = mode;
    g.jobs = ctx->dws.jobs;
    g.n_jobs = ctx->dws.n_jobs;
    g.rowrefs = ctx->dws.rowrefs;
    g.only_job = only_job;
    // the shared expert is an item of the routed launches when it has their
    // format; a BF16 shared expert runs in its own launches (its partial is
    // still summed by the combine: shared_rec non-null)
    g.shared_slot = (only_job < 0 && shared_here(ctx) && !shared_separate(ctx)) ? max_jobs(&D, T) : -1;
    g.arena = ctx->arena;
    g.rec_bytes = ctx->lay.bytes;
    g.shared_rec = shared_here(ctx) ? ctx->shared_recs + (int64_t)layer * ctx->slay.bytes : nullptr;
    g.T = T;
    g.k = D.k;
    g.d = D.d;
    g.F = D.F;
    g.lay = ctx->lay;
    g.act = mode == kGateUp ? ctx->dws.xh : ctx->dws.hh;
    g.hh_out = ctx->dws.hh;
    g.part_out = ctx->dws.part;
    g.page = ctx->page_d;
    g.combine = combine;
    g.n_misses = ctx->dws.n_misses;
    g.gates = ctx->dws.gates;
    g.y = nullptr;
    g.tile_ticket = ctx->dws.ticket2;
    g.idx = ctx->dws.idx;
    g.ep_rank = ctx->ep_rank;
    g.ep_size = ctx->ep_size;
    return g;
}

// Arguments of a streaming-kernel launch (expert_stream.cu): phase 1 gate/up,
// 2 down, 3 both (the hit experts); only_job >= 0: that miss alone (phase 3:
// its record has landed whole).
GemvArgs stream_args(moe_ctx *ctx, int layer, int T, int phase, int only_job, int combine) {
    GemvArgs g = gemv_args(ctx, layer, T, phase == 2 ? kDown : kGateUp, only_job, combine);
    g.act = ctx->dws.xh;
    g.phase = phase;
    g.shared_item = (only_job < 0 && shared_here(ctx) && !shared_separate(ctx)) ? 1 : 0;
    g.shared_part = shared_here(ctx) ? 1 : 0;
    g.done = ctx->dws.st_done;
    g.exit_ticket = ctx->dws.st_exit;
    g.wait_ns = (unsigned long long)(std::min(ctx->wait_limit, 5.0) * 1e9);
    if (ctx->inj_stream_skip > 0) {
        g.inj_skip = 1;
        --ctx->inj_stream_skip;
    }
    if (phase == 3 && only_job < 0 && ctx->trace_arm > 0 && ctx->trace_d) {
        if (cudaMemsetAsync(ctx->trace_d, 0, sizeof(unsigned long long) * kTraceCtas * kTraceSlots, ctx->cs) ==
            cudaSuccess)
            g.trace = ctx->trace_d;
        --ctx->trace_arm;
    }
    return g;
}

double w13_bytes(const moe_ctx *c) {
    return (double)(c->lay.w2_codes - c->lay.w13_codes) + (c->lay.tscales >= 0 ? 8.0 : 0.0);
}
double w2_bytes(const moe_ctx *c) {
    return (double)(c->lay.bytes - c->lay.w2_codes) + (c->lay.tscales >= 0 ? 4.0 : 0.0);
}

// A kernel reported a failed self-check through the mapped page (error word
// and a diagnostic record: check code, kernel mode, block, tile, sizes).
moe_status device_error(moe_ctx *ctx) {
    const volatile int32_t *dg = ctx->page_h->diag;
    char buf[256];
    snprintf(buf, sizeof buf, "device check %d failed: kernel mode %d, block (%d,%d), tile %d, sizes %d %d",
             (int)ctx->page_h->error, dg[1], dg[2], dg[3], dg[4], dg[5], dg[6]);
    ctx->err = buf;
    ctx->state = MOE_ERR_STATE;
    return MOE_ERR_CUDA;
}

// Bounded host wait for the device's miss list (sequence number `seq`).
moe_status wait_miss_list(moe_ctx *ctx, uint32_t seq) {
    const auto t0 = std::chrono::steady_clock::now();
    struct Account {  // time spent here, and the start of the issue phase that follows
        moe_ctx *c;
        std::chrono::steady_clock::time_point a;
        ~Account() {
            const auto now = std::chrono::steady_clock::now();
            c->stats.host_us[1] += std::chrono::duration<double, std::micro>(now - a).count();
            c->issue_t0 = now;
        }
    } account{ctx, t0};
    uint64_t spins = 0;
    while (ctx->page_h->seq != seq) {
        _mm_pause();
        if ((++spins & 4095) == 0) {
            const double el = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
            if (el > ctx->wait_limit) {
                ctx->state = MOE_ERR_STATE;
                ctx->err = "timed out waiting for the device miss list";
                return MOE_ERR_TIMEOUT;
            }
        }
    }
    std::atomic_thread_fence(std::memory_order_acquire);
    return MOE_OK;
}

void fill_trace(moe_ctx *ctx, int32_t layer, int nrouted, int nev, moe_layer_trace *trace) {
    if (!trace) return;
    const HostEvent *ev = ctx->page_h->ev;
    trace->count = nev;
    const int n = nev < trace->capacity ? nev : trace->capacity;
    for (int j = 0; j < n && trace->events; ++j) {
        moe_cache_event &o = trace->events[j];
        o.layer = j < nrouted ? layer : layer + 1;
        o.expert = ev[j].expert;
        o.slot = ev[j].slot;
        o.hit = ev[j].flags & 1;
        o.evicted_key = ev[j].evicted;
        o.prefetch = (ev[j].flags >> 1) & 1;
        o.reserved = 0;
    }
}

// Counters and trace of a decode call whose miss list (nev entries) is in the page.
moe_status finish_decode(moe_ctx *ctx, int32_t layer, int32_t T, int nev, moe_layer_trace *trace) {
    const HostEvent *ev = ctx->page_h->ev;
    int64_t hits = 0, evictions = 0;
    for (int j = 0; j < nev; ++j) {
        hits += ev[j].flags & 1;
        evictions += ev[j].evicted >= 0;
    }
    for (int i = 0; i < 8; ++i) ctx->stats.route_phase_us[i] += ctx->page_h->phase_ns[i] * 1e-3;
    ctx->stats.lookups += nev;
    ctx->stats.hits += hits;
    ctx->stats.misses += nev - hits;
    ctx->stats.evictions += evictions;
    ctx->stats.forward_calls += 1;
    ctx->stats.host_us[2] +=
        std::chrono::duration<double, std::micro>(std::chrono::steady_clock::now() - ctx->issue_t0).count();
    fill_trace(ctx, layer, nev, nev, trace);
    ctx->last_T = T;
    return MOE_OK;
}

moe_status forward_decode(moe_ctx *ctx, int32_t layer, const void *x, int32_t T, float *y,
                          moe_layer_trace *trace) {
    const moe_dims &D = ctx->dims;
    if (ctx->page_h->error) return device_error(ctx);
    const uint32_t seq = ++ctx->seq;
    RouteArgs ra{};
    ra.Wr = ctx->router_w + (size_t)layer * D.E * D.d;
    ra.Wr_next = layer + 1 < D.L ? ra.Wr + (size_t)D.E * D.d : nullptr;
    ra.L = D.L;
    ra.prefetch = 0;
    ra.x = static_cast<const __nv_bfloat16 *>(x);
    ra.T = T;
    ra.E = D.E;
    ra.d = D.d;
    ra.k = D.k;
    ra.renorm = D.renormalize;
    ra.layer = layer;
    ra.ws = ctx->dws;
    ra.tab = ctx->tab;
    ra.page = ctx->page_d;
    ra.seq = seq;
    ra.publish = 1;
    ra.ep_rank = ctx->ep_rank;
    ra.ep_size = ctx->ep_size;
    if (ctx->inj_drop_publish > 0) {
        ra.publish = 0;
        --ctx->inj_drop_publish;
    }
    if (ctx->pf_pending[layer]) {  // experts prefetched for this layer by a prefill call
        CK(cudaStreamWaitEvent(ctx->cs, ctx->ev_pf[layer], 0));
        ctx->pf_pending[layer] = 0;
    }
    TimedLaunch tl;
    time_begin(ctx, tl, MOE_K_ROUTE);
    ra.span = time_span(ctx, tl);
    CK(launch_route_lookup(ra, ctx->cs));
    time_end(ctx, tl, (double)D.E * D.d * 2 + (double)T * D.d * 2);

    const int nj = max_jobs(&D, T);
    if (shared_separate(ctx) && shared_here(ctx)) {  // BF16 shared expert: its own two launches
        TimedLaunch sg, sd;
        const uint8_t *rec = ctx->shared_recs + (int64_t)layer * ctx->slay.bytes;
        const int64_t sel0 = D.k, sel_stride = D.k + 1;  // selection p = k of row t
        time_begin(ctx, sg, MOE_K_GATEUP);
        CK(launch_shared_bf16(kGateUp, rec, D.d, D.F, T, ctx->dws.xh, ctx->dws.hh, ctx->dws.part, sel0, sel_stride,
                              ctx->cs));
        time_end(ctx, sg, 2.0 * 2 * D.F * D.d + (double)T * D.d * 2);
        time_begin(ctx, sd, MOE_K_DOWN);
        CK(launch_shared_bf16(kDown, rec, D.d, D.F, T, ctx->dws.xh, ctx->dws.hh, ctx->dws.part, sel0, sel_stride,
                              ctx->cs));
        time_end(ctx, sd, 2.0 * D.d * D.F + (double)T * D.F * 4);
    }
    const int in_launch_shared = (shared_here(ctx) && !shared_separate(ctx)) ? 1 : 0;
    if (ctx->fused) {
        // one launch for every expert GEMV of the layer: the hit and shared
        // experts at once, each miss when the copy stream flags its halves
        LayerArgs la{};
        la.jobs = ctx->dws.jobs;
        la.n_jobs = ctx->dws.n_jobs;
        la.rowrefs = ctx->dws.rowrefs;
        la.arena = ctx->arena;
        la.rec_bytes = ctx->lay.bytes;
        la.shared_rec = shared_here(ctx) ? ctx->shared_recs + (int64_t)layer * ctx->slay.bytes : nullptr;
        la.shared_item = in_launch_shared;
        la.T = T;
        la.k = D.k;
        la.d = D.d;
        la.F = D.F;
        la.lay = ctx->lay;
        la.xh = ctx->dws.xh;
        la.hh = ctx->dws.hh;
        la.part = ctx->dws.part;
        la.gates = ctx->dws.gates;
        la.y = y;
        la.tile_ticket = ctx->dws.ticket2;
        la.done_a = ctx->dws.lk_done_a;
        la.queue = ctx->dws.lk_queue;
        la.miss_flag = ctx->dws.lk_flags;
        la.release = ctx->dws.lk_release;
        la.seq = seq;
        la.wait_ns = (unsigned long long)(std::min(ctx->wait_limit, 5.0) * 1e9);
        la.page = ctx->page_d;
        la.idx = ctx->dws.idx;
        la.ep_rank = ctx->ep_rank;
        la.ep_size = ctx->ep_size;
        TimedLaunch tk, th;
        time_begin(ctx, tk, MOE_K_LAYER);
        la.span = time_span(ctx, tk);
        time_begin(ctx, th, MOE_K_LAYER_HITS);
        la.span_hit = time_span(ctx, th);
        CK(launch_expert_layer(la, ctx->cs));
        const long ik = time_end(ctx, tk, 0);
        const long ih = time_end(ctx, th, 0);
        // every way out before the last flag is written releases the kernel's waits
        struct Release {
            moe_ctx *c;
            uint32_t seq;
            bool armed = true;
            ~Release() {
                if (armed) stream_write(c->xs, c->dws.lk_release, seq);
            }
        } rel{ctx, seq};
        {
            const moe_status ws_ = wait_miss_list(ctx, seq);
            if (ws_ != MOE_OK) return ws_;
        }
        if (ctx->page_h->error) return device_error(ctx);
        const int nev = ctx->page_h->n_events;
        const HostEvent *ev = ctx->page_h->ev;
        int n_hit_jobs = 0;
        for (int j = 0; j < nev; ++j) n_hit_jobs += ev[j].flags & 1;
        const double rec = w13_bytes(ctx) + w2_bytes(ctx);
        if (ik >= 0) ctx->pending[ik].bytes = (nev + in_launch_shared) * rec + (double)T * D.d * 2;
        if (ih >= 0) ctx->pending[ih].bytes = (n_hit_jobs + in_launch_shared) * rec + (double)T * D.d * 2;
        // misses: the gate/up prefix, its flag, the W2 half, its flag
        const int64_t split = ctx->lay.w2_codes;
        int mo = 0;
        bool used2 = false;
        for (int j = 0; j < nev; ++j) {
            if (ev[j].flags & 1) continue;
            if (ctx->inj_copy_fail_at > 0 && --ctx->inj_copy_fail_at == 0) {
                ctx->state = MOE_ERR_STATE;
                ctx->err = "injected failure of an H2D copy issue";
                return MOE_ERR_CUDA;
            }
            const int64_t rec_idx = ((int64_t)layer * D.E + ev[j].expert) % ctx->P;
            uint8_t *dst = ctx->arena + (int64_t)ev[j].slot * ctx->lay.bytes;
            const uint8_t *src = ctx->pool + rec_idx * ctx->lay.bytes;
            const bool flags = !(ctx->inj_drop_flags > 0 && (--ctx->inj_drop_flags, true));
            cudaStream_t s;
            CK(miss_stream(ctx, mo++, &used2, &s));
            CK(cudaMemcpyAsync(dst, src, split, cudaMemcpyHostToDevice, s));
            if (flags) CK(stream_write(s, ctx->dws.lk_flags + 2 * j, seq));
            CK(cudaMemcpyAsync(dst + split, src + split, ctx->lay.bytes - split, cudaMemcpyHostToDevice, s));
            if (flags) CK(stream_write(s, ctx->dws.lk_flags + 2 * j + 1, seq));
            else rel.armed = false;  // injected: the kernel's own wait limit must end it
            ctx->stats.h2d_copies += 1;
            ctx->stats.h2d_bytes += ctx->lay.bytes;
        }
        if (mo > 0) CK(copy_tail(ctx, used2));
        rel.armed = false;
        return finish_decode(ctx, layer, T, nev, trace);
    }

    // hit experts and the shared expert, before the miss list is known
    const int grid_y = nj + in_launch_shared;
    const bool stream = ctx->gemv_kind == 1;
    long ig = -1, id = -1, ih = -1;
    if (stream) {  // one launch: their gate/up tiles, then their down tiles (+ combine if nothing missed)
        TimedLaunch th;
        time_begin(ctx, th, MOE_K_LAYER_HITS);
        GemvArgs ha = stream_args(ctx, layer, T, 3, -1, 2);
        ha.y = y;
        if (ctx->head_bytes && ctx->pool_d && !(ctx->flags & MOE_CACHE_STATIC_SPLIT)) {
            ha.pool_d = ctx->pool_d;
            ha.pool_P = ctx->P;
            ha.layer = layer;
            ha.E = D.E;
            ha.head_bytes = ctx->head_bytes;
        }
        ha.span = time_span(ctx, th);
        CK(launch_stream(ha, grid_y, ctx->cs));
        ih = time_end(ctx, th, 0);
    } else {
        TimedLaunch tg, td;
        time_begin(ctx, tg, MOE_K_GATEUP);
        GemvArgs hg = gemv_args(ctx, layer, T, kGateUp, -1);
        hg.span = time_span(ctx, tg);
        CK(launch_gemv(hg, grid_y, ctx->cs));
        ig = time_end(ctx, tg, 0);
        time_begin(ctx, td, MOE_K_DOWN);
        GemvArgs hd = gemv_args(ctx, layer, T, kDown, -1, 2);  // combines when nothing missed
        hd.y = y;
        hd.span = time_span(ctx, td);
        CK(launch_gemv(hd, grid_y, ctx->cs));
        id = time_end(ctx, td, 0);
    }

    // bounded host wait for the device's miss list
    {
        const moe_status ws_ = wait_miss_list(ctx, seq);
        if (ws_ != MOE_OK) return ws_;
    }
    if (ctx->page_h->error) return device_error(ctx);
    const int nev = ctx->page_h->n_events;
    const HostEvent *ev = ctx->page_h->ev;
    int n_hit_jobs = 0, last_miss = -1;
    for (int j = 0; j < nev; ++j) {
        n_hit_jobs += ev[j].flags & 1;
        if (!(ev[j].flags & 1)) last_miss = j;
    }
    {  // algorithmic bytes of the hit launches, now known
        const int nexp = n_hit_jobs + in_launch_shared;
        if (ig >= 0) ctx->pending[ig].bytes = nexp * w13_bytes(ctx) + (double)T * D.d * 2;
        if (id >= 0) ctx->pending[id].bytes = nexp * w2_bytes(ctx) + (double)T * D.F * 4;
        if (ih >= 0) ctx->pending[ih].bytes = nexp * (w13_bytes(ctx) + w2_bytes(ctx)) + (double)T * D.d * 2;
    }

    // misses: each record in one copy on the copy stream, an event after it;
    // or (split_copies) in two -- the gate/up half (tensor scales + W13, a
    // prefix of the record) and the down half -- with an event after each, so a
    // miss's gate/up runs while its down half streams in
    const int64_t split = ctx->lay.w2_codes;
    // the first miss's head came over with the SMs of the hit launch
    const bool stream_head = stream && ctx->head_bytes && ctx->pool_d && !(ctx->flags & MOE_CACHE_STATIC_SPLIT);
    int mo = 0;
    bool used2 = false;
    for (int j = 0; j < nev; ++j) {
        if (ev[j].flags & 1) continue;
        if (ctx->inj_copy_fail_at > 0 && --ctx->inj_copy_fail_at == 0) {
            ctx->state = MOE_ERR_STATE;
            ctx->err = "injected failure of an H2D copy issue";
            return MOE_ERR_CUDA;
        }
        const int64_t rec_idx = ((int64_t)layer * D.E + ev[j].expert) % ctx->P;
        uint8_t *dst = ctx->arena + (int64_t)ev[j].slot * ctx->lay.bytes;
        const uint8_t *src = ctx->pool + rec_idx * ctx->lay.bytes;
        const int64_t head = (stream_head && mo == 0) ? (int64_t)ctx->head_bytes : 0;
        cudaStream_t s;
        CK(miss_stream(ctx, mo++, &used2, &s));
        if (!ctx->split_copies) {  // one copy, one event (both halves)
            CK(cudaMemcpyAsync(dst + head, src + head, ctx->lay.bytes - head, cudaMemcpyHostToDevice, s));
            CK(cudaEventRecord(ctx->miss_ev[2 * j], s));
        } else {
            if (head < split) CK(cudaMemcpyAsync(dst + head, src + head, split - head, cudaMemcpyHostToDevice, s));
            CK(cudaEventRecord(ctx->miss_ev[2 * j], s));
            const int64_t w2 = head > split ? head : split;
            CK(cudaMemcpyAsync(dst + w2, src + w2, ctx->lay.bytes - w2, cudaMemcpyHostToDevice, s));
            CK(cudaEventRecord(ctx->miss_ev[2 * j + 1], s));
        }
        ctx->stats.h2d_copies += 1;
        ctx->stats.h2d_bytes += ctx->lay.bytes;
    }
    if (mo > 0) CK(copy_tail(ctx, used2));
    for (int j = 0; j < nev; ++j) {
        if (ev[j].flags & 1) continue;
        CK(cudaStreamWaitEvent(ctx->cs, ctx->miss_ev[2 * j], 0));
        const int comb = j == last_miss ? 1 : 0;
        if (stream && !ctx->split_copies) {  // the whole record is in: one launch, gate/up then down
            TimedLaunch mm;
            time_begin(ctx, mm, MOE_K_MISS);
            GemvArgs ma = stream_args(ctx, layer, T, 3, j, comb);
            ma.y = y;
            ma.span = time_span(ctx, mm);
            CK(launch_stream(ma, 1, ctx->cs));
            time_end(ctx, mm, w13_bytes(ctx) + w2_bytes(ctx) + (double)T * D.d * 2);
            continue;
        }
        TimedLaunch mg, md;
        time_begin(ctx, mg, MOE_K_GATEUP);
        GemvArgs mg_args = stream ? stream_args(ctx, layer, T, 1, j, 0) : gemv_args(ctx, layer, T, kGateUp, j);
        mg_args.span = time_span(ctx, mg);
        CK(stream ? launch_stream(mg_args, 1, ctx->cs) : launch_gemv(mg_args, 1, ctx->cs));
        time_end(ctx, mg, w13_bytes(ctx) + (double)T * D.d * 2);
        if (ctx->split_copies) CK(cudaStreamWaitEvent(ctx->cs, ctx->miss_ev[2 * j + 1], 0));
        time_begin(ctx, md, MOE_K_DOWN);
        GemvArgs md_args = stream ? stream_args(ctx, layer, T, 2, j, comb) : gemv_args(ctx, layer, T, kDown, j, comb);
        md_args.y = y;
        md_args.span = time_span(ctx, md);
        CK(stream ? launch_stream(md_args, 1, ctx->cs) : launch_gemv(md_args, 1, ctx->cs));
        time_end(ctx, md, w2_bytes(ctx) + (double)T * D.F * 4);
    }

    return finish_decode(ctx, layer, T, nev, trace);
}

// One layer of a prefill chunk (T > 32 rows): W4A4 grouped tensor-core GEMMs,
// with the next layer's experts prefetched when MOE_CACHE_PREFETCH_NEXT is set.
moe_status forward_prefill(moe_ctx *ctx, int32_t layer, const void *x, int32_t T, float *y,
                           moe_layer_trace *trace) {
    const moe_dims &D = ctx->dims;
    if (ctx->page_h->error) return device_error(ctx);
    const uint32_t seq = ++ctx->seq;
    RouteArgs ra{};
    ra.Wr = ctx->router_w + (size_t)layer * D.E * D.d;
    ra.Wr_next = nullptr;
    ra.L = D.L;
    ra.prefetch = (ctx->flags & MOE_CACHE_PREFETCH_NEXT) ? 1 : 0;
    ra.x = static_cast<const __nv_bfloat16 *>(x);
    ra.T = T;
    ra.E = D.E;
    ra.d = D.d;
    ra.k = D.k;
    ra.renorm = D.renormalize;
    ra.layer = layer;
    ra.ws = ctx->dws;
    ra.tab = ctx->tab;
    ra.page = ctx->page_d;
    ra.seq = seq;
    ra.publish = 1;
    ra.ep_rank = ctx->ep_rank;
    ra.ep_size = ctx->ep_size;
    if (ctx->inj_drop_publish > 0) {
        ra.publish = 0;
        --ctx->inj_drop_publish;
    }
    // the shared expert is a job of the grouped GEMMs when it has the routed
    // format; a BF16 one runs as two bf16 GEMMs of its own
    const bool sep = shared_separate(ctx) && shared_here(ctx);
    const int grouped_shared = (shared_here(ctx) && !shared_separate(ctx)) ? 1 : 0;
    const bool mx = ctx->lay.fmt == kFmtMxfp4;
    CK(cudaMemsetAsync(ctx->dws.cnt, 0, (size_t)D.E * 4, ctx->cs));
    TimedLaunch tr;
    time_begin(ctx, tr, MOE_K_PREFILL_ROUTE);
    CUtensorMap tm_x;  // logits on the tensor cores when x's rows can be TMA boxes
    const bool x_map = make_operand_map(&tm_x, x, 2 * (int64_t)D.d, T, 0, 0);
    if (sep && !x_map) return MOE_ERR_UNSUPPORTED;  // (x is 16-byte aligned and d a multiple of 64: not reached)
    if (x_map) {
        CK(launch_router_gemm(tm_x, ctx->maps.router, ctx->dws.z, T, D.E, D.d, layer, ctx->page_d, ctx->cs));
        CK(launch_prefill_select(ra, ctx->cs));
    } else {
        CK(launch_prefill_route(ra, ctx->cs));
    }
    time_end(ctx, tr, (double)D.E * D.d * 2 + (double)T * D.d * 2);
    CK(launch_prefill_scatter(ra, ctx->cs));
    CK(launch_tile_plan(ctx->dws.jobs, ctx->dws.n_jobs, T, grouped_shared, ctx->dws.pairs, ctx->dws.n_pairs,
                        ctx->cs));
    CK(launch_quant_x_grouped(ra.x, T, D.k, D.d, grouped_shared, ctx->dws.rowrefs, ctx->dws.n_grouped, ctx->dws.xq,
                              ctx->dws.xq_scales, ctx->dws.xq_st, mx ? 1 : 0, ctx->cs));

    const moe_status ws_ = wait_miss_list(ctx, seq);
    if (ws_ != MOE_OK) return ws_;
    if (ctx->page_h->error) return device_error(ctx);
    const int nev = ctx->page_h->n_events, n = ctx->page_h->n_jobs;
    const HostEvent *ev = ctx->page_h->ev;

    // copies on the copy stream: this layer's misses (the layer's compute waits
    // for them), then the next layer's prefetch misses (its compute waits)
    // Records whose pool indices and slots are both consecutive (a cold cache
    // hands out free slots in ascending order, and entries come in ascending
    // expert order) go in one copy.
    int64_t run_src = -1, run_dst = -1, run_n = 0;
    auto flush_run = [&]() -> moe_status {
        if (run_n == 0) return MOE_OK;
        if (ctx->inj_copy_fail_at > 0 && --ctx->inj_copy_fail_at == 0) {
            ctx->state = MOE_ERR_STATE;
            ctx->err = "injected failure of an H2D copy issue";
            return MOE_ERR_CUDA;
        }
        CK(cudaMemcpyAsync(ctx->arena + run_dst * ctx->lay.bytes, ctx->pool + run_src * ctx->lay.bytes,
                           run_n * ctx->lay.bytes, cudaMemcpyHostToDevice, ctx->xs));
        ctx->stats.h2d_copies += 1;
        ctx->stats.h2d_bytes += run_n * ctx->lay.bytes;
        run_n = 0;
        return MOE_OK;
    };
    auto copy_record = [&](int lyr, const HostEvent &e) -> moe_status {
        const int64_t rec_idx = ((int64_t)lyr * D.E + e.expert) % ctx->P;
        if (run_n > 0 && rec_idx == run_src + run_n && e.slot == run_dst + run_n) {
            ++run_n;
            return MOE_OK;
        }
        const moe_status st = flush_run();
        if (st != MOE_OK) return st;
        run_src = rec_idx;
        run_dst = e.slot;
        run_n = 1;
        return MOE_OK;
    };
    int nrm = 0, npm = 0;
    for (int j = 0; j < n; ++j) {
        if (ev[j].flags & 1) continue;
        const moe_status st = copy_record(layer, ev[j]);
        if (st != MOE_OK) return st;
        ++nrm;
    }
    if (nrm > 0) {
        const moe_status st = flush_run();
        if (st != MOE_OK) return st;
        CK(cudaEventRecord(ctx->ev_routed, ctx->xs));
        CK(cudaStreamWaitEvent(ctx->cs, ctx->ev_routed, 0));
    }
    if (ctx->pf_pending[layer]) {  // experts prefetched for this layer by the previous call
        CK(cudaStreamWaitEvent(ctx->cs, ctx->ev_pf[layer], 0));
        ctx->pf_pending[layer] = 0;
    }
    for (int j = n; j < nev; ++j) {
        if (ev[j].flags & 1) continue;
        const moe_status st = copy_record(layer + 1, ev[j]);
        if (st != MOE_OK) return st;
        ++npm;
    }
    if (npm > 0) {
        const moe_status st = flush_run();
        if (st != MOE_OK) return st;
        CK(cudaEventRecord(ctx->ev_pf[layer + 1], ctx->xs));
        ctx->pf_pending[layer + 1] = 1;
    }
    if (nrm + npm > 0) CK(copy_tail(ctx, false));

    // experts: grouped tensor-core GEMMs -- gate/up (+SwiGLU, fp32 h), h
    // quantized per row, down -- then the gate-weighted combine
    const int grid_y = n + grouped_shared;
    const int cap = grouped_pairs_cap(n, T, D.k, grouped_shared);
    GroupedGemmArgs gu{};
    gu.mode = kGateUp;
    gu.jobs = ctx->dws.jobs;
    gu.n_jobs = ctx->dws.n_jobs;
    gu.pairs = ctx->dws.pairs;
    gu.n_pairs = ctx->dws.n_pairs;
    gu.m_tiles = (2 * D.F + 127) / 128;
    gu.layer = layer;
    gu.T = T;
    gu.k = D.k;
    gu.d = D.d;
    gu.F = D.F;
    gu.arena = ctx->arena;
    gu.rec_bytes = ctx->lay.bytes;
    gu.shared_rec = grouped_shared ? ctx->shared_recs : nullptr;
    gu.lay = ctx->lay;
    gu.act_scales = ctx->dws.xq_scales;
    gu.act_st = ctx->dws.xq_st;
    gu.rowrefs = ctx->dws.rowrefs;
    gu.h32 = ctx->dws.h32;
    gu.part = ctx->dws.part;
    gu.page = ctx->page_d;
    gu.wait_ns = (unsigned long long)(std::min(ctx->wait_limit, 4.0) * 1e9);
    gu.inj_skip = 0;
    if (ctx->inj_gemm_skip > 0) {
        --ctx->inj_gemm_skip;
        gu.inj_skip = 1;
    }
    TimedLaunch tg;
    time_begin(ctx, tg, MOE_K_PREFILL_GATEUP);
    gu.span = time_span(ctx, tg);
    CK(launch_grouped_gemm(ctx->maps, gu, cap, ctx->cs));
    time_end(ctx, tg, grid_y * w13_bytes(ctx));
    CK(launch_quant_h_grouped(ctx->dws.h32, T, D.k, grouped_shared, ctx->dws.n_grouped, D.F, ctx->dws.hq,
                              ctx->dws.hq_scales, ctx->dws.hq_st, mx ? 1 : 0, ctx->cs));
    GroupedGemmArgs dn = gu;
    dn.inj_skip = 0;
    dn.mode = kDown;
    dn.m_tiles = (D.d + 127) / 128;
    dn.act_scales = ctx->dws.hq_scales;
    dn.act_st = ctx->dws.hq_st;
    TimedLaunch td;
    time_begin(ctx, td, MOE_K_PREFILL_DOWN);
    dn.span = time_span(ctx, td);
    CK(launch_grouped_gemm(ctx->maps, dn, cap, ctx->cs));
    time_end(ctx, td, grid_y * w2_bytes(ctx));
    if (sep) {  // BF16 shared expert: [g u] = x W13^T, h = silu(g) u as bf16 (hi, lo), W2 h into part[t][k]
        TimedLaunch sg_t, sd_t;
        time_begin(ctx, sg_t, MOE_K_PREFILL_GATEUP);
        CK(launch_bf16_gemm(tm_x, ctx->maps.w13_sbf, ctx->dws_sg, 2 * (int64_t)D.F, T, 2 * D.F, 2 * D.d, 0, layer,
                            ctx->page_d, ctx->cs));
        time_end(ctx, sg_t, 2.0 * 2 * D.F * D.d + (double)T * D.d * 2);
        CK(launch_swiglu_split(ctx->dws_sg, T, D.F, ctx->dws_hs, ctx->cs));
        time_begin(ctx, sd_t, MOE_K_PREFILL_DOWN);
        CK(launch_bf16_gemm(ctx->maps.hs, ctx->maps.w2_sbf, ctx->dws.part + (int64_t)D.k * D.d,
                            (int64_t)(D.k + 1) * D.d, T, D.d, 4 * D.F, 2 * D.F, layer, ctx->page_d, ctx->cs));
        time_end(ctx, sd_t, 2.0 * D.d * D.F + (double)T * D.F * 4);
    }
    CK(launch_combine(ctx->dws.part, ctx->dws.gates, ctx->dws.idx, ctx->ep_rank, ctx->ep_size, y, T, D.k, D.d,
                      shared_here(ctx) ? 1 : 0, ctx->cs));

    int64_t hits = 0, evictions = 0, pf_evict = 0;
    for (int j = 0; j < n; ++j) {  // (npm: prefetch misses counted above)
        hits += ev[j].flags & 1;
        evictions += ev[j].evicted >= 0;
    }
    for (int j = n; j < nev; ++j) pf_evict += ev[j].evicted >= 0;
    ctx->stats.lookups += n;
    ctx->stats.hits += hits;
    ctx->stats.misses += n - hits;
    ctx->stats.evictions += evictions + pf_evict;
    ctx->stats.prefetch_lookups += nev - n;
    ctx->stats.prefetch_misses += npm;
    ctx->stats.forward_calls += 1;
    ctx->stats.host_us[2] +=
        std::chrono::duration<double, std::micro>(std::chrono::steady_clock::now() - ctx->issue_t0).count();
    fill_trace(ctx, layer, n, nev, trace);
    ctx->last_T = T;
    return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_record_bytes(const moe_dims *dims) {
    if (!dims_valid(dims)) return 0;
    return (size_t)layout_of(dims).bytes;
}

size_t moe_shared_record_bytes(const moe_dims *dims) {
    if (!dims_valid(dims)) return 0;
    return (size_t)shared_layout_of(dims).bytes;
}

moe_status moe_record_layout(const moe_dims *dims, int64_t off[6]) {
    if (!dims_valid(dims) || !off) return MOE_ERR_ARG;
    RecordLayout r = layout_of(dims);
    off[0] = r.w13_codes; off[1] = r.w13_scales; off[2] = r.w2_codes;
    off[3] = r.w2_scales; off[4] = r.tscales; off[5] = r.bytes;
    return MOE_OK;
}

size_t moe_workspace_bytes(const moe_dims *dims) {
    if (!dims_valid(dims)) return 0;
    return (size_t)ws_layout(dims).total;
}

size_t moe_arena_bytes(const moe_dims *dims, int64_t num_slots) {
    if (!dims_valid(dims) || num_slots <= 0) return 0;
    return (size_t)(up256(num_slots * layout_of(dims).bytes) + table_layout(dims, num_slots).total);
}

moe_status moe_layer_init(const moe_dims *dims, const void *host_pool, size_t host_pool_bytes,
                          const void *router_w, const void *shared_recs, void *workspace,
                          size_t workspace_bytes, void *compute_stream, void *copy_stream,
                          moe_ctx **out) {
    if (!out) return MOE_ERR_ARG;
    *out = nullptr;
    if (!dims_valid(dims) || !host_pool || !router_w || !workspace || !compute_stream ||
        !copy_stream || (dims->has_shared && !shared_recs))
        return MOE_ERR_ARG;
    if (!dims_supported(dims)) return MOE_ERR_UNSUPPORTED;
    const RecordLayout lay = layout_of(dims);
    const int64_t P = dims->pool_records ? dims->pool_records : (int64_t)dims->L * dims->E;
    if (P > (int64_t)dims->L * dims->E) return MOE_ERR_ARG;
    if ((int64_t)host_pool_bytes < P * lay.bytes) return MOE_ERR_ARG;
    if (workspace_bytes < moe_workspace_bytes(dims)) return MOE_ERR_ARG;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, host_pool) != cudaSuccess || attr.type != cudaMemoryTypeHost) {
        cudaGetLastError();
        return MOE_ERR_NOT_PINNED;
    }
    moe_ctx *ctx = new moe_ctx();
    ctx->dims = *dims;
    ctx->lay = lay;
    ctx->slay = shared_layout_of(dims);
    ctx->P = P;
    ctx->pool = static_cast<const uint8_t *>(host_pool);
    {  // the pool's device address (SM reads of the first miss's head); none: the option stays off
        void *pd = nullptr;
        if (cudaHostGetDevicePointer(&pd, const_cast<void *>(host_pool), 0) == cudaSuccess)
            ctx->pool_d = static_cast<const uint8_t *>(pd);
        cudaGetLastError();
    }
    ctx->router_w = static_cast<const __nv_bfloat16 *>(router_w);
    ctx->shared_recs = static_cast<const uint8_t *>(shared_recs);
    ctx->ws = static_cast<uint8_t *>(workspace);
    ctx->wl = ws_layout(dims);
    ctx->cs = static_cast<cudaStream_t>(compute_stream);
    ctx->xs = static_cast<cudaStream_t>(copy_stream);
    memset(&ctx->stats, 0, sizeof ctx->stats);
    uint8_t *w = ctx->ws;
    const WsLayout &L = ctx->wl;
    ctx->dws.z = reinterpret_cast<float *>(w + L.z);
    ctx->dws.idx = reinterpret_cast<int32_t *>(w + L.idx);
    ctx->dws.gates = reinterpret_cast<float *>(w + L.gates);
    ctx->dws.jobs = reinterpret_cast<Job *>(w + L.jobs);
    ctx->dws.n_jobs = reinterpret_cast<int32_t *>(w + L.n_jobs);
    ctx->dws.n_misses = reinterpret_cast<int32_t *>(w + L.n_misses);
    ctx->dws.ticket = reinterpret_cast<uint32_t *>(w + L.ticket);
    ctx->dws.ticket2 = reinterpret_cast<uint32_t *>(w + L.ticket2);
    ctx->dws.lk_queue = reinterpret_cast<uint32_t *>(w + L.lk);
    ctx->dws.lk_release = ctx->dws.lk_queue + 2;
    ctx->dws.lk_done_a = ctx->dws.lk_queue + 4;
    ctx->dws.lk_flags = ctx->dws.lk_done_a + kMaxSlots;
    ctx->dws.st_done = ctx->dws.lk_flags + 2 * kMaxSlots;
    ctx->dws.st_exit = ctx->dws.st_done + kMaxSlots;
    ctx->dws.rowrefs = reinterpret_cast<RowRef *>(w + L.rowrefs);
    ctx->dws.xh = reinterpret_cast<__half *>(w + L.xh);
    ctx->dws.hh = reinterpret_cast<__half *>(w + L.hh);
    ctx->dws.part = reinterpret_cast<float *>(w + L.part);
    ctx->dws.cnt = L.cnt >= 0 ? reinterpret_cast<int32_t *>(w + L.cnt) : nullptr;
    ctx->dws.fill = L.fill >= 0 ? reinterpret_cast<int32_t *>(w + L.fill) : nullptr;
    ctx->dws.jobidx = L.jobidx >= 0 ? reinterpret_cast<int32_t *>(w + L.jobidx) : nullptr;
    ctx->dws.h32 = L.h32 >= 0 ? reinterpret_cast<float *>(w + L.h32) : nullptr;
    if (L.xq >= 0) {
        ctx->dws.xq = w + L.xq;
        ctx->dws.xq_scales = w + L.xq_scales;
        ctx->dws.xq_st = reinterpret_cast<float *>(w + L.xq_st);
        ctx->dws.hq = w + L.hq;
        ctx->dws.hq_scales = w + L.hq_scales;
        ctx->dws.hq_st = reinterpret_cast<float *>(w + L.hq_st);
        ctx->dws.pairs = reinterpret_cast<int2 *>(w + L.pairs);
        ctx->dws.n_pairs = reinterpret_cast<int32_t *>(w + L.n_pairs);
        ctx->dws.n_grouped = reinterpret_cast<int32_t *>(w + L.n_grouped);
        const int64_t R = (int64_t)dims->max_rows * (dims->k + 1);
        bool ok = make_operand_map(&ctx->maps.xq, ctx->dws.xq, dims->d / 2, R, 0, 0) &&
                  make_operand_map(&ctx->maps.hq, ctx->dws.hq, dims->F / 2, R, 0, 0) &&
                  make_operand_map(&ctx->maps.router, router_w, 2 * (int64_t)dims->d, dims->E, dims->L,
                                   2 * (int64_t)dims->E * dims->d);
        if (ok && dims->has_shared && ctx->slay.fmt == lay.fmt) {  // the shared expert as a grouped-GEMM job
            ok = make_operand_map(&ctx->maps.w13_shared, ctx->shared_recs + lay.w13_codes, dims->d / 2,
                                  2 * dims->F, dims->L, ctx->slay.bytes) &&
                 make_operand_map(&ctx->maps.w2_shared, ctx->shared_recs + lay.w2_codes, dims->F / 2, dims->d,
                                  dims->L, ctx->slay.bytes);
        } else if (ok && dims->has_shared) {  // a BF16 shared expert: two bf16 GEMMs of its own
            ctx->dws_sg = reinterpret_cast<float *>(w + L.sg);
            ctx->dws_hs = reinterpret_cast<uint16_t *>(w + L.hs);
            ok = make_operand_map(&ctx->maps.w13_sbf, ctx->shared_recs + ctx->slay.w13_codes, 2 * (int64_t)dims->d,
                                  2 * dims->F, dims->L, ctx->slay.bytes) &&
                 make_operand_map(&ctx->maps.w2_sbf, ctx->shared_recs + ctx->slay.w2_codes, 2 * (int64_t)dims->F,
                                  dims->d, dims->L, ctx->slay.bytes) &&
                 make_operand_map(&ctx->maps.hs, ctx->dws_hs, 4 * (int64_t)dims->F, dims->max_rows, 0, 0);
        }
        if (!ok) {
            delete ctx;
            return MOE_ERR_UNSUPPORTED;
        }
    }

    ctx->page_cap = 2 * dims->E + 8;
    const size_t page_bytes = sizeof(HostPage) + sizeof(HostEvent) * ctx->page_cap;
    moe_status st = MOE_OK;
    cudaError_t e = cudaHostAlloc(reinterpret_cast<void **>(&ctx->page_h), page_bytes, cudaHostAllocMapped);
    if (e == cudaSuccess) e = cudaHostGetDevicePointer(reinterpret_cast<void **>(&ctx->page_d), ctx->page_h, 0);
    if (e == cudaSuccess) {
        memset((void *)ctx->page_h, 0, page_bytes);
        ctx->miss_ev.resize(2 * ctx->page_cap, nullptr);
        for (auto &ev : ctx->miss_ev) {
            e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
            if (e != cudaSuccess) break;
        }
    }
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ctx->ev_routed, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ctx->ev_xs_tail, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ctx->ev_xs2_tail, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&ctx->xs2, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventRecord(ctx->ev_xs_tail, ctx->xs);
    if (e == cudaSuccess) {
        ctx->ev_pf.resize(dims->L, nullptr);
        ctx->pf_pending.assign(dims->L, 0);
        for (auto &ev : ctx->ev_pf) {
            e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
            if (e != cudaSuccess) break;
        }
    }
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->dws.ticket, 0, 4, ctx->cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->dws.ticket2, 0, 4 * kMaxTiles, ctx->cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->dws.lk_queue, 0, 4 * (size_t)kLkWords, ctx->cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->cs);
    // the persistent layer kernel needs stream memory writes on the copy stream:
    // one trial write (of the value already there) decides
    if (e == cudaSuccess) {
        ctx->fused_ok = stream_write(ctx->xs, ctx->dws.lk_release, 0u) == cudaSuccess &&
                        cudaStreamSynchronize(ctx->xs) == cudaSuccess;
        cudaGetLastError();
    }
    if (e != cudaSuccess) {
        st = cuda_fail(ctx, e, "moe_layer_init");
        moe_layer_destroy(ctx);
        return st;
    }
    *out = ctx;
    return MOE_OK;
}

moe_status cache_configure(moe_ctx *ctx, int64_t num_slots, void *slot_arena, size_t arena_bytes,
                           uint32_t flags) {
    if (!ctx || !slot_arena || num_slots <= 0) return MOE_ERR_ARG;
    const bool stat = (flags & MOE_CACHE_STATIC_SPLIT) != 0;
    if (stat && (flags & MOE_CACHE_PREFETCH_NEXT)) return MOE_ERR_ARG;
    if (stat && ctx->ep_size > 1) return MOE_ERR_UNSUPPORTED;
    const moe_dims &D = ctx->dims;
    const int64_t need = max_jobs(&D, D.max_rows);
    if (num_slots < need) return MOE_ERR_CAPACITY;
    if ((flags & MOE_CACHE_PREFETCH_NEXT) && num_slots < 2ll * D.E) return MOE_ERR_CAPACITY;
    if (num_slots > 65536) return MOE_ERR_UNSUPPORTED;
    if (arena_bytes < moe_arena_bytes(&D, num_slots)) return MOE_ERR_ARG;
    const bool reset = (flags & MOE_CACHE_RESET) || !ctx->configured || ctx->arena != slot_arena ||
                       ctx->C != num_slots || ((ctx->flags ^ flags) & MOE_CACHE_STATIC_SPLIT);
    // static split: the resident experts per layer, after `need` scratch slots
    int64_t per_layer = stat ? (num_slots - need) / D.L : 0;
    if (per_layer > D.E) per_layer = D.E;
    uint8_t *a = static_cast<uint8_t *>(slot_arena);
    ctx->arena = a;
    ctx->C = num_slots;
    const TableLayout tl = table_layout(&D, num_slots);
    uint8_t *tb = a + up256(num_slots * ctx->lay.bytes);
    ctx->tab.hdr = reinterpret_cast<TableHdr *>(tb + tl.hdr);
    ctx->tab.map = reinterpret_cast<int32_t *>(tb + tl.map);
    ctx->tab.owner = reinterpret_cast<int32_t *>(tb + tl.owner);
    ctx->tab.stamp = reinterpret_cast<unsigned long long *>(tb + tl.stamp);
    ctx->tab.C = num_slots;
    ctx->tab.scratch_base = stat ? (int32_t)(D.L * per_layer) : -1;
    ctx->flags = flags & ~MOE_CACHE_RESET;
    if (ctx->wl.xq >= 0) {  // prefill GEMM descriptors of the arena's weight codes
        if (!make_operand_map(&ctx->maps.w13, a + ctx->lay.w13_codes, D.d / 2, 2 * D.F, num_slots, ctx->lay.bytes) ||
            !make_operand_map(&ctx->maps.w2, a + ctx->lay.w2_codes, D.F / 2, D.d, num_slots, ctx->lay.bytes)) {
            ctx->configured = false;
            return MOE_ERR_UNSUPPORTED;
        }
        if (!D.has_shared || shared_separate(ctx)) {  // no shared job in the grouped GEMMs
            ctx->maps.w13_shared = ctx->maps.w13;
            ctx->maps.w2_shared = ctx->maps.w2;
        }
    }
    if (reset) {
        // unusable until the reset below completes (a failed step returns with
        // configured = false, so forward calls refuse to run on a half-reset table)
        ctx->configured = false;
        // finish outstanding work of the old state first
        CK(cudaStreamSynchronize(ctx->xs2));
        CK(cudaStreamSynchronize(ctx->xs));
        CK(cudaStreamSynchronize(ctx->cs));
        if (stat) {
            CK(launch_table_static(ctx->tab, D.L, D.E, (int)per_layer, ctx->cs));
        } else {
            CK(launch_table_reset(ctx->tab, (int64_t)D.L * D.E, ctx->cs));
        }
        CK(cudaMemsetAsync(ctx->dws.ticket, 0, 4, ctx->cs));
        CK(cudaMemsetAsync(ctx->dws.ticket2, 0, 4 * kMaxTiles, ctx->cs));
        // layer-kernel counters (flags and the release word keep their values:
        // they are compared with sequence numbers that only grow)
        CK(cudaMemsetAsync(ctx->dws.lk_queue, 0, 8, ctx->cs));
        CK(cudaMemsetAsync(ctx->dws.lk_done_a, 0, 4 * (size_t)kMaxSlots, ctx->cs));
        CK(cudaMemsetAsync(ctx->dws.st_done, 0, 4 * ((size_t)kMaxSlots + 1), ctx->cs));
        for (auto &t : ctx->pending) {  // timing records of the old state
            ctx->ev_pool.push_back(t.a);
            ctx->ev_pool.push_back(t.b);
        }
        ctx->pending.clear();
        if (ctx->kspan && ctx->kspan_used > 0)
            CK(cudaMemset(ctx->kspan, 0xff, 2 * ctx->kspan_used * sizeof(unsigned long long)));
        ctx->kspan_used = 0;
        ctx->page_h->error = 0;
        std::fill(ctx->pf_pending.begin(), ctx->pf_pending.end(), 0);
        memset(&ctx->stats, 0, sizeof ctx->stats);
        ctx->state = MOE_OK;
        ctx->err.clear();
        if (stat && per_layer > 0) {
            // fill the resident set (layer l's experts 0 .. per_layer-1 in consecutive
            // slots), merging records consecutive in both the pool and the arena;
            // the compute stream waits for the fill
            int64_t run_src = -1, run_dst = -1, run_n = 0;
            auto flush = [&]() -> cudaError_t {
                if (run_n == 0) return cudaSuccess;
                const cudaError_t e = cudaMemcpyAsync(a + run_dst * ctx->lay.bytes, ctx->pool + run_src * ctx->lay.bytes,
                                                      run_n * ctx->lay.bytes, cudaMemcpyHostToDevice, ctx->xs);
                run_n = 0;
                return e;
            };
            for (int l = 0; l < D.L; ++l)
                for (int64_t e = 0; e < per_layer; ++e) {
                    const int64_t src = ((int64_t)l * D.E + e) % ctx->P, dst = l * per_layer + e;
                    if (run_n > 0 && src == run_src + run_n && dst == run_dst + run_n) {
                        ++run_n;
                        continue;
                    }
                    CK(flush());
                    run_src = src;
                    run_dst = dst;
                    run_n = 1;
                }
            CK(flush());
            CK(cudaEventRecord(ctx->ev_routed, ctx->xs));
            CK(cudaStreamWaitEvent(ctx->cs, ctx->ev_routed, 0));
            CK(copy_tail(ctx, false));
        }
    }
    ctx->configured = true;
    return MOE_OK;
}

moe_status moe_layer_forward(moe_ctx *ctx, int32_t layer, const void *x, int32_t T, float *y,
                             moe_layer_trace *trace) {
    if (!ctx) return MOE_ERR_ARG;
    if (ctx->state != MOE_OK) return MOE_ERR_STATE;
    if (!ctx->configured) return MOE_ERR_STATE;
    const moe_dims &D = ctx->dims;
    if (layer < 0 || layer >= D.L || T < 1 || T > D.max_rows || !x || !y) return MOE_ERR_ARG;
    // x rows are read as 16-byte vectors (and as TMA boxes in prefill); y as floats
    if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(y) & 3)) return MOE_ERR_ARG;
    const auto t0 = std::chrono::steady_clock::now();
    const moe_status st = T <= kDecodeMaxRows ? forward_decode(ctx, layer, x, T, y, trace)
                                              : forward_prefill(ctx, layer, x, T, y, trace);
    ctx->stats.host_us[0] += std::chrono::duration<double, std::micro>(std::chrono::steady_clock::now() - t0).count();
    // a failure after the lookup may leave slots assigned whose copies were
    // never issued: nothing may run on this cache until a reset
    if (st != MOE_OK) ctx->state = MOE_ERR_STATE;
    return st;
}

moe_status moe_layer_forward_host(moe_ctx *ctx, int32_t layer, const void *x_host, int32_t T,
                                  float *y_host, moe_layer_trace *trace) {
    if (!ctx) return MOE_ERR_ARG;
    if (ctx->state != MOE_OK || !ctx->configured) return MOE_ERR_STATE;
    const moe_dims &D = ctx->dims;
    if (layer < 0 || layer >= D.L || T < 1 || T > D.max_rows || !x_host || !y_host) return MOE_ERR_ARG;
    if (T <= kDecodeMaxRows) {
        // decode: the kernels read x and write y through the buffers' mapped device
        // addresses (a few KB over PCIe, no copy launches); unmapped or unaligned
        // buffers take the copy path below
        void *xm = nullptr, *ym = nullptr;
        if (((reinterpret_cast<uintptr_t>(x_host) | reinterpret_cast<uintptr_t>(y_host)) & 15) == 0 &&
            cudaHostGetDevicePointer(&xm, const_cast<void *>(x_host), 0) == cudaSuccess &&
            cudaHostGetDevicePointer(&ym, y_host, 0) == cudaSuccess)
            return moe_layer_forward(ctx, layer, xm, T, static_cast<float *>(ym), trace);
        cudaGetLastError();
    }
    void *xd = ctx->ws + ctx->wl.xstage;
    float *yd = reinterpret_cast<float *>(ctx->ws + ctx->wl.ystage);
    CK(cudaMemcpyAsync(xd, x_host, (size_t)T * D.d * 2, cudaMemcpyHostToDevice, ctx->cs));
    moe_status st = moe_layer_forward(ctx, layer, xd, T, yd, trace);
    if (st != MOE_OK) return st;
    CK(cudaMemcpyAsync(y_host, yd, (size_t)T * D.d * 4, cudaMemcpyDeviceToHost, ctx->cs));
    return MOE_OK;
}

moe_status moe_get_routing(moe_ctx *ctx, int32_t *idx, float *gates, int32_t T) {
    if (!ctx || T < 1 || T != ctx->last_T) return MOE_ERR_ARG;
    CK(cudaStreamSynchronize(ctx->cs));
    if (ctx->page_h->error) return device_error(ctx);
    const size_t n = (size_t)T * ctx->dims.k;
    if (idx) CK(cudaMemcpy(idx, ctx->dws.idx, n * 4, cudaMemcpyDeviceToHost));
    if (gates) CK(cudaMemcpy(gates, ctx->dws.gates, n * 4, cudaMemcpyDeviceToHost));
    return MOE_OK;
}

moe_status moe_cache_export(moe_ctx *ctx, int32_t *map, int32_t *owner, uint64_t *stamp,
                            uint64_t *clock) {
    if (!ctx || !ctx->configured) return MOE_ERR_ARG;
    CK(cudaStreamSynchronize(ctx->cs));
    const int64_t nk = (int64_t)ctx->dims.L * ctx->dims.E;
    if (map) CK(cudaMemcpy(map, ctx->tab.map, nk * 4, cudaMemcpyDeviceToHost));
    if (owner) CK(cudaMemcpy(owner, ctx->tab.owner, ctx->C * 4, cudaMemcpyDeviceToHost));
    if (stamp) CK(cudaMemcpy(stamp, ctx->tab.stamp, ctx->C * 8, cudaMemcpyDeviceToHost));
    if (clock) {
        TableHdr h;
        CK(cudaMemcpy(&h, ctx->tab.hdr, sizeof h, cudaMemcpyDeviceToHost));
        *clock = h.clock;
    }
    return MOE_OK;
}

moe_status moe_get_stats(moe_ctx *ctx, moe_stats *out) {
    if (!ctx || !out) return MOE_ERR_ARG;
    moe_status st = resolve_timing(ctx);
    if (st != MOE_OK) return st;
    if (ctx->page_h->error) return device_error(ctx);
    *out = ctx->stats;
    return MOE_OK;
}

moe_status moe_set_timing(moe_ctx *ctx, int32_t enable) {
    if (!ctx) return MOE_ERR_ARG;
    if (!enable) {
        moe_status st = resolve_timing(ctx);
        ctx->timing = false;
        return st;
    }
    ctx->timing = true;
    return MOE_OK;
}

moe_status moe_set_expert_shard(moe_ctx *ctx, int32_t rank, int32_t size) {
    if (!ctx || size < 1 || rank < 0 || rank >= size || size > ctx->dims.E) return MOE_ERR_ARG;
    // (a shard may own none of a layer's experts: the layer kernel and the
    // streaming kernels write its zero / shared-only partial output)
    if (size > 1 && ((!ctx->fused && ctx->gemv_kind != 1) || (ctx->flags & MOE_CACHE_STATIC_SPLIT)))
        return MOE_ERR_UNSUPPORTED;
    if (rank != ctx->ep_rank || size != ctx->ep_size) ctx->configured = false;  // a new cache: reset first
    ctx->ep_rank = rank;
    ctx->ep_size = size;
    return MOE_OK;
}

moe_status moe_debug_trace(moe_ctx *ctx, uint64_t *out, int32_t n) {
    if (!ctx || !out || n < 0) return MOE_ERR_ARG;
    if (!ctx->trace_d) return MOE_ERR_STATE;
    const int64_t total = (int64_t)kTraceCtas * kTraceSlots;
    const int64_t m = n < total ? n : total;
    CK(cudaStreamSynchronize(ctx->cs));
    CK(cudaMemcpy(out, ctx->trace_d, sizeof(unsigned long long) * m, cudaMemcpyDeviceToHost));
    return MOE_OK;
}

moe_status moe_set_wait_limit(moe_ctx *ctx, double seconds) {
    if (!ctx || !(seconds > 0)) return MOE_ERR_ARG;
    ctx->wait_limit = seconds;
    return MOE_OK;
}

moe_status moe_debug_inject(moe_ctx *ctx, int32_t what, int64_t n) {
    if (!ctx || n < 0) return MOE_ERR_ARG;
    if (what == 0) {
        ctx->inj_copy_fail_at = 0;
        ctx->inj_drop_publish = 0;
        ctx->inj_drop_flags = 0;
        ctx->inj_gemm_skip = 0;
        ctx->inj_stream_skip = 0;
    }
    else if (what == 1) ctx->inj_copy_fail_at = n;
    else if (what == 2) ctx->inj_drop_publish = n;
    else if (what == 3) {  // decode path: 0 = a launch per miss, 1 = the layer kernel
        if (n == 0 && ctx->ep_size > 1 && ctx->gemv_kind != 1) return MOE_ERR_UNSUPPORTED;
        if (n == 1 && !ctx->fused_ok) return MOE_ERR_UNSUPPORTED;
        ctx->fused = n == 1;
    } else if (what == 4) ctx->inj_drop_flags = n;
    else if (what == 8) ctx->inj_stream_skip = n;
    else if (what == 11) {  // decode misses: two copies per record (n = 1) or one (n = 0, default)
        if (n < 0 || n > 1) return MOE_ERR_ARG;
        ctx->split_copies = n == 1;
    } else if (what == 10) {  // decode: the SMs copy the first n bytes of a layer's first miss
        if (n < 0 || (n & 15) || n >= ctx->lay.bytes) return MOE_ERR_ARG;
        if (n > 0 && !ctx->pool_d) return MOE_ERR_UNSUPPORTED;
        ctx->head_bytes = (uint32_t)n;
    }
    else if (what == 9) {  // diagnostic: trace the next n streaming hit launches
        if (!ctx->trace_d &&
            cudaMalloc(reinterpret_cast<void **>(&ctx->trace_d), sizeof(unsigned long long) * kTraceCtas * kTraceSlots) !=
                cudaSuccess) {
            ctx->trace_d = nullptr;
            return MOE_ERR_CUDA;
        }
        ctx->trace_arm = n;
    }
    else if (what == 7) {  // per-miss path expert kernels: 1 streaming, 0 split-K
        if (n < 0 || n > 1) return MOE_ERR_ARG;
        if (n == 0 && ctx->ep_size > 1 && !ctx->fused) return MOE_ERR_UNSUPPORTED;
        ctx->gemv_kind = (int)n;
    } else if (what == 6) {  // decode misses on 1 or 2 copy streams
        if (n < 1 || n > 2) return MOE_ERR_ARG;
        ctx->copy_streams = (int)n;
    }
    else if (what == 5) ctx->inj_gemm_skip = n;
    else return MOE_ERR_ARG;
    return MOE_OK;
}

moe_status plan_split(int32_t m, double B_P, double B_H, double threshold, double expert_bytes,
                      moe_split *out) {
    if (!out || m < 0 || !(B_P > 0) || !(B_H >= 0) || !(expert_bytes > 0)) return MOE_ERR_ARG;
    const bool faster_host = B_H > B_P;
    const double q_real = faster_host ? (double)m * B_P / B_H : (double)m;
    const int32_t mode = (faster_host && B_H / B_P > threshold) ? 1 : 0;
    int64_t q = mode ? (int64_t)(q_real + 0.5) : m;
    if (q > m) q = m;
    out->q = (int32_t)q;
    out->cpu = m - (int32_t)q;
    out->mode = mode;
    out->reserved = 0;
    out->q_real = q_real;
    const double t_pcie = q * expert_bytes / B_P;
    const double t_host = out->cpu > 0 ? out->cpu * expert_bytes / (B_H - B_P) : 0.0;
    out->t_finish = t_pcie > t_host ? t_pcie : t_host;
    return MOE_OK;
}

moe_status moe_measure_h2d(void *dev_buf, const void *host_buf, size_t bytes, size_t chunk_bytes,
                           int32_t reps, void *stream, double *gbs) {
    moe_ctx *ctx = nullptr;
    if (!dev_buf || !host_buf || !bytes || reps < 1 || !stream || !gbs) return MOE_ERR_ARG;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, host_buf) != cudaSuccess || attr.type != cudaMemoryTypeHost) {
        cudaGetLastError();
        return MOE_ERR_NOT_PINNED;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaEvent_t a, b;
    CK(cudaEventCreate(&a));
    CK(cudaEventCreate(&b));
    const size_t chunk = chunk_bytes ? chunk_bytes : bytes;
    double best = 0.0;
    for (int r = 0; r < reps; ++r) {
        CK(cudaEventRecord(a, s));
        for (size_t o = 0; o < bytes; o += chunk) {
            const size_t n = bytes - o < chunk ? bytes - o : chunk;
            CK(cudaMemcpyAsync(static_cast<uint8_t *>(dev_buf) + o,
                               static_cast<const uint8_t *>(host_buf) + o, n,
                               cudaMemcpyHostToDevice, s));
        }
        CK(cudaEventRecord(b, s));
        CK(cudaEventSynchronize(b));
        float ms = 0.f;
        CK(cudaEventElapsedTime(&ms, a, b));
        const double rate = (double)bytes / (ms * 1e-3) / 1e9;
        if (rate > best) best = rate;
    }
    cudaEventDestroy(a);
    cudaEventDestroy(b);
    *gbs = best;
    return MOE_OK;
}

// SM-driven copy from mapped page-locked host memory: every thread streams
// 16-byte loads (4 in flight) over PCIe and stores them to device memory.
__global__ void h2d_sm_copy_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, size_t n16) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    for (; i + 3 * stride < n16; i += 4 * stride) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldcv(src + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) dst[i + u * stride] = v[u];
    }
    for (; i < n16; i += stride) dst[i] = __ldcv(src + i);
}

moe_status moe_measure_h2d_sm(void *dev_buf, const void *host_buf, size_t bytes, size_t chunk_bytes,
                              int32_t reps, void *stream, double *gbs) {
    moe_ctx *ctx = nullptr;
    if (!dev_buf || !host_buf || !bytes || reps < 1 || !stream || !gbs) return MOE_ERR_ARG;
    const size_t chunk = chunk_bytes ? chunk_bytes : bytes;
    if ((bytes & 15) || (chunk & 15) || (reinterpret_cast<uintptr_t>(dev_buf) & 15) ||
        (reinterpret_cast<uintptr_t>(host_buf) & 15))
        return MOE_ERR_ARG;
    void *src = nullptr;
    if (cudaHostGetDevicePointer(&src, const_cast<void *>(host_buf), 0) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_NOT_PINNED;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaEvent_t a, b;
    CK(cudaEventCreate(&a));
    CK(cudaEventCreate(&b));
    double best = 0.0;
    for (int r = 0; r < reps; ++r) {
        CK(cudaEventRecord(a, s));
        for (size_t o = 0; o < bytes; o += chunk) {
            const size_t n = bytes - o < chunk ? bytes - o : chunk;
            h2d_sm_copy_kernel<<<296, 512, 0, s>>>(
                reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(src) + o),
                reinterpret_cast<uint4 *>(static_cast<uint8_t *>(dev_buf) + o), n / 16);
        }
        CK(cudaGetLastError());
        CK(cudaEventRecord(b, s));
        CK(cudaEventSynchronize(b));
        float ms = 0.f;
        CK(cudaEventElapsedTime(&ms, a, b));
        const double rate = (double)bytes / (ms * 1e-3) / 1e9;
        if (rate > best) best = rate;
    }
    cudaEventDestroy(a);
    cudaEventDestroy(b);
    *gbs = best;
    return MOE_OK;
}

const char *moe_status_str(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_ARG: return "invalid argument";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_NOT_PINNED: return "host pool is not page-locked";
        case MOE_ERR_CAPACITY: return "cache too small";
        case MOE_ERR_TIMEOUT: return "timed out waiting for the device";
        case MOE_ERR_STATE: return "context needs a cache reset";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    }
    return "unknown status";
}

const char *moe_last_error(const moe_ctx *ctx) { return ctx ? ctx->err.c_str() : ""; }

void moe_layer_destroy(moe_ctx *ctx) {
    if (!ctx) return;
    if (ctx->cs) cudaStreamSynchronize(ctx->cs);
    if (ctx->xs) cudaStreamSynchronize(ctx->xs);
    if (ctx->xs2) {
        cudaStreamSynchronize(ctx->xs2);
        cudaStreamDestroy(ctx->xs2);
    }
    if (ctx->ev_xs_tail) cudaEventDestroy(ctx->ev_xs_tail);
    if (ctx->ev_xs2_tail) cudaEventDestroy(ctx->ev_xs2_tail);
    for (auto &t : ctx->pending) {
        if (t.a) cudaEventDestroy(t.a);
        if (t.b) cudaEventDestroy(t.b);
    }
    for (auto e : ctx->ev_pool) cudaEventDestroy(e);
    for (auto e : ctx->miss_ev)
        if (e) cudaEventDestroy(e);
    for (auto e : ctx->ev_pf)
        if (e) cudaEventDestroy(e);
    if (ctx->ev_routed) cudaEventDestroy(ctx->ev_routed);
    if (ctx->page_h) cudaFreeHost(ctx->page_h);
    if (ctx->kspan) cudaFree(ctx->kspan);
    if (ctx->trace_d) cudaFree(ctx->trace_d);
    delete ctx;
}

}  // extern "C"
