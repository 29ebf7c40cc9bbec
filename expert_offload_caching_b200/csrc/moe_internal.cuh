// Internal definitions shared by the kernels and the C-ABI host code.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace moe {

constexpr int kDecodeMaxRows = 32;  // T <= this takes the GEMV (decode) path
constexpr int kMaxK = 32;
constexpr int kMaxE = 1024;
constexpr int kMaxTiles = 512;  // GEMV tiles per launch: max(d / 16, F / 8) with d, F <= 4096
constexpr int kMaxSlots = kMaxK * kDecodeMaxRows + 1;  // experts of one decode layer (+ shared)

// Record formats (the values of the C ABI's MOE_FMT_* constants).
constexpr int kFmtNvfp4 = 0, kFmtMxfp4 = 1, kFmtBf16 = 2;

// Record sections (byte offsets, -1 for a section the format lacks), computed
// once per context; fmt is the record format (MOE_FMT_NVFP4 / MXFP4 / BF16).
struct RecordLayout {
    int64_t w13_codes, w13_scales, w2_codes, w2_scales, tscales, bytes;
    int32_t fmt;
};

// Device cache table, in the slot arena after the slots.  The least recently
// used slots are the resident slots with the smallest stamps (the global clock
// at last use; stamps are unique), so victims are found by a parallel scan of
// the stamps rather than by walking a list.
struct TableHdr {
    unsigned long long clock;
    int32_t next_free;  // slots [next_free, C) have never been filled since the reset
    int32_t pad[13];
};

struct Table {
    TableHdr *hdr;
    int32_t *map;               // [L*E] slot of key or -1
    int32_t *owner;             // [C] key in slot or -1
    unsigned long long *stamp;  // [C]
    int64_t C;
    // static per-layer split (scratch_base >= 0): map holds the fixed resident
    // set and never changes; the m-th miss of a batch goes to slot
    // scratch_base + m, reused by every batch
    int32_t scratch_base;
};

// One distinct expert of a lookup batch, in ascending expert order.
struct Job {
    int32_t expert, slot, hit, nrows, row_off, pad[3];
};
// A (row, selection position) pair that uses a job's expert.
struct RowRef {
    int16_t t, p;
};

// Miss list published to the host through mapped pinned memory: one 16-byte
// record per lookup entry (one PCIe write each).  flags: bit 0 hit, bit 1 prefetch.
struct __align__(16) HostEvent {
    int32_t expert, slot, flags, evicted;  // evicted: key or -1
};
struct HostPage {
    volatile uint32_t seq;    // written last by the device
    int32_t n_events;         // routed entries first, then prefetch entries
    int32_t n_jobs;           // routed entries
    int32_t n_misses;         // routed misses
    volatile int32_t error;   // nonzero: a kernel check failed (see diag)
    int32_t n_prefetch_misses;
    int32_t pad[2];
    int32_t diag[16];         // where: kernel mode, block, sizes, address low bits
    uint32_t phase_ns[8];     // route kernel, last CTA: ns spent in each phase (globaltimer)
    HostEvent ev[1];          // [capacity]
};

// Device scratch of the decode path (carved from the caller's workspace).
struct DecodeWs {
    float *z;            // [maxT][E] router logits
    int32_t *idx;        // [maxT][k]
    float *gates;        // [maxT][k]
    Job *jobs;           // [max_jobs]
    int32_t *n_jobs;     // [1]
    int32_t *n_misses;   // [1]
    RowRef *rowrefs;     // [maxT*k]
    __half *xh;          // [maxT][2][d] fp16 hi/lo split of x
    __half *hh;          // [maxT][k+1][2][F] fp16 hi/lo split of h
    float *part;         // [maxT][k+1][d] per-selection expert outputs (p = k: shared)
    uint32_t *ticket;    // last-CTA counter of the route kernel
    uint32_t *ticket2;   // [kMaxTiles] per-tile counters of the combining down launch
    // persistent layer kernel (see LayerArgs)
    uint32_t *lk_queue;    // [2]
    uint32_t *lk_release;  // [1]
    uint32_t *lk_done_a;   // [kMaxSlots]
    uint32_t *lk_flags;    // [2 * kMaxSlots]
    // streaming expert kernel, phase 3: gate/up tiles done per launch expert; CTAs out
    uint32_t *st_done;     // [kMaxSlots]
    uint32_t *st_exit;     // [1]
    // prefill only (T > 32)
    int32_t *cnt;        // [E] rows per expert
    int32_t *fill;       // [E] scatter cursors
    int32_t *jobidx;     // [E] job of an expert, -1 if unused
    float *h32;          // grouped rows x F: fp32 h before its activation quantization
    uint8_t *xq;         // grouped rows x d/2: E2M1 codes of x (NVFP4, per-row scale)
    uint8_t *xq_scales;  // grouped rows x d/16: E4M3 block scales
    float *xq_st;        // grouped rows: fp32 row scales
    uint8_t *hq;         // grouped rows x F/2: E2M1 codes of h
    uint8_t *hq_scales;  // grouped rows x F/16
    float *hq_st;        // grouped rows
    int2 *pairs;         // (job, n tile) pairs of the grouped GEMMs
    int32_t *n_pairs;
    int32_t *n_grouped;  // routed grouped rows of the chunk (all T*k, or the owned ones with expert parallelism)
};

struct RouteArgs {
    const __nv_bfloat16 *Wr;  // [E][d] of this layer
    int L;                    // layers (prefill prefetches layer + 1 < L)
    int prefetch;             // prefill: also look up all experts of the next layer
    const __nv_bfloat16 *Wr_next;  // next layer's router (prefetched into L2) or null
    const __nv_bfloat16 *x;   // [T][d]
    int T, E, d, k, renorm, layer;
    DecodeWs ws;
    Table tab;
    HostPage *page;          // device alias of the mapped page
    uint32_t seq;
    int publish;
    unsigned long long *span;  // launch timing slot (see span_mark), or null
    // expert parallelism: this context serves the experts e with e % ep_size == ep_rank
    int ep_rank, ep_size;
};

enum GemvMode { kGateUp = 0, kDown = 1 };

struct GemvArgs {
    int mode;
    const Job *jobs;
    const int32_t *n_jobs;
    const RowRef *rowrefs;
    int only_job;          // >= 0: process just this job; -1: every hit job (+ shared)
    int slots;             // job slots of the launch, shared expert included (set by launch_gemv)
    int shared_slot;       // gridDim.y index of the shared job, -1 if none
    const uint8_t *arena;
    int64_t rec_bytes;
    const uint8_t *shared_rec;
    int T, k, d, F;
    RecordLayout lay;
    const __half *act;     // gate_up: xh; down: hh
    __half *hh_out;
    float *part_out;
    HostPage *page;        // device alias of the mapped page (error word + diagnostics)
    // combine (down launches only): 1 = always, 2 = only if the lookup had no
    // miss; performed per 16-row output tile by the CTA that completes the
    // tile's last expert
    int combine;
    const int32_t *n_misses;
    const float *gates;
    float *y;
    uint32_t *tile_ticket;  // [tiles] per-tile counters of the combining launch, kept at 0
    unsigned long long *span;  // launch timing slot (see span_mark), or null
    const int32_t *idx;     // [T][k] selected experts: the combine takes the owned ones only
    int ep_rank, ep_size;
    // streaming kernel (expert_stream.cu): phase 1 = gate/up, 2 = down, 3 =
    // gate/up then down of the same experts in one launch (down items wait on
    // done[expert] == F / 8 gate/up tiles); the shared expert is an expert of the
    // launch when shared_item; y gets the shared partial when shared_part
    int phase = 0;
    int shared_item = 0, shared_part = 0;
    uint32_t *done = nullptr;        // [kMaxSlots] phase 3: gate/up tiles completed per launch expert
    uint32_t *exit_ticket = nullptr; // phase 3: CTAs finished (the last one resets done)
    unsigned long long wait_ns = 0;  // every wait of the kernel ends by then (from its start)
    // set by launch_stream
    int tpa = 0, tpb = 0;            // weight tiles per work item (gate/up, down)
    int ns = 0, nc = 0;              // shared-memory stages, consumer warps
    uint32_t stage_bytes = 0, meta_off = 0, rr_off = 0, x_off = 0;
    int exp_cap = 0;                 // experts the metadata area holds
    int inj_skip = 0;                // test injection: CTA 0 issues no copies for its first item
    unsigned long long *trace = nullptr;  // diagnostic: [CTA][kTraceSlots] globaltimer stamps, or null
    // phase 3: the first head_bytes of the layer's first miss, copied by the SMs
    // from the page-locked pool (its device address) into the miss's slot while
    // the host starts the copy engine on the rest (0: off)
    const uint8_t *pool_d = nullptr;
    int64_t pool_P = 0;
    int layer = 0, E = 0;
    uint32_t head_bytes = 0;
};
constexpr int kTraceSlots = 32;
constexpr int kTraceCtas = 160;

// Persistent decode layer kernel (all expert GEMVs of one layer, misses as
// their copies land).  Counters in the workspace, zero between launches (the
// kernel's last CTA resets them): queue[0] next item, queue[1] CTAs done,
// done_a[job] gate/up tiles completed (slot kMaxSlots - 1: the shared expert),
// tile_ticket[d / 16] experts completed per output tile.  miss_flag[2 j] /
// [2 j + 1]: the call's sequence number once job j's gate/up prefix / W2 half
// is in its slot (written by the copy stream); release: the host gives up the
// call (>= seq), every wait ends.
struct LayerArgs {
    const Job *jobs;
    const int32_t *n_jobs;
    const RowRef *rowrefs;
    const uint8_t *arena;
    int64_t rec_bytes;
    const uint8_t *shared_rec;  // this layer's shared record (any format), or null
    int shared_item;            // 1: the shared expert is an item of the launch (routed format)
    int T, k, d, F;
    RecordLayout lay;
    const __half *xh;           // [T][2][d] x as fp16 (hi, lo)
    __half *hh;                 // [T][k+1][2][F]
    float *part;                // [T][k+1][d]
    const float *gates;         // [T][k]
    float *y;                   // [T][d]
    uint32_t *tile_ticket;
    uint32_t *done_a;
    uint32_t *queue;
    const uint32_t *miss_flag;
    const uint32_t *release;
    uint32_t seq;
    unsigned long long wait_ns;  // bound of every wait, from the kernel's start
    HostPage *page;
    unsigned long long *span;      // launch timing slot, or null
    unsigned long long *span_hit;  // [start, end of the last hit/shared item], or null
    const int32_t *idx;            // [T][k] selected experts: the combine takes the owned ones only
    int ep_rank, ep_size;
};

// Grouped W4A4 expert GEMMs of a prefill chunk (tcgen05 block-scaled MMA).
// Activation rows are in expert-grouped order: the routed rows of job j at
// [row_off_j, row_off_j + nrows_j) (RowRef gives (t, p)), then the shared
// expert's rows t at T*k + t.
struct GroupedGemmArgs {
    int mode;                 // kGateUp: h = silu(g) * u into h32; kDown: into part
    const Job *jobs;
    const int32_t *n_jobs;
    const int2 *pairs;        // (job, n tile) per tile pair; job == n_jobs: shared expert
    const int32_t *n_pairs;
    int m_tiles;              // 128-row tiles of the weight matrix
    int layer, T, k, d, F;
    const uint8_t *arena;
    int64_t rec_bytes;
    const uint8_t *shared_rec;  // the L shared-expert records, or null
    RecordLayout lay;
    const uint8_t *act_scales;  // grouped rows x K/16 E4M3
    const float *act_st;        // grouped rows: per-row fp32 scale
    const RowRef *rowrefs;
    float *h32;               // gate/up output: grouped rows x F
    float *part;              // down output: [T][k+1][d]
    HostPage *page;
    unsigned long long *span;  // launch timing slot (see span_mark), or null
    unsigned long long wait_ns;  // bound of each mbarrier wait
    int inj_skip;             // test injection: block 0 does not issue its first stage's copies
};
// TMA descriptors of the operands: weight codes of the slot arena (3D: byte,
// row, slot) and of the shared records (3D: byte, row, layer); grouped
// activation codes (2D: byte, row).
struct GroupedGemmMaps {
    CUtensorMap w13, w2, w13_shared, w2_shared, xq, hq;
    CUtensorMap router;  // router weights (3D: byte, expert row, layer) for the logits GEMM
    // a BF16 shared expert: W13 and W2 of the L records (3D), and its h as bf16 (hi, lo) halves (2D)
    CUtensorMap w13_sbf, w2_sbf, hs;
};

// Launch timing: slot[0] = min over CTAs of the start time, slot[1] = min of
// ~end (so both start at all ones and take atomicMin); one thread per CTA.
__device__ __forceinline__ void span_mark(unsigned long long *slot, int which) {
    if (slot == nullptr) return;
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    atomicMin(slot + which, which ? ~t : t);
}

// launchers (one per .cu)
cudaError_t launch_route_lookup(const RouteArgs &a, cudaStream_t s);
// slots: job slots of the launch (max jobs + shared expert), 1 with only_job
// Streaming expert GEMVs (expert_stream.cu): max_exp = the launch's largest
// possible expert count (hit jobs + shared, or 1 with only_job).
cudaError_t launch_stream(const GemvArgs &a, int max_exp, cudaStream_t s);
cudaError_t launch_gemv(const GemvArgs &a, int slots, cudaStream_t s);
cudaError_t launch_expert_layer(const LayerArgs &a, cudaStream_t s);
// BF16 shared expert of a decode call (T <= 32 rows; x as DecodeWs::xh):
// kGateUp writes h = silu(W1 x) * (W3 x) as fp16 (hi, lo) into hh at selection
// sel0 + t * sel_stride (layout of DecodeWs::hh); kDown reads that h and
// writes W2 h into part at the same selection.
cudaError_t launch_shared_bf16(int mode, const uint8_t *rec, int d, int F, int T, const __half *xh,
                               __half *hh, float *part, int64_t sel0, int64_t sel_stride, cudaStream_t s);
cudaError_t launch_table_reset(Table t, int64_t nkeys, cudaStream_t s);
cudaError_t launch_table_static(Table t, int L, int E, int per_layer, cudaStream_t s);
cudaError_t launch_prefill_route(const RouteArgs &a, cudaStream_t s);
cudaError_t launch_prefill_scatter(const RouteArgs &a, cudaStream_t s);
cudaError_t launch_prefill_select(const RouteArgs &a, cudaStream_t s);
// y[t] = sum of the owned selections' gated partials (all with ep_size 1) + the shared one
cudaError_t launch_combine(const float *part, const float *gates, const int32_t *idx, int ep_rank, int ep_size,
                           float *y, int T, int k, int d, int has_shared, cudaStream_t s);
// mx = 0: NVFP4 (E4M3 per 16 + fp32 row scale st); mx = 1: MXFP4 (E8M0 per 32, st unused).
// Grouped rows: the routed ones [0, *n_routed) of [0, T*k), then (has_shared) T*k + t.
cudaError_t launch_quant_x_grouped(const __nv_bfloat16 *x, int T, int k, int d, int has_shared,
                                   const RowRef *rowrefs, const int32_t *n_routed, uint8_t *codes,
                                   uint8_t *scales, float *st, int mx, cudaStream_t s);
cudaError_t launch_quant_h_grouped(const float *h32, int T, int k, int has_shared, const int32_t *n_routed,
                                   int F, uint8_t *codes, uint8_t *scales, float *st, int mx, cudaStream_t s);
int grouped_pairs_cap(int n_jobs, int T, int k, int has_shared);
cudaError_t launch_tile_plan(const Job *jobs, const int32_t *n_jobs, int T, int has_shared, int2 *pairs,
                             int32_t *n_pairs, cudaStream_t s);
cudaError_t launch_grouped_gemm(const GroupedGemmMaps &maps, const GroupedGemmArgs &a, int pairs_cap,
                                cudaStream_t s);
cudaError_t launch_router_gemm(const CUtensorMap &tm_x, const CUtensorMap &tm_w, float *z, int T, int E, int d,
                               int layer, HostPage *page, cudaStream_t s);
// out[t * out_stride + n] = sum_K A[t][K] B[n][K] (bf16, fp32 accumulation) for
// t < M, n < N; kbytes of K per A row; B's K coordinate modulo wrap bytes (0: none);
// zb: B's matrix in its 3D map.  kbytes and wrap multiples of 128.
cudaError_t launch_bf16_gemm(const CUtensorMap &tm_a, const CUtensorMap &tm_b, float *out, int64_t out_stride,
                             int M, int N, int kbytes, int wrap, int zb, HostPage *page, cudaStream_t s);
// h = silu(g) * u from the gate/up GEMM's [T][2F] output (gate_j in column 2j,
// up_j in 2j + 1), written as bf16 halves: hs[t][j] = bf16(h), hs[t][F + j] =
// bf16(h - that), so that hi + lo keeps about 16 bits of h.
cudaError_t launch_swiglu_split(const float *sg, int T, int F, uint16_t *hs, cudaStream_t s);
bool make_operand_map(CUtensorMap *out, const void *base, int64_t row_bytes, int64_t rows, int64_t count,
                      int64_t matrix_stride);

}  // namespace moe
