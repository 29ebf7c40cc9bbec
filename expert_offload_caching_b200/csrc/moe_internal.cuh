// Internal definitions shared by the kernels and the C-ABI host code.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace moe {

constexpr int kDecodeMaxRows = 32;  // T <= this takes the GEMV (decode) path
constexpr int kMaxK = 32;
constexpr int kMaxE = 1024;

// Record sections (byte offsets), computed once per context.
struct RecordLayout {
    int64_t w13_codes, w13_scales, w2_codes, w2_scales, tscales, bytes;
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
    uint32_t *ticket2;   // last-CTA counter of the combining down launch
    // prefill only (T > 32)
    int32_t *cnt;        // [E] rows per expert
    int32_t *fill;       // [E] scatter cursors
    int32_t *jobidx;     // [E] job of an expert, -1 if unused
    float *h32;          // [T][k+1][F] fp32 h before its activation quantization
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
};

enum GemvMode { kGateUp = 0, kDown = 1 };

struct GemvArgs {
    int mode;
    const Job *jobs;
    const int32_t *n_jobs;
    const RowRef *rowrefs;
    int only_job;          // >= 0: process just this job; -1: every hit job (+ shared)
    int all_jobs;          // with only_job = -1: hit and missed jobs alike (prefill)
    float *h32_out;        // gate/up: write fp32 h here instead of the fp16 (hi, lo) pair
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
    // miss; performed by the last CTA of the launch
    int combine;
    const int32_t *n_misses;
    const float *gates;
    float *y;
    uint32_t *ticket;
};

// launchers (one per .cu)
cudaError_t launch_route_lookup(const RouteArgs &a, cudaStream_t s);
cudaError_t launch_gemv(const GemvArgs &a, int grid_y, cudaStream_t s);
cudaError_t launch_table_reset(Table t, int64_t nkeys, cudaStream_t s);
cudaError_t launch_prefill_route(const RouteArgs &a, cudaStream_t s);
cudaError_t launch_prefill_scatter(const RouteArgs &a, cudaStream_t s);
cudaError_t launch_quant_x(const __nv_bfloat16 *x, int T, int d, __half *xh, cudaStream_t s);
cudaError_t launch_quant_h(const float *h32, int T, int k, int F, int has_shared, __half *hh,
                           cudaStream_t s);
cudaError_t launch_combine(const float *part, const float *gates, float *y, int T, int k, int d,
                           int has_shared, cudaStream_t s);

}  // namespace moe
