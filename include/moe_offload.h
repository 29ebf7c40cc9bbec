/*
 * moe_offload.h -- C ABI of the per-layer routed-expert step of an
 * expert-offloading MoE engine (one B200, sm_100a).
 *
 * The step, per layer (FreeToken offload backend: experts live in host RAM,
 * the GPU holds an LRU cache of expert slots and misses stream over PCIe --
 * florigen.ai "FreeTokenは何をしているのか"; pirouter.ai "32 GB に 65 GB が載る仕組み"):
 *   1. router logits z = W_r x, softmax, top-k, gates renormalised over the k;
 *   2. lookup of the selected (layer, expert) pairs in one global LRU cache of
 *      HBM slots (ai-hardware-zukan "GPUに載らない分をどう間に合わせるか";
 *      gaming-st.com "技術的背景");
 *   3. misses: the NVFP4 expert record is copied from the pinned host pool
 *      into its slot (cudaMemcpyAsync on the copy stream), overlapped with the
 *      hit experts' compute;
 *   4. SwiGLU expert FFN over NVFP4 weights (florigen.ai "NVFP4で約135GBまで縮める":
 *      E2M1 values with block scaling);
 *   5. y = sum over selected experts in ascending id of g_e * E_e(x) + S(x)
 *      (S = the layer's shared expert, weight 1, when present).
 * For prefill chunks, the next layer's experts are streamed in while the
 * current layer computes (holude.com "長いプロンプトとエージェント処理も意識している").
 *
 * Expert record (one contiguous block per (layer, expert)) in the default
 * format, NVFP4 (other formats: MOE_FMT_* below); moe_record_layout returns
 * the offsets off[0..5] of the sections named below:
 *   off[4] 3 fp32 tensor scales: gate, up, down (at the record head)
 *   off[0] W13 codes  [2F x d/2] bytes; row 2j = gate_j, row 2j+1 = up_j; E2M1,
 *                     two per byte, element 2i in the low nibble
 *   off[1] W13 scales [2F x d/16] E4M3 bytes, one per 16 consecutive elements of a row
 *   off[2] W2 codes   [d x F/2] bytes (row = output dim, K = F)
 *   off[3] W2 scales  [d x F/16]
 *   off[5] total size; every section starts on a 256-byte boundary.  The
 *   gate/up half (tensor scales + W13) is the prefix [0, off[2]).
 *   w = e2m1(code) * e4m3(scale) * tensor_scale.
 *
 * Conventions: all functions return a moe_status and never throw; pointers
 * documented as "device" must be device memory of the current CUDA device;
 * the library allocates no device memory on the step's path -- the caller
 * passes every device buffer.  The library owns its context, a few CUDA
 * events, one small mapped pinned page for the device-to-host miss list, and
 * (only once moe_set_timing enables timing) a 4 MB device buffer of timing slots.
 */
#ifndef MOE_OFFLOAD_H
#define MOE_OFFLOAD_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_ARG = 1,         /* null pointer, bad size, layer or row count out of range */
    MOE_ERR_CUDA = 2,        /* a CUDA runtime call failed; moe_last_error() has the text */
    MOE_ERR_NOT_PINNED = 3,  /* the host pool is not page-locked (cudaHostAlloc/Register) */
    MOE_ERR_CAPACITY = 4,    /* cache slots fewer than one lookup batch needs */
    MOE_ERR_TIMEOUT = 5,     /* the host's wait for the device miss list ran out */
    MOE_ERR_STATE = 6,       /* context unusable until cache_configure(..., MOE_CACHE_RESET) */
    MOE_ERR_UNSUPPORTED = 7  /* shape outside what the kernels handle (see moe_layer_init) */
} moe_status;

/* Layer-stack dimensions.  L layers of E routed experts, top-k, hidden width d,
 * expert FFN width F (SwiGLU: gate and up [F x d], down [d x F]).
 * has_shared: one always-used shared expert per layer (FreeToken pages: Qwen3.8-Flash-Next
 * uses 10 routed + 1 shared per token, florigen.ai).  renormalize: gates are
 * the softmax renormalised over the selected k (1) or the plain softmax probabilities (0).
 * max_rows: largest T passed to moe_layer_forward.
 * pool_records: P, the records in the host pool; expert (l, e) is record (l*E + e) mod P;
 * 0 means P = L*E.
 * weight_format: MOE_FMT_NVFP4 (0) or MOE_FMT_MXFP4, the routed experts' records.
 * shared_format: the shared experts' records (has_shared): the routed
 *   format or MOE_FMT_BF16.  Zeros (both NVFP4) keep the default layout. */
typedef struct {
    int32_t L, E, k, d, F;
    int32_t has_shared;
    int32_t renormalize;
    int32_t max_rows;
    int64_t pool_records;
    int32_t weight_format;
    int32_t shared_format;
} moe_dims;

/* Record formats.  NVFP4: the layout below.  MXFP4 (OCP microscaling; the
 * pages' model tables list gpt-oss and DeepSeek-V4 routed experts in MXFP4):
 * E2M1 codes as in NVFP4, one E8M0 scale byte 2^(c - 127) per 32 consecutive
 * elements of a row (c = 255: NaN), no tensor scales; sections off[0] W13
 * codes [2F x d/2], off[1] W13 scales [2F x d/32], off[2] W2 codes [d x F/2],
 * off[3] W2 scales [d x F/32], 256-byte aligned, off[4] = -1, off[5] total.
 * BF16 (shared experts only; florigen.ai "NVFP4で約135GBまで縮める" keeps
 * them in BF16): W13 [2F x d] bf16 (row 2j = gate_j, 2j+1 = up_j) at 0, then
 * W2 [d x F] at 4Fd bytes; 6Fd bytes.  On the prefill path MXFP4 experts are
 * W4A4 with MXFP4 activations (OCP: E8M0 scale 2^e per 32 values, e =
 * floor(log2 amax) - 2, E2M1 codes, no row scale) and a BF16 shared expert is
 * not quantized (bf16 GEMMs, fp32 accumulation, h carried as bf16 (hi, lo)). */
#define MOE_FMT_NVFP4 0
#define MOE_FMT_MXFP4 1
#define MOE_FMT_BF16 2

typedef struct moe_ctx moe_ctx; /* opaque, library-owned host state */

/* One cache event of a lookup batch. key = layer*E + expert. */
typedef struct {
    int32_t layer, expert, slot, hit; /* hit: 1 = hit, 0 = miss (slot newly filled) */
    int64_t evicted_key;              /* key evicted from slot, -1 if the slot was free */
    int32_t prefetch;                 /* 1 = entry of a next-layer prefetch batch */
    int32_t reserved;
} moe_cache_event;

/* Caller-owned host array that moe_layer_forward fills with the call's cache
 * events, in batch order (ascending expert id per batch).  count is set to the
 * number of events; if capacity is smaller, only capacity are written and count
 * still reports the total. */
typedef struct {
    moe_cache_event *events;
    int32_t capacity;
    int32_t count;
} moe_layer_trace;

/* Cumulative counters since the last MOE_CACHE_RESET.
 * lookups/hits/misses count routed lookups (each distinct (layer, expert) of a
 * batch once); prefetch_* count next-layer prefetch entries separately. */
/* Kernel classes of the timing counters.  MOE_K_GATEUP / MOE_K_DOWN: the
 * per-miss launches when a missed record comes in two copies (and, with the
 * split-K kernels, the hit launches); MOE_K_MISS: the default path's one
 * launch per miss (its gate/up, then its down, after its record landed whole);
 * MOE_K_LAYER: the decode layer kernel (every expert GEMV of a layer in one
 * launch, misses as their copies land); MOE_K_LAYER_HITS: the hit and shared
 * experts' gate/up and down -- the default path's hit launch, or the layer
 * kernel up to the end of its last resident-expert item (the part bounded by
 * HBM, not by the copies; then not a launch of its own). */
enum { MOE_K_ROUTE = 0, MOE_K_GATEUP, MOE_K_DOWN, MOE_K_COMBINE, MOE_K_PREFILL_ROUTE,
       MOE_K_PREFILL_GATEUP, MOE_K_PREFILL_DOWN, MOE_K_LAYER, MOE_K_LAYER_HITS, MOE_K_MISS, MOE_K_COUNT };
typedef struct {
    int64_t lookups, hits, misses, evictions;
    int64_t prefetch_lookups, prefetch_misses;
    int64_t h2d_copies, h2d_bytes;
    int64_t forward_calls;
    /* with timing on (moe_set_timing): per kernel class, launches, summed device
     * milliseconds (CUDA events on the launching stream) and algorithmic bytes */
    int64_t kernel_launches[MOE_K_COUNT];
    double kernel_ms[MOE_K_COUNT];
    double kernel_bytes[MOE_K_COUNT];
    /* decode route kernel, summed over calls: microseconds its last CTA spent in
     * [0] logits + split of x, [1] CTA election, [2] softmax/top-k, [3] job list,
     * [4] table reads, [5] victim selection + table writes, [6] publishing the
     * miss list; [7] launch to start (waiting for the previous layer; the
     * kernel is launched early).  Device %globaltimer. */
    double route_phase_us[8];
    /* host side, summed over forward calls (steady clock): [0] time inside the
     * calls, [1] of which waiting for the device's miss list, [2] of which
     * issuing the copies and launches that follow it */
    double host_us[3];
    /* with timing on, per kernel class: summed device spans of the launches,
     * from the first CTA's start (after its wait on the previous kernel) to the
     * last CTA's end (%globaltimer); 0 for classes not instrumented */
    double kernel_span_ms[MOE_K_COUNT];
} moe_stats;

/* Hybrid split plan (ai-hardware-zukan "GPUに載らない分をどう間に合わせるか";
 * florigen.ai "CPU/PCIe ratio 1.70x"). */
typedef struct {
    int32_t q;        /* misses sent over PCIe */
    int32_t cpu;      /* misses left to host-side processing (m - q) */
    int32_t mode;     /* 0 = offload (all over PCIe), 1 = hybrid */
    int32_t reserved;
    double q_real;    /* m*B_P/B_H for B_H > B_P, else m */
    double t_finish;  /* seconds until both sides finish, for experts of expert_bytes */
} moe_split;

/* cache_configure flags */
#define MOE_CACHE_RESET 1u          /* empty the cache (cold start), zero the counters */
#define MOE_CACHE_PREFETCH_NEXT 2u  /* prefill: stream layer l+1's experts during layer l */
/* The pages' comparison policy (ai-hardware-zukan.com, "GPUに載らない分をどう間に合わせるか":
 * experts split over the layers statically, without looking at the routing):
 * with R = min(k * max_rows, E) scratch slots, each layer keeps its experts
 * 0 .. s-1 resident, s = min((num_slots - R) / L, E), in slots l*s .. l*s+s-1,
 * copied in at the reset (before the next call's kernels); every other
 * selected expert is a miss, copied on each use into scratch slot L*s + m (m:
 * its rank among the batch's misses, ascending id), and nothing is evicted.
 * Not with MOE_CACHE_PREFETCH_NEXT (MOE_ERR_ARG).  Changing the policy resets. */
#define MOE_CACHE_STATIC_SPLIT 4u

/* Bytes of one routed expert record (weight_format); 0 if dims are invalid. */
MOE_API size_t moe_record_bytes(const moe_dims *dims);

/* Bytes of one shared-expert record (shared_format); 0 if dims are invalid. */
MOE_API size_t moe_shared_record_bytes(const moe_dims *dims);

/* Section offsets of one routed record into off[6] (see the layouts above;
 * -1 for a section the format does not have). */
MOE_API moe_status moe_record_layout(const moe_dims *dims, int64_t off[6]);

/* Device workspace bytes moe_layer_init needs for these dims (caller-owned). */
MOE_API size_t moe_workspace_bytes(const moe_dims *dims);

/* Device bytes of a slot arena of num_slots slots plus its cache table. */
MOE_API size_t moe_arena_bytes(const moe_dims *dims, int64_t num_slots);

/* Create a context: the layer stack's routers, shared experts and the pinned
 * host pool that every miss is copied from (pirouter.ai "32 GB に 65 GB が載る仕組み":
 * the expert pool lives in page-locked host RAM that the GPU reads by DMA).
 *   host_pool: P expert records back to back, page-locked host memory
 *              (else MOE_ERR_NOT_PINNED); read by DMA only; caller-owned, must
 *              outlive the context; host_pool_bytes >= P * record bytes.
 *   router_w:  device, bf16 [L][E][d] router weights.
 *   shared_recs: device, L shared-expert records (moe_shared_record_bytes each)
 *              back to back (has_shared), else NULL.
 *   workspace: device, >= moe_workspace_bytes(dims), caller-owned.
 *   compute_stream, copy_stream: cudaStream_t handles (NULL = legacy stream not
 *              accepted: pass real streams); work is issued on them only.
 * Shapes handled: d and F multiples of 64, 1 <= k <= 32, k <= E <= 1024,
 * 1 <= max_rows <= 4096, and with max_rows > 32 (prefill) d >= 256 and
 * F >= 256; else MOE_ERR_UNSUPPORTED.  MOE_ERR_ARG for
 * an unknown format, a BF16 routed format, or (has_shared) a shared format
 * that is neither the routed one nor BF16. */
MOE_API moe_status moe_layer_init(const moe_dims *dims, const void *host_pool, size_t host_pool_bytes,
                          const void *router_w, const void *shared_recs, void *workspace,
                          size_t workspace_bytes, void *compute_stream, void *copy_stream,
                          moe_ctx **out);

/* Attach the HBM slot arena (device, >= moe_arena_bytes(dims, num_slots),
 * caller-owned) holding num_slots expert slots and the cache table, and set
 * flags.  One slot holds one (layer, expert) record and the slots form one LRU
 * cache shared by all layers (ai-hardware-zukan "GPUに載らない分をどう間に合わせるか":
 * the cache unit is the (layer, expert) pair, replaced least-recently-used;
 * gaming-st.com "技術的背景": one global expert cache across the layers).  MOE_CACHE_RESET (required the first time and after an error) empties
 * the cache on the compute stream.  MOE_ERR_CAPACITY if num_slots < k * max_rows
 * distinct experts could need (min(k*max_rows, E)), or, with
 * MOE_CACHE_PREFETCH_NEXT, num_slots < 2*E; MOE_ERR_UNSUPPORTED above 65536 slots.
 * Each miss is copied in two parts (the prefix [0, off[2]) holding the tensor
 * scales and W13, then W2), so the gate/up of a miss overlaps its W2 transfer. */
MOE_API moe_status cache_configure(moe_ctx *ctx, int64_t num_slots, void *slot_arena, size_t arena_bytes,
                           uint32_t flags);

/* One MoE layer on T rows (1 <= T <= max_rows), stream-ordered on compute_stream.
 *   x: device, bf16 [T][d] hidden states, 16-byte aligned; y: device, fp32
 *      [T][d] output, 4-byte aligned (else MOE_ERR_ARG, before any work).
 * Selection order: logits descending, equal logits to the lower id, a NaN
 * logit counted as -inf (in the softmax too), so k distinct ids in [0, E)
 * always come out; non-finite inputs give non-finite gates and outputs, not
 * a fault.
 *   trace: optional host struct filled with the cache events (NULL = none).
 * Returns after the layer's copies and kernels are issued; y is valid when
 * compute_stream reaches that point.  The call waits (host side, bounded) for
 * the device's miss list; on timeout it returns MOE_ERR_TIMEOUT and the
 * context is in MOE_ERR_STATE until a reset.  T <= 32 takes the decode path
 * (W4A16: bf16 activations against NVFP4 or MXFP4 weights; a BF16 shared
 * expert runs in its own two launches before the routed ones; where stream
 * memory writes work, every expert GEMV of the layer runs in one persistent
 * launch that starts each miss when the copy stream flags its record, else
 * each miss gets its own launches gated by copy events).  Larger T takes the
 * prefill path: the activations are quantized like the weights -- NVFP4 per
 * row (E2M1 values, E4M3 scale per 16, one fp32 scale per row: x per token, h
 * per token and expert), or MXFP4 (E8M0 per 32) for MXFP4 records -- and
 * multiplied against the weights (W4A4); the lookup batch is
 * the layer's distinct experts, and with MOE_CACHE_PREFETCH_NEXT a second
 * batch of all experts of layer + 1 follows, whose misses are copied while
 * this layer computes (the next call for layer + 1 waits for them; records
 * with consecutive pool indices and slots go in one copy).  The expert FFNs
 * of a prefill call run as grouped block-scaled FP4 GEMMs on the tensor cores
 * (rows grouped by expert, fp32 accumulation); a BF16 shared expert as two
 * bf16 GEMMs.  The trace lists the
 * routed entries, then the prefetch entries (prefetch = 1, layer + 1).
 * Any failure after the argument checks (MOE_ERR_CUDA, MOE_ERR_TIMEOUT, a
 * failed device check) leaves the context in MOE_ERR_STATE until
 * cache_configure(..., MOE_CACHE_RESET): the lookup may have assigned slots
 * whose copies were not issued. */
MOE_API moe_status moe_layer_forward(moe_ctx *ctx, int32_t layer, const void *x, int32_t T, float *y,
                             moe_layer_trace *trace);

/* Same step with HOST buffers: x_host bf16 [T][d] and y_host fp32 [T][d]
 * (page-locked).  Decode (T <= 32) with both buffers mapped into the device
 * address space (cudaHostGetDevicePointer succeeds; true for page-locked
 * memory on systems with unified addressing) and 16-byte aligned: the kernels
 * read x and write y in place over PCIe, with no copies.  Otherwise the copies
 * run on compute_stream through the workspace.  y_host is valid after
 * compute_stream synchronises. */
MOE_API moe_status moe_layer_forward_host(moe_ctx *ctx, int32_t layer, const void *x_host, int32_t T,
                                  float *y_host, moe_layer_trace *trace);

/* Routing of the last forward call: idx int32 [T][k] (ascending per row) and
 * gates fp32 [T][k], host arrays.  Synchronises compute_stream. */
MOE_API moe_status moe_get_routing(moe_ctx *ctx, int32_t *idx, float *gates, int32_t T);

/* Copy of the device cache table: map int32 [L*E] (slot or -1), owner int32
 * [num_slots] (key or -1), stamp uint64 [num_slots], clock.  Any may be NULL.
 * Synchronises compute_stream. */
MOE_API moe_status moe_cache_export(moe_ctx *ctx, int32_t *map, int32_t *owner, uint64_t *stamp,
                            uint64_t *clock);

/* Counters; resolves pending kernel timings (synchronises compute_stream if timing is on). */
MOE_API moe_status moe_get_stats(moe_ctx *ctx, moe_stats *out);

/* Per-kernel-class timing on (1) or off (0): CUDA events around every launch
 * on compute_stream, and device spans (%globaltimer, kernel_span_ms) for the
 * route, expert GEMV and prefill GEMM kernels.  The first enable allocates a
 * 4 MB device buffer of span slots, freed by moe_layer_destroy. */
MOE_API moe_status moe_set_timing(moe_ctx *ctx, int32_t enable);

/* Expert parallelism over several GPUs (one context per GPU; the pages'
 * engine offloads to host RAM from one GPU -- ai-hardware-zukan
 * "GPUに載らない分をどう間に合わせるか" -- and this spreads the cache and the
 * PCIe links over G of them): this context serves the routed experts e with
 * e mod size == rank -- its cache holds and its lookups count only those --
 * and the shared expert only when rank == 0; moe_layer_forward then writes
 * to y this rank's partial sum over its experts of the selected ones (zero if
 * it owns none), and the layer's output is the sum of the partials over the
 * ranks, which the caller forms (e.g. an all-reduce on compute_stream).  Every
 * rank computes the same routing from the same x (moe_get_routing returns all
 * k).  size = 1 (the default) is the whole layer.  A change needs
 * cache_configure(..., MOE_CACHE_RESET) before the next call (MOE_ERR_STATE
 * until then).  Prefill chunks likewise: the lookup and prefetch batches, the
 * grouped GEMMs and the combine cover this rank's experts only.  MOE_ERR_ARG
 * unless 0 <= rank < size <= E; MOE_ERR_UNSUPPORTED for size > 1 with the
 * static split, or with the split-K per-miss kernels selected (debug option
 * what = 7, n = 0) and no decode layer kernel. */
MOE_API moe_status moe_set_expert_shard(moe_ctx *ctx, int32_t rank, int32_t size);

/* Longest wait, in seconds (default 60): the host's wait for the device miss
 * list; (capped at 5 s, counted from the kernel's start) every wait of the
 * decode layer kernel for a miss's copy or for another CTA's tiles; and
 * (capped at 4 s) each mbarrier wait of the prefill expert GEMMs.  A device
 * wait that runs out records a failed check (MOE_ERR_CUDA at the next call). */
MOE_API moe_status moe_set_wait_limit(moe_ctx *ctx, double seconds);

/* Host-side fault injection and path selection for tests.  what = 1: the n-th
 * H2D copy issue (counted from now, 1-based) fails with MOE_ERR_CUDA before it
 * is issued; what = 2: the next n lookups do not publish their miss list, so
 * the host wait runs out (MOE_ERR_TIMEOUT); what = 4: the next n misses are
 * copied without their completion flags, so the decode layer kernel's bounded
 * wait runs out (a failed device check, reported by the next call); what = 5:
 * in the next n prefill calls, one CTA of the gate/up expert GEMM does not
 * issue its first stage's tensor copies, so its bounded mbarrier waits run out
 * (the CTA records the check, frees its tensor memory and returns; the next
 * call reports MOE_ERR_CUDA); what = 3:
 * decode runs the persistent layer kernel (n = 1; MOE_ERR_UNSUPPORTED where
 * stream memory writes do not work) or, the default, a launch for the hit
 * experts and a gate/up and a down launch per miss, gated by copy events
 * (n = 0); what = 6: decode misses go on n copy
 * streams (1: the caller's copy stream; 2: every other miss on a second copy
 * stream the library owns, so that one copy's start-up overlaps another's
 * transfer; the caller's copy stream still waits for it at the end of each
 * call); what = 7: the per-miss path's expert kernels are the streaming
 * kernels (n = 1, the default: bulk-copied tiles, a warp per tile, the hit
 * experts' gate/up and down in one launch) or the split-K kernels (n = 0);
 * what = 8: in the next n streaming-kernel launches, CTA 0 issues no copies
 * for its first work item, so a consumer's bounded wait runs out (the CTA
 * records the check, lets its other copies land and returns; the next call
 * reports MOE_ERR_CUDA); what = 9: diagnostics -- the next n hit-expert
 * launches of the streaming kernels record per-CTA %globaltimer stamps (read
 * them with moe_debug_trace); what = 10: decode (default path) -- the hit
 * launch's SMs copy the first n bytes (a multiple of 16, less than a record)
 * of the layer's first miss from the pool (through its device address) into
 * the miss's slot, and the copy engine moves only the rest (n = 0: off, the
 * default; MOE_ERR_UNSUPPORTED if the pool has no device address); what = 11:
 * decode (default path) copies each missed record as one copy and runs the
 * miss as one launch, gate/up then down (n = 0, the default), or as two
 * copies, the gate/up prefix then W2, with a gate/up and a down launch, so a
 * miss's gate/up runs while its W2 streams (n = 1); what = 0 clears 1, 2, 4,
 * 5 and 8. */
MOE_API moe_status moe_debug_inject(moe_ctx *ctx, int32_t what, int64_t n);

/* Diagnostics: copies the first n (<= 160 * 32) stamps of the last traced
 * launch (see moe_debug_inject what = 9) to out (host, n uint64 values; CTA b's
 * 32 slots at out[32 b ...]: 0 start, 1 set-up done, 2 gate/up counts published,
 * 3 end, and for its first consumer group's first 8 items k: 4 + 3k stage wait
 * begins, 5 + 3k data in, 6 + 3k sums in; 0 = not reached).  Synchronizes the
 * compute stream.  MOE_ERR_STATE if nothing was traced. */
MOE_API moe_status moe_debug_trace(moe_ctx *ctx, uint64_t *out, int32_t n);

/* Hybrid split: m missing experts, PCIe bandwidth B_P, host expert-processing
 * bandwidth B_H (bytes/s), auto threshold (2.0 on the pages).  Equal finish
 * times q/B_P = (m - q)/(B_H - B_P) give q = m*B_P/B_H when B_H > B_P; mode is
 * hybrid iff B_H/B_P > threshold, and then q = round-half-up(q_real); in offload
 * mode q = m.  expert_bytes sizes t_finish.  MOE_ERR_ARG for m < 0, B_P <= 0,
 * B_H < 0 or expert_bytes <= 0.  Pure host function. */
MOE_API moe_status plan_split(int32_t m, double B_P, double B_H, double threshold, double expert_bytes,
                      moe_split *out);

/* Pinned host -> device copy bandwidth (the roofline's H2D term; the pages'
 * "ft bench bw" H2D line, florigen.ai): reps copies of `bytes` from host_buf
 * (page-locked) to dev_buf on `stream`, timed with CUDA events; best rate in
 * GB/s (1e9 B/s) into *gbs.  With chunk_bytes > 0 the copy is issued as
 * back-to-back copies of chunk_bytes each (record-sized copies). */
MOE_API moe_status moe_measure_h2d(void *dev_buf, const void *host_buf, size_t bytes, size_t chunk_bytes,
                           int32_t reps, void *stream, double *gbs);

/* The same measurement with the copy done by the SMs instead of a copy engine:
 * a kernel reads host_buf through its mapped device address with 16-byte loads
 * and writes dev_buf (one launch per chunk).  This is the transfer rate a
 * device-initiated miss fetch would get.  bytes, chunk_bytes and both
 * addresses must be multiples of 16 (MOE_ERR_ARG); MOE_ERR_NOT_PINNED when
 * host_buf has no device mapping.  No counterpart on the pages: it measures
 * the alternative to their copy-engine transfers. */
MOE_API moe_status moe_measure_h2d_sm(void *dev_buf, const void *host_buf, size_t bytes, size_t chunk_bytes,
                              int32_t reps, void *stream, double *gbs);

/* Router logits, softmax and top-k for T rows with no workspace (the routing
 * part of moe_layer_forward: same selection rule -- NaN logits as -inf, ties
 * to the lower id -- gates and ascending id order).
 * The FreeToken pages have no counterpart: this serves callers that cannot
 * allocate device memory when they run -- e.g. a host framework that owns the
 * whole device memory pool and passes only inputs and outputs, or a process
 * whose memory is planned before start-up -- and so cannot give
 * moe_layer_init a workspace.  Its scratch (the [T][E] fp32 logits and a CTA
 * counter, 128 KB + 256 B) lives in an array built into the library, present
 * on every GPU that loads it until the process exits; the call allocates
 * nothing.  All calls share that array and it keeps the last call's contents:
 * each call clears the counter it needs at zero, and calls that overlap on
 * the GPU race -- serialise them.  The first call on a device looks up the
 * array's address with that device current; make it before any stream capture.
 *   router_w: device bf16 [E][d]; x: device bf16 [T][d]; both 16-byte aligned
 *             (MOE_ERR_ARG otherwise, before anything is launched);
 *   idx: device int32 [T][k] out (ascending per row); gates: device fp32 [T][k] out;
 *   stream: cudaStream_t the work is issued on (stream-ordered, returns at once).
 * Limits: T <= 32, E <= 1024, k <= 32, d a multiple of 64; larger sizes return
 * MOE_ERR_UNSUPPORTED.  MOE_ERR_ARG for null pointers or k > E. */
MOE_API moe_status moe_route_noalloc(const void *router_w, const void *x, int32_t T, int32_t E,
                                     int32_t d, int32_t k, int32_t renormalize, int32_t *idx,
                                     float *gates, void *stream);

MOE_API const char *moe_status_str(moe_status s);
MOE_API const char *moe_last_error(const moe_ctx *ctx);
MOE_API void moe_layer_destroy(moe_ctx *ctx);

#ifdef __cplusplus
}
#endif
#endif /* MOE_OFFLOAD_H */
