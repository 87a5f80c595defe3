/*
 * slora.h -- C ABI of the B200 paged multi-adapter LoRA delta library.
 *
 * The library computes, for a batch in which every token (or request) i uses
 * its own adapter a = a(i),
 *
 *     y_i  <-  y_i + (alpha_a / r_a) * ((x_i . A_a) . B_a)
 *
 * with the adapters' weights held in a pool of fixed-size pages in device
 * memory and reached through a page table.  Sources:
 *   [S1] "Paper explainer: S-LoRA -- memory management for serving thousands of
 *        LoRA adapters" (0h-n0.github.io/posts/paper-2311-04928): section
 *        "LoRA arithmetic" (h = W0 x + A B x per request), section "Unified
 *        Paging" (adapter tensors paged between host RAM and VRAM, LRU
 *        eviction), section "BGMV kernel" (one launch, weights gathered from
 *        paged memory by adapter id; the reference loop skips adapter id < 0).
 *   [S2] "Multi-LoRA serving: S-LoRA, Punica, SGMV, vLLM"
 *        (produtoramaxvision.com.br/blog/multi-lora-serving-s-lora-punica-sgmv-vllm):
 *        section on how the SGMV kernel runs concurrent adapters (scaled form
 *        Y = X.W0 + (alpha/r).((X.A).B); index vector token -> adapter; shrink
 *        d -> r then expand r -> d_out), section on the unified paged pool
 *        (fixed-size non-contiguous pages, asynchronous PCIe page-in on
 *        dedicated streams, internal fragmentation only in the last page of
 *        each adapted layer), metrics section (LRU keeps frequent adapters,
 *        rare ones loaded from host), vLLM flags (--max-loras,
 *        --max-lora-rank, --max-cpu-loras: the analogues of the pool limits
 *        below).
 * The base term X.W0 is not computed here: y holds it on entry.
 *
 * Conventions
 *   - Every call returns slora_status_t.  No call throws.  On any error other
 *     than SLORA_ERR_DEVICE_CHECK nothing is enqueued and the pool is unchanged.
 *     slora_last_error(pool) gives a message for the last failing call.
 *   - Calls on one pool are not thread-safe: the caller serialises them.
 *   - "stream" / "event" arguments are cudaStream_t / cudaEvent_t handles passed
 *     as void*.  NULL means the legacy default stream.  Every device-side effect
 *     of a call is enqueued on the given stream and is asynchronous to the host.
 *   - Ownership: the caller owns ALL device memory (pool pages, tables,
 *     scratch, x, y, index arrays) and all host weight copies.  The library
 *     owns host-side bookkeeping, a small pinned staging ring for page-in
 *     descriptors, and a ring of CUDA events.
 *   - Element types are 16-bit (fp16 or bf16, chosen per pool); x, y and all
 *     adapter weights of a pool share it.  Accumulation is fp32; y is rounded
 *     once, to nearest even.
 *   - Matrices are row-major with a leading dimension in elements.
 *   - Adapter weights are registered as A transposed (r rows of d_in; the
 *     storage PEFT uses for lora_A) and B (r rows of d_out).
 *   - Rank 0 is legal: the adapter has no pages and leaves y unchanged.
 *     Adapter id -1 in an index array means "no adapter": the row is left
 *     unchanged [S1 BGMV reference loop].
 *   - Device-side checks: kernels validate adapter ids and residency.  A bad
 *     token is skipped (its y row unchanged) and recorded in a device error
 *     word; slora_check_device() reads and clears it.  Kernels never trap.
 *
 * Page layout (the pool): each adapter tensor (A_t of projection p: r x d_in,
 * B of projection p: r x d_out) is laid out flat and cut into pages of
 * page_elems elements; only the last page of each tensor is partly empty
 * [S2 paged pool].  The page table maps (adapter, projection, tensor, page
 * number) -> physical page id.
 */
#ifndef SLORA_H
#define SLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SLORA_OK = 0,
  SLORA_ERR_INVALID_ARG = 1,   /* bad argument, shape, id or layout           */
  SLORA_ERR_OOM = 2,           /* page-in cannot fit even after LRU eviction  */
  SLORA_ERR_NOT_RESIDENT = 3,  /* a host-checked batch names a paged-out adapter */
  SLORA_ERR_CUDA = 4,          /* a CUDA runtime call failed                  */
  SLORA_ERR_TIMEOUT = 5,       /* a bounded host wait on an event ran out     */
  SLORA_ERR_DEVICE_CHECK = 6,  /* a kernel recorded a bad token (see check_device) */
  SLORA_ERR_NOT_REGISTERED = 7,/* adapter id was never registered             */
  SLORA_ERR_INJECTED = 8,      /* a failure planted by slora_inject_fault     */
  SLORA_ERR_UNSUPPORTED = 9    /* shape outside what a kernel supports        */
} slora_status_t;

typedef enum { SLORA_F16 = 0, SLORA_BF16 = 1 } slora_dtype_t;

/* How slora_adapter_page_in moves weights from pinned host memory. */
typedef enum {
  SLORA_PAGEIN_KERNEL = 0,     /* one gather kernel reads host memory over PCIe and
                                  writes the scattered pages (default)          */
  SLORA_PAGEIN_MEMCPY = 1      /* one cudaMemcpyAsync per run of consecutive pages */
} slora_pagein_mode_t;

/* Kernels that run slora_lora_delta (and slora_lora_delta_noalloc).  All give
 * fp32 partials per 2048-element slice of d_in, summed in slice order, and one
 * rounding of y; they differ in launches, scheduling and the summation order
 * inside a slice (the FMA pipe for SPLIT and FUSED, the tensor cores' fp32
 * accumulation for STREAM's shrink); the one-CTA-per-token kernel of small
 * AUTO calls sums each rank row in one pass.  slora_decode_kernels() tells
 * how many kernels a call launches. */
typedef enum {
  SLORA_DECODE_AUTO = 0,       /* the library's choice: 16-bit pools run calls of
                                  up to 16 tokens as one CTA per token (plain
                                  loads, no scratch: a latency-bound batch),
                                  17..1024 tokens on STREAM and larger calls on
                                  SPLIT; e4m3 pools take STREAM up to 1024
                                  tokens                                         */
  SLORA_DECODE_SPLIT = 1,      /* always three kernels: segment build, shrink,
                                  expand                                         */
  SLORA_DECODE_FUSED = 2,      /* one persistent kernel with a bulk-copy ring for
                                  calls of up to 1024 tokens (every CTA builds the
                                  segment table, then the shrink and expand tasks
                                  in one launch); SPLIT above that               */
  SLORA_DECODE_STREAM = 3      /* one kernel of streaming stages for calls of up
                                  to 1024 tokens: every CTA plans the call and
                                  claims chunks of shrink tasks, then of expand
                                  tasks, from a counter; a producer warp moves each
                                  stage's rank rows from the pages by bulk copies,
                                  the shrink runs on mma.sync.  SPLIT above 1024
                                  tokens                                         */
} slora_decode_path_t;

/* How a pool stores adapter weights in its pages. */
typedef enum {
  SLORA_WEIGHTS_16 = 0,        /* the pool's 16-bit dtype (fp16 / bf16)             */
  SLORA_WEIGHTS_E4M3 = 1       /* 8-bit e4m3 codes (finite-only form: 4 exponent bits,
                                  bias 7, 3 fraction bits, max 448) with one fp32
                                  scale per rank row of each tensor: weight =
                                  scale[row] * value(code).  A page holds
                                  2 * page_elems codes, so an adapter takes about half
                                  the pages and half the HBM and PCIe bytes
                                  [S2 trade-offs section: adapters quantised to FP8
                                  halve PCIe traffic and keep more of them warm].
                                  x and y stay 16-bit; accumulation is fp32.  Decode
                                  calls of up to 1024 tokens (slora_lora_delta and
                                  slora_lora_delta_noalloc on the one-kernel path) take
                                  such pools; the other compute calls return
                                  SLORA_ERR_UNSUPPORTED.                           */
} slora_weight_format_t;

#define SLORA_MAX_PROJ 8

typedef struct slora_pool slora_pool;

typedef struct {
  int32_t dtype;            /* slora_dtype_t                                         */
  int32_t n_proj;           /* projections per adapter, 1..SLORA_MAX_PROJ            */
  int32_t d_in[SLORA_MAX_PROJ];  /* multiples of 64, at most 32768                   */
  int32_t d_out[SLORA_MAX_PROJ]; /* multiples of 64                                  */
  int32_t max_adapters;     /* adapter ids are 0..max_adapters-1 (<= 16384)          */
  int32_t max_rank;         /* ranks in [0, max_rank], max_rank <= 128               */
  int32_t max_tokens;       /* largest T of any compute call (<= 1<<20)              */
  int32_t pagein_mode;      /* slora_pagein_mode_t                                   */
  int64_t page_elems;       /* elements per page: a power of two, >= 512             */
  int64_t n_pages;          /* pages in dev_pool                                     */
  void* dev_pool;           /* n_pages * page_elems elements, 16-byte aligned        */
  void* dev_tables;         /* slora_tables_bytes(desc) bytes, 256-byte aligned      */
  void* dev_scratch;        /* slora_scratch_bytes(desc) bytes, 256-byte aligned     */
  size_t scratch_bytes;
  int32_t host_only;        /* 1: bookkeeping only, no device memory and no CUDA calls
                               (LRU, page accounting and validation run; compute
                               calls return SLORA_ERR_UNSUPPORTED).  For tests on
                               machines without a GPU.                               */
  int32_t decode_path;      /* slora_decode_path_t: kernels of slora_lora_delta     */
  int32_t weight_format;    /* slora_weight_format_t of every adapter in the pool    */
  int32_t reserved[5];
} slora_pool_desc;

typedef struct {
  int64_t page_ins;         /* adapters copied host -> device by page_in             */
  int64_t hits;             /* page-in requests that found the adapter resident      */
  int64_t evictions;        /* adapters evicted by LRU or slora_adapter_evict        */
  int64_t bytes_paged_in;   /* weight bytes copied host -> device                    */
  int64_t free_pages;
  int64_t resident;         /* adapters resident now                                 */
  int64_t copy_calls;       /* cudaMemcpyAsync calls (memcpy mode) or gather launches */
  int64_t epoch;            /* page-in calls so far                                  */
  int64_t prefetched;       /* adapters copied in by slora_adapter_prefetch          */
  int64_t bytes_prefetched; /* their weight bytes (not counted in bytes_paged_in)    */
  int64_t kv_pages;         /* pages held as KV blocks (slora_kv_alloc)              */
} slora_pool_stats_t;

/* ---- sizing ------------------------------------------------------------- */

/* Bytes of device memory the caller must provide as dev_tables: per adapter
 * rank, scale and a page list sized for max_rank, plus the device error word. */
size_t slora_tables_bytes(const slora_pool_desc* desc);

/* Bytes of device scratch for compute calls with up to max_tokens tokens:
 * segment arrays, work counters and the fp32 shrink partials.  All compute
 * calls of a pool use this one scratch, so their kernels must not overlap on
 * the GPU: issue them on one stream, or order streams with events. */
size_t slora_scratch_bytes(const slora_pool_desc* desc);

/* Pages one adapter of rank `rank` occupies: sum over projections of
 * ceil(rank*d_in/page_elems) + ceil(rank*d_out/page_elems) [S2 paged pool];
 * with e4m3 weights, of ceil(rank*d/(2*page_elems)) (two codes per element). */
int64_t slora_pages_for_rank(const slora_pool_desc* desc, int32_t rank);

/* ---- pool lifetime -------------------------------------------------------- */

/* Creates a pool over caller-owned device buffers.  All pages start free, in
 * ascending id order; all adapters start unregistered.  Initialises dev_tables
 * (synchronously, on the legacy default stream).
 * Errors: INVALID_ARG (sizes, alignment, dtype), CUDA.                         */
slora_status_t slora_pool_create(const slora_pool_desc* desc, slora_pool** out);

/* Waits for the library's own pending page-in work (bounded), frees host
 * bookkeeping.  Caller-owned buffers are left alone. */
slora_status_t slora_pool_destroy(slora_pool* pool);

/* Message for the last failing call on this pool (static storage of the pool). */
const char* slora_last_error(const slora_pool* pool);

/* Replaces the free-page order (the order page-in takes free pages in).
 * order: n_pages distinct page ids, host memory.  Only while no adapter is
 * resident.  Used to scatter adapters over a shuffled pool.                   */
slora_status_t slora_pool_set_page_order(slora_pool* pool, const int32_t* order, int64_t n);

/* ---- adapters ------------------------------------------------------------- */

/* Records adapter `id` (host catalogue only; nothing is copied).
 * host_A_t[p]: rank x d_in[p] elements, host_B[p]: rank x d_out[p] elements,
 * row-major, in PINNED host memory (cudaHostAlloc / cudaHostRegister), 16-byte
 * aligned, valid until the adapter is unregistered.  alpha: LoRA alpha; the
 * scale applied is alpha / rank [S2 scaled form].  Re-registering a resident
 * adapter is INVALID_ARG; a non-resident one is replaced.                     */
slora_status_t slora_adapter_register(slora_pool* pool, int32_t id, int32_t rank, float alpha,
                                      const void* const* host_A_t, const void* const* host_B);

/* As slora_adapter_register, for a pool whose weight_format is
 * SLORA_WEIGHTS_E4M3: codes_A_t[p] (rank x d_in[p] bytes) and codes_B[p]
 * (rank x d_out[p] bytes) are e4m3 codes, row-major, in PINNED host memory,
 * 16-byte aligned, valid until the adapter is unregistered; scales_A_t[p] and
 * scales_B[p] hold one fp32 scale per rank row (host memory, copied by this
 * call).  slora_quantize_e4m3_rows produces both from 16-bit rows.  Weight
 * (k, j) of A_t is scales_A_t[p][k] * value(codes_A_t[p][k * d_in + j]).
 * Errors: as slora_adapter_register; INVALID_ARG on a 16-bit pool (and
 * slora_adapter_register is INVALID_ARG on an e4m3 pool), or for a scale that
 * is negative or not finite.                                                  */
slora_status_t slora_adapter_register_e4m3(slora_pool* pool, int32_t id, int32_t rank, float alpha,
                                           const void* const* codes_A_t, const float* const* scales_A_t,
                                           const void* const* codes_B, const float* const* scales_B);

/* Makes every adapter in ids[0..n) resident and pins them for the compute
 * calls that follow, until the next page_in call [S1 Unified Paging: on-demand
 * load, LRU eviction; S2: asynchronous page-in on dedicated streams].
 *   - resident ones are touched (LRU age refreshed);
 *   - missing ones take free pages; when too few are free, resident adapters
 *     not in ids are evicted, least recently used first (equal ages: lower id
 *     first);
 *   - copies and page-table updates are enqueued on side_stream, after a
 *     device-side wait for the compute that last read the evicted pages;
 *   - done_event (may be NULL) is recorded on side_stream after them: compute
 *     streams must cudaStreamWaitEvent on it before reading these adapters.
 * Contract: a compute call may only use adapters named by the latest page_in
 * call (the step's adapter set); that is what makes eviction safe without a
 * host synchronisation.
 * Errors: INVALID_ARG, NOT_REGISTERED, OOM (nothing changed), TIMEOUT (the
 * staging ring did not drain), INJECTED, CUDA.                                */
slora_status_t slora_adapter_page_in(slora_pool* pool, const int32_t* ids, int32_t n,
                                     void* side_stream, void* done_event);

/* Pages in, ahead of the step that will use them, the ids[0..n) that are not
 * resident, taken in the given order (most wanted first) while they fit:
 *   - at most max_pages pages in total; an id that does not fit is skipped and
 *     the next ones are still tried;
 *   - pages come from the free list, then from resident adapters not named by
 *     the latest page_in call and not prefetched since it, least recently used
 *     first: the current step's set is never touched, nor is it changed;
 *   - copies go on side_stream exactly as page_in's (device-side waits for the
 *     compute that last read reused pages); done_event (may be NULL) is
 *     recorded after them.
 * A prefetched adapter is as recent as the current step's set in the LRU
 * order, and a compute call may use it only after a later page_in names it
 * (that call finds it resident, and its done_event orders after these copies)
 * [S1 implementation notes: with skewed traffic, frequently used adapters are
 * loaded into VRAM ahead of time to avoid cold-start latency; S2 unified pool
 * section: the scheduler anticipates requests with asynchronous PCIe loads on
 * dedicated streams, overlapped with compute].
 * *n_done (may be NULL) = adapters whose copies were enqueued.
 * Errors: INVALID_ARG (also max_pages < 0), NOT_REGISTERED, TIMEOUT,
 * INJECTED, CUDA; never OOM (what does not fit is skipped).                   */
slora_status_t slora_adapter_prefetch(slora_pool* pool, const int32_t* ids, int32_t n, int64_t max_pages,
                                      void* side_stream, void* done_event, int32_t* n_done);

/* Prefetch policy: writes to out[0..*n_out) up to max_n registered adapters
 * that are not resident, most popular first (equal scores: lower id first).
 * Popularity = sum over the adapter's most recent 32 namings by page_in of
 * 2^(-age / half_life), age = page_in calls since that naming [S1
 * implementation notes: pre-load the adapters that skewed traffic uses most;
 * S2 metrics section: LRU keeps frequent adapters, rare ones come from host].
 * Adapters never named are not candidates.  Host only.
 * Errors: INVALID_ARG (half_life <= 0, max_n < 0, NULL out / n_out).          */
slora_status_t slora_prefetch_candidates(const slora_pool* pool, double half_life, int32_t max_n,
                                         int32_t* out, int32_t* n_out);

/* ---- KV-cache blocks in the same pool ------------------------------------- */

/* Takes n pages of the pool for KV-cache blocks (or any other page-granular
 * owner), so that adapters and the KV cache share one pool of one page size
 * [S1 Unified Paging: one unified pool for the KV cache and adapter weights;
 * S2 unified pool section: adapter memory and the KV cache under one paged
 * abstraction]:
 *   - free pages first; when too few are free, resident adapters older than
 *     the current step (not named by the latest page_in, not prefetched since)
 *     are evicted, least recently used first (equal ages: lower id first);
 *   - ids_out[0..n) = the page ids; page g is elements [g*page_elems,
 *     (g+1)*page_elems) of dev_pool, in the pool's 16-bit element type;
 *   - the caller may write the pages after done_event (may be NULL; then use
 *     `stream` itself): it is recorded on `stream` after the evicted adapters'
 *     table entries are cleared and after the compute, page-in copies and KV
 *     owners that last touched those pages.
 * KV pages are never evicted: they stay the caller's until slora_kv_free.
 * Errors: INVALID_ARG, OOM (nothing changed), CUDA.                           */
slora_status_t slora_kv_alloc(slora_pool* pool, int64_t n, int32_t* ids_out, void* stream, void* done_event);

/* Returns KV pages to the pool.  stream: where the last kernels that use these
 * pages were enqueued (an event recorded there orders later adapter copies
 * into the pages after them); NULL: that work has completed.
 * Errors: INVALID_ARG (an id not held as a KV page, or repeated; nothing
 * changed), TIMEOUT, CUDA.                                                    */
slora_status_t slora_kv_free(slora_pool* pool, const int32_t* ids, int64_t n, void* stream);

/* Evicts one resident adapter now (its pages become free once the compute that
 * last used it has finished; the device table entry is cleared on `stream`). */
slora_status_t slora_adapter_evict(slora_pool* pool, int32_t id, void* stream);

/* *out = 1 if resident, 0 if not (host mirror; no device access). */
slora_status_t slora_adapter_is_resident(const slora_pool* pool, int32_t id, int32_t* out);

/* Host-side check of a batch before launch: every idx_host[i] is -1 or a
 * resident adapter named by the latest page_in call.
 * Errors: INVALID_ARG (out of range), NOT_RESIDENT.                           */
slora_status_t slora_check_batch(const slora_pool* pool, const int32_t* idx_host, int32_t T);

/* ---- the hot path --------------------------------------------------------- */

/* Segment build: a stable counting sort of tokens by adapter id, on the device.
 * idx: T int32 (device), -1 = none.  Outputs (device): perm[n_valid] token ids
 * ordered by adapter then position; seg_start[S+1]; seg_adapter[S]; *S_out
 * (device int32).  Tokens whose id is out of range or not resident are left
 * out and recorded in the device error word.  [S2 SGMV: index vector, per-
 * adapter segments; S1 BGMV: -1 = none]                                       */
slora_status_t slora_build_segments(slora_pool* pool, const int32_t* idx, int32_t T,
                                    int32_t* perm, int32_t* seg_start, int32_t* seg_adapter,
                                    int32_t* S_out, void* stream);

/* Prefill segments from requests: request q covers tokens
 * [req_start[q], req_start[q+1]) with adapter req_adapter[q] (-1 = none);
 * neighbouring requests with the same adapter merge into one segment; empty
 * requests are dropped.  All arrays device: seg_start has n+1 entries,
 * seg_adapter n, *S_out one.  Entries after the S-th are filled with empty
 * segments (adapter -1) so the arrays can be passed to slora_sgmv with S = n
 * without reading S back to the host.                                         */
slora_status_t slora_build_sgmv_segments(slora_pool* pool, const int32_t* req_start,
                                         const int32_t* req_adapter, int32_t n,
                                         int32_t* seg_start, int32_t* seg_adapter,
                                         int32_t* S_out, void* stream);

/* BGMV shrink for one projection (decode): t[i, k] = sum_j x[i, j] * A_a[j, k]
 * for k < r_a, a = idx[i]; t[i, k] = 0 for k >= r_a and for rows with no
 * adapter.  x: T x d_in[proj] (ldx), t: T x ldt fp32 (ldt >= max_rank, a multiple
 * of 8, 16-byte aligned), idx: T
 * int32; all device.  [S2 SGMV first phase; S1 BGMV]                           */
slora_status_t slora_bgmv_shrink(slora_pool* pool, int32_t proj, const void* x, int64_t ldx,
                                 const int32_t* idx, int32_t T, float* t, int64_t ldt,
                                 void* stream);

/* BGMV expand for one projection (decode):
 * y[i, l] <- round(y[i, l] + (alpha_a / r_a) * sum_{k < r_a} t[i, k] * B_a[k, l]).
 * t: T x ldt fp32 (as for slora_bgmv_shrink), y: T x d_out[proj] (ldy); device.
 * [S2 second phase]        */
slora_status_t slora_bgmv_expand(slora_pool* pool, int32_t proj, const float* t, int64_t ldt,
                                 const int32_t* idx, int32_t T, void* y, int64_t ldy,
                                 void* stream);

/* The fused delta over several projections of one layer (decode or mixed
 * batches), one segment build and one grouped shrink + one grouped expand
 * launch for all of them; the rank-r intermediate stays in fp32 and is never
 * rounded.  Projections whose x pointers are equal share the reads of x.
 * projs[n], x[n], ldx[n], y[n], ldy[n]: host arrays of device pointers; each
 * x[k] is T x d_in[projs[k]], y[k] is T x d_out[projs[k]] (updated in place).
 * idx: T int32, device.  [S1 BGMV y_i += A_i (B_i x_i) for all i in one
 * launch; S2 two phases; the multi-projection grouping is the "several LoRA
 * linear maps in one kernel" fusion]                                          */
slora_status_t slora_lora_delta(slora_pool* pool, int32_t n, const int32_t* projs,
                                const void* const* x, const int64_t* ldx, void* const* y,
                                const int64_t* ldy, const int32_t* idx, int32_t T,
                                void* stream);

/* SGMV (prefill) on the tensor cores: segments are contiguous token ranges
 * [seg_start[s], seg_start[s+1]) using seg_adapter[s] (-1: skipped).  Same
 * arithmetic as slora_lora_delta; projections as there.  seg_start (S+1) and
 * seg_adapter (S) are device arrays; S and T (= rows of x and y) host ints.
 * Segment bounds and adapters are checked on the device: a segment outside
 * [0, T) or with a bad or non-resident adapter is skipped and recorded in the
 * device error word (codes 6, 1, 2; info = segment index; code 7 marks an
 * inconsistent plan and is never expected).  Segments may not overlap.  Ranks are padded to a multiple of 16 for the tensor cores.
 * [S2 SGMV on Tensor Cores, rank bands padded for tensor-core alignment]      */
slora_status_t slora_sgmv(slora_pool* pool, int32_t n, const int32_t* projs,
                          const void* const* x, const int64_t* ldx, void* const* y,
                          const int64_t* ldy, const int32_t* seg_start,
                          const int32_t* seg_adapter, int32_t S, int32_t T, void* stream);

/* The whole linear layer with its LoRA delta, for prefill segments, in one
 * tensor-core kernel:
 *     y[i, :] = x[i, :] . W0 + (alpha_a / r_a) (x[i, :] . A_a) . B_a
 * for the tokens i of a segment whose adapter is a, and y[i, :] = x[i, :] . W0
 * for a segment without one (seg_adapter -1).  y is written, not accumulated.
 * [S2 SGMV section: Y = X.W0 + (alpha/r).((X.A).B); metrics section: the delta
 * fused into the linear layer's output]
 * Per projection k: x[k] (T x d_in, ldx), w0[k] (d_out rows of d_in: the
 * layout of a linear layer's weight, leading dimension ldw[k] >= d_in, a
 * multiple of 8, 16-byte aligned), y[k] (T x d_out, ldy).  seg_start (S + 1)
 * and seg_adapter (S) are device arrays; the segments must cover [0, T) in
 * order (seg_start[0] = 0, seg_start[S] = T), checked on the device (code 6,
 * info = segment; a bad adapter: codes 1, 2, and the segment gets the base map
 * only).  The shrink X.A is computed in the same K loop as X.W0 (the A rows as
 * extra output columns), t enters the tensor cores as two 16-bit halves, and
 * t.B is accumulated into X.W0's accumulator before y is stored once.
 * Errors: INVALID_ARG (also S < 1, T < 1); UNSUPPORTED for max_rank > 64 and
 * for e4m3 pools.                                                             */
slora_status_t slora_sgmv_linear(slora_pool* pool, int32_t n, const int32_t* projs,
                                 const void* const* x, const int64_t* ldx, const void* const* w0,
                                 const int64_t* ldw, void* const* y, const int64_t* ldy,
                                 const int32_t* seg_start, const int32_t* seg_adapter, int32_t S,
                                 int32_t T, void* stream);

/* The decode delta of slora_lora_delta, for callers that cannot allocate
 * device memory at the point of the call: a plug-in whose host framework owns
 * every device allocation and hands it only inputs and outputs, or a serving
 * loop that must not risk an allocation blocking the device.
 * The pages have no counterpart of this entry point; it is an addition of this
 * library.
 * Same arguments, semantics and kernels as slora_lora_delta, but the call's
 * scratch (segments, work plan, counters, fp32 partials) is taken from a fixed
 * device array that the library reserves on every GPU that loads it
 * (slora_noalloc_scratch_bytes(), 8 MiB) instead of the pool's dev_scratch.
 * Nothing is allocated or freed by the call.
 *   - The first call on a device looks up that array's device address (once
 *     per device, with the device current) and keeps it for the life of the
 *     process; make that first call before any stream capture.  Resetting the
 *     device while the library is loaded is not supported.
 *   - All calls share the one array and it keeps the last call's contents; the
 *     kernels clear what must start at zero themselves.  Calls whose kernels
 *     overlap on the GPU (other streams, other threads) race on it: serialise
 *     them.
 *   - A call whose scratch need exceeds the array fails with
 *     SLORA_ERR_INVALID_ARG and a message giving both sizes; nothing is
 *     enqueued.  The need grows with T, max_rank and the projections the call
 *     names (their fp32 partials: ceil(d_in / 2048) x T x round8(max_rank)
 *     floats each), plus about 40 KB of tables.                               */
slora_status_t slora_lora_delta_noalloc(slora_pool* pool, int32_t n, const int32_t* projs,
                                        const void* const* x, const int64_t* ldx,
                                        void* const* y, const int64_t* ldy, const int32_t* idx,
                                        int32_t T, void* stream);

/* Number of kernels slora_lora_delta launches for a call of T tokens on this
 * pool (1: one kernel -- one CTA per token, FUSED or STREAM; 3: segment
 * build, shrink, expand); 0 for T <= 0 or a NULL pool.  Host only. */
int32_t slora_decode_kernels(const slora_pool* pool, int32_t T);

/* Which kernels slora_lora_delta launches for a call of T tokens on this pool
 * (the AUTO choice resolved): one CTA per token, the streaming-stage kernel,
 * the persistent bulk-copy kernel, or segment build + shrink + expand; NONE
 * for T <= 0 or a NULL pool.  Host only. */
typedef enum {
  SLORA_KIND_NONE = 0,
  SLORA_KIND_TOKEN = 1,
  SLORA_KIND_STREAM = 2,
  SLORA_KIND_FUSED = 3,
  SLORA_KIND_SPLIT = 4
} slora_decode_kind_t;
int32_t slora_decode_kind(const slora_pool* pool, int32_t T);

/* Size in bytes of the fixed scratch array used by slora_lora_delta_noalloc. */
size_t slora_noalloc_scratch_bytes(void);

/* ---- diagnostics ---------------------------------------------------------- */

/* Reads back adapter `id`'s weights for projection `proj` from its pages into
 * host_A_t (rank x d_in) and host_B (rank x d_out), synchronously: 16-bit
 * elements, or e4m3 codes (one byte each) in an e4m3 pool.  For tests of the
 * page-table gather (bit-exact).                                               */
slora_status_t slora_debug_gather(slora_pool* pool, int32_t id, int32_t proj, void* host_A_t,
                                  void* host_B);

/* Synchronises `stream`, reads and clears the device error word.  Returns
 * DEVICE_CHECK if a kernel recorded a bad token since the last check; *code
 * and *info (may be NULL) receive the first one (code 1: adapter id out of
 * range, 2: adapter not resident; info: the token index).                      */
slora_status_t slora_check_device(slora_pool* pool, void* stream, int32_t* code, int32_t* info);

slora_status_t slora_pool_stats(const slora_pool* pool, slora_pool_stats_t* out);

/* Quantises `rows` rows of n 16-bit values (in, row-major, fp16 or bf16 per
 * dtype; host memory) to e4m3 codes with one fp32 scale per row, the storage
 * of 8-bit adapter pages [S2 trade-offs section: adapters quantised to FP8
 * halve their PCIe traffic]: scales[r] = max|row r| / 448 (computed in fp64,
 * stored as fp32); codes[r*n + j] = the e4m3 value nearest to in / scales[r]
 * (fp64 quotient; ties to the even fraction; saturating at +-448; e4m3 in its
 * finite-only form, 4 exponent bits with bias 7 and 3 fraction bits).  An
 * all-zero row gets scale 0 and zero codes.  Host work only.
 * Errors: INVALID_ARG (bad dtype or sizes, NULL buffers, a NaN or infinite
 * input).                                                                    */
slora_status_t slora_quantize_e4m3_rows(int32_t dtype, const uint16_t* in, int64_t rows, int64_t n,
                                        uint8_t* codes, float* scales);

/* Timing hook for measuring device time without host gaps.  n = 2: every
 * following compute call records events[0] on its stream right before its
 * first kernel and events[1] right after its last one (the kernels stay back
 * to back).  n >= 4: events[0] before the first kernel and events[k] right
 * after its k-th kernel (segment build, shrink, expand for slora_lora_delta;
 * plan, shrink, expand for slora_sgmv).  Events are cudaEvent_t created by
 * the caller with timing enabled; n = 0 switches the hook off.                */
slora_status_t slora_set_phase_events(slora_pool* pool, void* const* events, int32_t n);

/* Fault injection, host side only: the `after`-th next page-in copy submission
 * (0 = the next one) fails with SLORA_ERR_INJECTED before anything is
 * enqueued, leaving the pool unchanged.  after < 0 disarms.                    */
slora_status_t slora_inject_fault(slora_pool* pool, int32_t after);

#ifdef __cplusplus
}
#endif

#endif /* SLORA_H */
