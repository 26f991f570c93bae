/*
 * rae.h -- C ABI of the B200 (sm_100a) attention hot path for encoder context.
 *
 * The library computes, for packed queries, O = softmax(Q K^T * s + M) V per request and
 * query head, in three families that the M* serving-engine pages describe:
 *
 *   - paged cross-attention (page "mstar.engine.resources.attn.cross",
 *     FlashInferCrossManager): non-causal attention of packed decoder queries over an
 *     encoder context whose K/V were written once into a paged cache and are never
 *     extended; the query side is given per plan label as a cumulative qo_indptr
 *     (QueryPacking);
 *   - cacheless ragged block-causal self-attention within each span of one packed forward
 *     (page "mstar.engine.resources.attn.ragged.base", RaggedBlockCausalAttnManager);
 *   - cacheless two-span cross-attention per request (same page, RaggedCrossAttnManager);
 *   - paged causal self-attention of a step's queries over their own KV stream, after the
 *     step's K/V are appended to it (page "mstar.engine.resources.attn.config",
 *     AttentionStep with causal=True);
 *
 * and writes the context K/V into the pages, plain (the encode step) or with the K/V
 * projections fused in (page "mstar.model.components.attention", CrossAttention.compute_kv).
 *
 * GQA follows the model page ("mstar.model.components.attention", Attention: fewer KV heads
 * than query heads); query head h reads KV head h / (Hq / Hkv).
 *
 * The calls mirror the pages' plan/run split (FlashInferCrossManager.plan and .run): a
 * plan is built on the host once per step and label, copied asynchronously into a device
 * slot, and then reused by every layer's run.  The result of a plan is immutable and opaque
 * to the caller.  Two plan slots exist per context: the pages (FlashInferCrossManager,
 * force_double_buffer) describe the race of a host staging buffer that is overwritten by
 * plan(N+1) while step N's copy is still in flight; each slot here has its own pinned host
 * buffer and its own event, and a slot's host buffer is only rewritten after that event has
 * completed.
 *
 * Conventions
 *   - Every call returns an rae_status.  RAE_OK is 0.  No C++ exception crosses the ABI.
 *     rae_last_error() gives a message for the last failing call on that context.
 *   - All device memory is allocated and owned by the caller (queries, pools, outputs and the
 *     workspace).  The library owns only pinned host staging buffers and CUDA events.  It
 *     never allocates KV storage (the cross manager of the pages allocates nothing either).
 *   - "stream" arguments are cudaStream_t values passed as void*.  Device work is enqueued
 *     asynchronously on that stream; no call synchronises the device except
 *     rae_check_device_status (and a plan or write call that must wait for its own previous
 *     use of a pinned staging buffer).
 *   - Host arrays ("host" below) are read during the call only.  Device pointers ("device")
 *     must stay valid until the enqueued work has completed.
 *   - Layouts (row-major, bf16 = IEEE bfloat16):
 *       q, out         [total_q, Hq, head_dim]
 *       k_pool, v_pool [num_pages, Hkv, page_size, head_dim]   (paged calls)
 *       k, v           [total_kv, Hkv, head_dim]              (ragged calls)
 *     All device buffers must be 16-byte aligned; torch allocations are.
 *   - One rae_ctx may be used from one host thread at a time.  Calls given the same
 *     workspace share its split partials, arrival counters and error word: their device work
 *     must not overlap (one stream per context, or streams ordered by events).
 */
#ifndef RAE_H_
#define RAE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rae_status {
  RAE_OK = 0,
  RAE_ERR_INVALID_ARG = 1,    /* malformed arrays, pointers, sizes or slot */
  RAE_ERR_UNSUPPORTED = 2,    /* not sm_100, head_dim not 64/128, page_size not 16/32/64,
                                 Hq not a multiple of Hkv, group size > 128 */
  RAE_ERR_CAPACITY = 3,       /* a size exceeds a capacity given at rae_create */
  RAE_ERR_CUDA = 4,           /* a CUDA runtime call failed */
  RAE_ERR_DEVICE_TIMEOUT = 5  /* a kernel gave up a bounded wait and set the error word */
} rae_status;

/* Creation-time geometry and capacities. */
typedef struct rae_config {
  int32_t num_qo_heads;      /* Hq */
  int32_t num_kv_heads;      /* Hkv; Hq % Hkv == 0 and Hq / Hkv <= 128 */
  int32_t head_dim;          /* 64 or 128 */
  int32_t page_size;         /* 16, 32 or 64 (paged calls) */
  int32_t max_batch;         /* max requests (paged) or spans (ragged) in one plan */
  int32_t max_q_tokens;      /* max packed query tokens in one plan */
  int32_t max_kv_pages;      /* max page-table entries (nnz) in one plan or write call */
  int32_t max_tiles;         /* max work tiles in one plan */
  int32_t max_partial_rows;  /* rows (of head_dim fp32 plus one lse) of split-KV partials */
  int32_t num_sms;           /* 0: take the device's multiprocessor count */
} rae_config;

typedef struct rae_ctx rae_ctx;

/* A plan, returned by value.  Opaque: the caller stores it and passes it back to run. */
typedef struct rae_plan {
  int32_t kind;              /* internal kernel family */
  int32_t slot;              /* plan slot (0 or 1) in the workspace */
  int32_t num_tiles;
  int32_t num_ctas;
  int32_t num_merge_rows;
  int32_t batch;
  int32_t total_q;
  int32_t rows_max;          /* internal: rows per work unit of the chosen kernel */
  int32_t block_size;
  int32_t image_words;       /* int32 words of the plan image actually used */
  int64_t generation;        /* increments per plan on a context */
  int32_t off_cta_ptr;       /* word offsets of the image's arrays (internal) */
  int32_t off_tiles;
  int32_t off_merge;         /* unused, 0: the split merge is fused into the attention kernels */
  int32_t off_a;
  int32_t off_b;
  int32_t off_c;
  int32_t off_d;
  int32_t kv_extent;         /* what a run's K/V must hold: 1 + the largest page id listed
                                (paged plans: the run's num_pages must be at least this) or
                                the key tokens the spans read (ragged plans: total_kv) */
} rae_plan;

/* Creates a context on the current CUDA device.  Fails with RAE_ERR_UNSUPPORTED on a GPU
 * that is not sm_100 or for an unsupported geometry.  *out is set only on success. */
int rae_create(rae_ctx** out, const rae_config* cfg);

/* Waits for the context's pending staging copies and frees its host resources. */
int rae_destroy(rae_ctx* ctx);

/* Message for the last failing call on ctx.  With ctx NULL: the message of the calling
 * thread's last failing rae_write_context_noalloc call ("no context" if there was none). */
const char* rae_last_error(const rae_ctx* ctx);

/* Bytes of device workspace the caller must allocate (256-byte aligned) and pass to every
 * write, plan and run call on this context: an error word, the two plan slots, a staging
 * area for context writes, and the split-KV partial buffer. */
size_t rae_workspace_bytes(const rae_ctx* ctx);

/* Bytes of one host plan image (for rae_plan_*_host). */
size_t rae_plan_image_bytes(const rae_ctx* ctx);

/*
 * Context write (encode step; CrossAttention.compute_kv gives k, v [enc_len, heads, d] and the
 * KV resource appends them once under the context label; later steps only read them).
 * Scatters packed k_src, v_src [cu_enc[B], Hkv, d] (device, bf16) into k_pool, v_pool
 * [num_pages, Hkv, P, d] (device, bf16): token t of request b goes to page
 * page_indices[page_indptr[b] + t / P], slot t % P.  Nothing else in the pools is touched.
 * cu_enc [B+1], page_indptr [B+1], page_indices [page_indptr[B]] are host int32 arrays.
 * Errors: RAE_ERR_INVALID_ARG for non-monotone arrays, too few pages for a request, a page id
 * outside [0, num_pages) or a page id written twice in one call.
 */
int rae_write_context(rae_ctx* ctx, const void* k_src, const void* v_src, const int32_t* cu_enc,
                      const int32_t* page_indptr, const int32_t* page_indices, int32_t batch,
                      void* k_pool, void* v_pool, int32_t num_pages, void* workspace,
                      void* stream);

/*
 * Context write for callers that cannot allocate device memory.  The M* pages have no
 * counterpart of this call.  It does what rae_write_context does (same arguments, layouts and
 * validation; Hkv, head_dim and page_size given directly), but needs neither a context nor a
 * workspace: its page-copy list goes to a 1 MiB array inside the library's own device memory,
 * which every GPU that loads the library holds until the process exits.  It is meant for code
 * whose device memory is owned by another allocator, or that must not call cudaMalloc (for
 * example inside a latency-critical serving loop).  It calls no allocation routine.
 *   - At most 65536 page copies (pages written) per call; more returns RAE_ERR_CAPACITY
 *     before any device work.
 *   - The first call on a device looks up the array's device address (with that device
 *     current); make that first call before any stream capture.
 *   - The list reaches the device array by a copy from one host array of the library, which
 *     the next call rewrites.  While `stream` is capturing, the call therefore enqueues
 *     nothing and returns RAE_ERR_UNSUPPORTED.
 *   - All calls share the one array, which keeps the last call's list: calls that overlap on
 *     the GPU (different streams, not ordered) race on it and must be serialised by the caller.
 *   - The host arrays may be reused as soon as the call returns.
 *   - A failing call leaves its message for rae_last_error(NULL) on the calling thread.
 */
int rae_write_context_noalloc(const void* k_src, const void* v_src, const int32_t* cu_enc,
                              const int32_t* page_indptr, const int32_t* page_indices,
                              int32_t batch, void* k_pool, void* v_pool, int32_t num_pages,
                              int32_t num_kv_heads, int32_t head_dim, int32_t page_size,
                              void* stream);

/*
 * Fused K/V projection and context write (page "mstar.model.components.attention",
 * CrossAttention.compute_kv: (enc_len, hidden) -> (k, v), each (enc_len, heads, head_dim),
 * through nn.Linear weights; page "mstar.engine.resources.attn.cross": the context written
 * once).  For every packed encoder token row x of `hidden` [cu_enc[B], hidden_dim] (device,
 * bf16, row-major): k = x . w_k^T (+ b_k), v = x . w_v^T (+ b_v), with w_k, w_v
 * [num_kv_heads * head_dim, hidden_dim] (device, bf16, nn.Linear layout) and b_k, b_v
 * [num_kv_heads * head_dim] bf16 or NULL; fp32 accumulation, one bf16 rounding.  Token t of
 * request b is stored where rae_write_context would store row cu_enc[b] + t (same host arrays
 * and checks), so the projected K/V are never materialised elsewhere.  Requires
 * hidden_dim % 64 == 0 and num_kv_heads * head_dim % 128 == 0 (RAE_ERR_UNSUPPORTED
 * otherwise); every device buffer 16-byte aligned; at most 8388480 tokens.  Asynchronous on
 * `stream`.
 */
int rae_project_write_context(rae_ctx* ctx, const void* hidden, int32_t hidden_dim,
                              const void* w_k, const void* b_k, const void* w_v, const void* b_v,
                              const int32_t* cu_enc, const int32_t* page_indptr,
                              const int32_t* page_indices, int32_t batch, void* k_pool,
                              void* v_pool, int32_t num_pages, void* workspace, void* stream);

/*
 * One tensor-parallel rank's share of the output projection (page
 * "mstar.model.components.distributed.attention", ParallelAttention: query and KV heads are
 * sharded over ranks -- KVConfig.shard narrows the head counts to one rank's slice -- and the
 * only exchange of the layer is the all-reduce inside o_proj).  A rank holding query heads
 * [h0, h0 + Hq_r) multiplies its attention output attn [m, k] (device, bf16, row-major,
 * k = Hq_r * head_dim: the run's output of its heads) by its columns of W_o, given as
 * w_o [n, k] (device, bf16, nn.Linear layout: row j holds W_o[j, h0*d ... (h0+Hq_r)*d)), and
 * writes out [m, n] (device, fp32, row-major) = attn . w_o^T (+ bias [n], bf16, or NULL).
 * The caller sums the ranks' outputs (one all-reduce); exactly one rank passes the bias.
 * fp32 accumulation.  Requires k % 64 == 0 and n % 128 == 0 (RAE_ERR_UNSUPPORTED otherwise);
 * every device buffer 16-byte aligned.  Asynchronous on `stream`; bounded waits report
 * through the workspace's error word like the attention calls.
 */
int rae_o_proj_partial(rae_ctx* ctx, const void* attn, int32_t m, int32_t k, const void* w_o,
                       int32_t n, const void* bias, void* out, void* workspace, void* stream);

/*
 * Append (page "mstar.engine.resources.attn.config", AttentionStep: a step's own tokens join
 * its KV stream; page "mstar.engine.resources.attn.cross": a stream is written through
 * ordinary Segments).  Writes the append_indptr[b+1] - append_indptr[b] new tokens of
 * request b -- rows append_indptr[b]... of k_new, v_new [append_indptr[B], Hkv, d] (device,
 * bf16) -- to sequence positions kv_len[b] - n_b ... kv_len[b] - 1 of its pages, where kv_len
 * counts the request's tokens after the append.  Host int32 arrays as for rae_plan_paged;
 * the pages must cover kv_len tokens, a page may be written by one request only per call,
 * and nothing outside those slots is touched.  Asynchronous on `stream`; bit-exact copy.
 */
int rae_append_kv(rae_ctx* ctx, const void* k_new, const void* v_new,
                  const int32_t* append_indptr, const int32_t* kv_page_indptr,
                  const int32_t* kv_page_indices, const int32_t* kv_len, int32_t batch,
                  void* k_pool, void* v_pool, int32_t num_pages, void* workspace, void* stream);

/*
 * Plan of paged cross-attention (FlashInferCrossManager.plan; QueryPacking.qo_indptr).
 * Host int32 arrays: qo_indptr [B+1] (cumulative query lengths, qo_indptr[0] == 0),
 * kv_page_indptr [B+1], kv_page_indices [kv_page_indptr[B]], kv_len [B] (context tokens of
 * each request; request b needs kv_page_indptr[b+1] - kv_page_indptr[b] >= ceil(kv_len[b]/P),
 * extra pages are never read).  Validates, builds the work tiles and the split-KV schedule
 * (partial rows and an arrival counter for every unit whose keys are split), stages them in
 * slot `slot` (0 or 1) and copies them into the workspace on `stream`.  *out describes the
 * plan.
 */
int rae_plan_paged(rae_ctx* ctx, int32_t slot, const int32_t* qo_indptr,
                   const int32_t* kv_page_indptr, const int32_t* kv_page_indices,
                   const int32_t* kv_len, int32_t batch, int32_t num_pages, void* workspace,
                   void* stream, rae_plan* out);

/*
 * Plan of paged causal self-attention (page "mstar.engine.resources.attn.config",
 * AttentionStep with causal=True): the same arrays as rae_plan_paged, where the
 * qo_indptr[b+1] - qo_indptr[b] queries of request b are the last tokens of its kv_len[b]
 * tokens (already appended), and query i of the request sees keys 0 ... kv_len[b] - qlen + i.
 * qlen <= kv_len for every request (RAE_ERR_INVALID_ARG otherwise).  Run with rae_run_paged.
 */
int rae_plan_paged_causal(rae_ctx* ctx, int32_t slot, const int32_t* qo_indptr,
                          const int32_t* kv_page_indptr, const int32_t* kv_page_indices,
                          const int32_t* kv_len, int32_t batch, int32_t num_pages,
                          void* workspace, void* stream, rae_plan* out);

/*
 * Plan of cacheless ragged attention (RaggedBlockCausalAttnManager / RaggedCrossAttnManager).
 * Host int32 arrays cu_q [S+1] and cu_kv [S+1] (NULL: self-attention, keys are the query
 * span).  block_size > 0: block-causal, local position i sees j iff j / bs <= i / bs (blocks
 * counted from each span's start); block_size == 0: every key of the span is visible.
 */
int rae_plan_ragged(rae_ctx* ctx, int32_t slot, const int32_t* cu_q, const int32_t* cu_kv,
                    int32_t num_spans, int32_t block_size, void* workspace, void* stream,
                    rae_plan* out);

/*
 * One layer's paged cross-attention (FlashInferCrossManager.run): reads q [total_q, Hq, d],
 * k_pool, v_pool (device, bf16; never written) and writes out [total_q, Hq, d] (device, bf16).
 * sm_scale <= 0 selects 1/sqrt(head_dim).  The plan must come from rae_plan_paged (or
 * rae_plan_paged_causal) on this context with the same workspace, and its slot must not have
 * been re-planned since.  num_pages is the number of pages the pools hold; a plan that lists
 * a page id >= num_pages (num_pages < plan->kv_extent) is rejected with RAE_ERR_INVALID_ARG
 * before anything is launched.
 */
int rae_run_paged(rae_ctx* ctx, const rae_plan* plan, const void* q, const void* k_pool,
                  const void* v_pool, int32_t num_pages, void* out, float sm_scale,
                  void* workspace, void* stream);

/* One layer's ragged attention: q [cu_q[S], Hq, d], k, v [cu_kv[S], Hkv, d] -> out (device,
 * bf16).  total_kv is the number of key tokens k and v hold; fewer than the plan's spans read
 * (total_kv < plan->kv_extent) is rejected with RAE_ERR_INVALID_ARG before any launch. */
int rae_run_ragged(rae_ctx* ctx, const rae_plan* plan, const void* q, const void* k,
                   const void* v, int32_t total_kv, void* out, float sm_scale, void* workspace,
                   void* stream);

/* Synchronises `stream`, reads and clears the workspace's device error word.  Returns
 * RAE_ERR_DEVICE_TIMEOUT when a kernel gave up a bounded wait since the last check. */
int rae_check_device_status(rae_ctx* ctx, void* workspace, void* stream);

/* Bounded-wait limit of the kernels, in nanoseconds (default 4e9).  A kernel whose wait
 * exceeds it sets the error word, stops its work and exits cleanly. */
int rae_set_wait_timeout_ns(rae_ctx* ctx, int64_t timeout_ns);

/*
 * Kernel timing (instrumentation for measurement).  With max_records > 0, every run call
 * records CUDA events on its stream immediately before and after its attention kernel, for up
 * to max_records calls; max_records == 0 turns it off.  rae_read_kernel_timing synchronises
 * those events, writes the elapsed milliseconds of each recorded call to attn_ms[i] (the split
 * merge runs inside that kernel, so merge_ms[i] is 0), sets *count, and clears the records.
 * Timing adds no work to the kernels, but an event between two kernels serialises their
 * launches: time whole sequences without it.
 */
int rae_enable_kernel_timing(rae_ctx* ctx, int32_t max_records);
int rae_read_kernel_timing(rae_ctx* ctx, float* attn_ms, float* merge_ms, int32_t max,
                           int32_t* count);

/*
 * Host-only plan builders, for inspection and tests: the same validation and tiling as
 * rae_plan_paged / rae_plan_ragged, written into a caller-provided host buffer `image` of
 * image_bytes >= rae_plan_image_bytes bytes, with no CUDA call.  cfg->num_sms must be > 0.
 * The image is int32 words: a 16-word header (magic, kind, num_tiles, num_ctas,
 * num_merge_rows, batch, total_q, block_size, word offsets of the CTA pointer array and of
 * the tiles, the number of split units, word offsets of the four request arrays, the largest
 * rows per unit) followed by those arrays, packed; out->image_words words are used.
 * Tiles are 12 words {request, first KV head, first query token, query tokens, first key,
 * end key, first partial row or -1, split index, arrival counter of the split unit or -1,
 * number of splits of the unit, KV heads of the unit, 0}.  A unit's rows are (token, query
 * head) pairs, token-major, over the query heads of its KV heads.
 */
int rae_plan_paged_host(const rae_config* cfg, const int32_t* qo_indptr,
                        const int32_t* kv_page_indptr, const int32_t* kv_page_indices,
                        const int32_t* kv_len, int32_t batch, int32_t num_pages, void* image,
                        size_t image_bytes, rae_plan* out, char* err, size_t err_len);

int rae_plan_paged_causal_host(const rae_config* cfg, const int32_t* qo_indptr,
                               const int32_t* kv_page_indptr, const int32_t* kv_page_indices,
                               const int32_t* kv_len, int32_t batch, int32_t num_pages,
                               void* image, size_t image_bytes, rae_plan* out, char* err,
                               size_t err_len);

int rae_plan_ragged_host(const rae_config* cfg, const int32_t* cu_q, const int32_t* cu_kv,
                         int32_t num_spans, int32_t block_size, void* image, size_t image_bytes,
                         rae_plan* out, char* err, size_t err_len);

/* Bytes of a host plan image for cfg (no context needed). */
size_t rae_plan_image_bytes_for(const rae_config* cfg);

#ifdef __cplusplus
}
#endif

#endif /* RAE_H_ */
