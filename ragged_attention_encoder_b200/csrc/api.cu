// C ABI of the library (include/rae.h): contexts, plan slots, tensor maps and launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <new>
#include <string>
#include <vector>

#include "kernels.h"
#include "plan.h"
#include "rae.h"

using namespace rae;

namespace {

int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

struct rae_ctx {
  rae_config cfg{};
  int device = 0;
  int64_t image_words = 0;
  int32_t* host_slot[2] = {nullptr, nullptr};   // pinned staging of the plan images
  cudaEvent_t slot_event[2] = {nullptr, nullptr};
  bool slot_pending[2] = {false, false};
  int64_t slot_generation[2] = {-1, -1};
  WriteItem* host_write = nullptr;              // pinned staging of context-write items
  cudaEvent_t write_event = nullptr;
  bool write_pending = false;
  int64_t generation = 0;
  int64_t off_slot[2] = {0, 0};
  int64_t off_write = 0, off_part_o = 0, off_part_lse = 0, off_counters = 0, ws_bytes = 0;
  int64_t timeout_ns = 4000000000LL;
  EncodeTiledFn encode = nullptr;
  std::string last_error;
  // kernel timing records: events [4 * i .. 4 * i + 3] = attn start/stop, merge start/stop
  std::vector<cudaEvent_t> timing_events;
  std::vector<uint8_t> timing_has_merge;
  int32_t timing_max = 0, timing_count = 0;
};

namespace {

int set_err(rae_ctx* ctx, int code, const std::string& msg) {
  if (ctx) ctx->last_error = msg;
  return code;
}

int cuda_err(rae_ctx* ctx, cudaError_t e, const char* what) {
  return set_err(ctx, RAE_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// Waits for the previous host->device copy out of a pinned staging buffer.
int wait_staging(rae_ctx* ctx, cudaEvent_t ev, bool* pending) {
  if (!*pending) return RAE_OK;
  cudaError_t e = cudaEventSynchronize(ev);
  if (e != cudaSuccess) return cuda_err(ctx, e, "cudaEventSynchronize");
  *pending = false;
  return RAE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

DevPlan dev_plan(const rae_ctx* ctx, const rae_plan* plan, void* workspace) {
  const int32_t* img = reinterpret_cast<const int32_t*>(static_cast<uint8_t*>(workspace) +
                                                        ctx->off_slot[plan->slot]);
  DevPlan d;
  d.cta_ptr = img + plan->off_cta_ptr;
  d.tiles = reinterpret_cast<const Tile*>(img + plan->off_tiles);
  d.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + ctx->off_counters);
  d.a = img + plan->off_a;
  d.b = img + plan->off_b;
  d.c = img + plan->off_c;
  d.d = img + plan->off_d;
  d.num_ctas = plan->num_ctas;
  d.block_size = plan->block_size;
  return d;
}

Geometry geometry(const rae_config& c) {
  Geometry g;
  g.hq = c.num_qo_heads;
  g.hkv = c.num_kv_heads;
  g.g = c.num_qo_heads / c.num_kv_heads;
  g.d = c.head_dim;
  g.page_size = c.page_size;
  return g;
}

int make_map(rae_ctx* ctx, CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
             const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = ctx->encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cuuint32_t(rank),
                           const_cast<void*>(base), dims, strides_bytes, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_err(ctx, RAE_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string(int(r)));
  return RAE_OK;
}

// Q (and ragged K/V) as a 3D tensor {d, heads, tokens}.
int map_3d(rae_ctx* ctx, CUtensorMap* map, const void* base, int d, int heads, int tokens,
           int box_heads, int box_tokens) {
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(heads), cuuint64_t(tokens > 0 ? tokens : 1)};
  const cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(heads) * d * 2};
  const cuuint32_t box[3] = {64, cuuint32_t(box_heads), cuuint32_t(box_tokens)};
  return make_map(ctx, map, base, 3, dims, strides, box);
}

// A paged pool as a 2D tensor {d, pages * Hkv * P}.
int map_pool(rae_ctx* ctx, CUtensorMap* map, const void* base, int d, int64_t rows, int page) {
  const cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows > 0 ? rows : 1)};
  const cuuint64_t strides[1] = {cuuint64_t(d) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(page)};
  return make_map(ctx, map, base, 2, dims, strides, box);
}

int check_plan(rae_ctx* ctx, const rae_plan* plan, bool paged) {
  if (!plan) return set_err(ctx, RAE_ERR_INVALID_ARG, "plan is NULL");
  if (plan->slot != 0 && plan->slot != 1) return set_err(ctx, RAE_ERR_INVALID_ARG, "bad plan slot");
  if (ctx->slot_generation[plan->slot] != plan->generation)
    return set_err(ctx, RAE_ERR_INVALID_ARG, "plan slot was re-planned since this plan was made");
  const bool is_paged = plan->kind == kKindDecodeSimt || plan->kind == kKindTcPaged ||
                        plan->kind == kKindTcPagedSwap;
  const bool is_ragged = plan->kind == kKindTcRagged;
  if (paged ? !is_paged : !is_ragged)
    return set_err(ctx, RAE_ERR_INVALID_ARG, "plan kind does not match the run call");
  return RAE_OK;
}

// Event pair around one kernel of the current run (nullptr when timing is off or full).
cudaEvent_t timing_event(rae_ctx* ctx, int which) {
  if (ctx->timing_count >= ctx->timing_max) return nullptr;
  return ctx->timing_events[size_t(ctx->timing_count) * 4 + which];
}

void record(cudaEvent_t ev, cudaStream_t st) {
  if (ev) cudaEventRecord(ev, st);
}

float scale_log2_of(const rae_ctx* ctx, float sm_scale) {
  const float s = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt(float(ctx->cfg.head_dim));
  return s * 1.4426950408889634f;   // log2(e): scores are exponentiated with exp2
}

// Stops the attention-kernel timer and closes the record (the split-KV merge runs inside
// the attention kernels).
int finish_run(rae_ctx* ctx, cudaStream_t st) {
  record(timing_event(ctx, 1), st);
  if (ctx->timing_count < ctx->timing_max) {
    ctx->timing_has_merge[size_t(ctx->timing_count)] = 0;
    ++ctx->timing_count;
  }
  return RAE_OK;
}

int stage_plan(rae_ctx* ctx, int32_t slot, void* workspace, void* stream, rae_plan* out,
               int rc) {
  if (rc) return rc;
  const size_t bytes = size_t(out->image_words) * sizeof(int32_t);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(static_cast<uint8_t*>(workspace) + ctx->off_slot[slot],
                                  ctx->host_slot[slot], bytes, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_err(ctx, e, "plan copy");
  e = cudaEventRecord(ctx->slot_event[slot], st);
  if (e != cudaSuccess) return cuda_err(ctx, e, "cudaEventRecord");
  ctx->slot_pending[slot] = true;
  out->slot = slot;
  out->generation = ++ctx->generation;
  ctx->slot_generation[slot] = out->generation;
  return RAE_OK;
}

}  // namespace

extern "C" {

int rae_create(rae_ctx** out, const rae_config* cfg_in) {
  if (!out || !cfg_in) return RAE_ERR_INVALID_ARG;
  rae_config cfg = *cfg_in;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return RAE_ERR_CUDA;
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return RAE_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return RAE_ERR_UNSUPPORTED;
  if (cfg.num_sms <= 0) cfg.num_sms = prop.multiProcessorCount;
  std::string msg;
  int rc = check_config(cfg, &msg);
  if (rc) return rc;

  rae_ctx* ctx = new (std::nothrow) rae_ctx();
  if (!ctx) return RAE_ERR_CAPACITY;
  ctx->cfg = cfg;
  ctx->device = dev;
  ctx->image_words = image_words_for(cfg);
  const int64_t image_bytes = align256(ctx->image_words * 4);
  const int64_t write_bytes = align256(int64_t(cfg.max_kv_pages) * int64_t(sizeof(WriteItem)));
  int64_t off = kErrWordsBytes;
  ctx->off_slot[0] = off;
  off += image_bytes;
  ctx->off_slot[1] = off;
  off += image_bytes;
  ctx->off_write = off;
  off += write_bytes;
  ctx->off_part_o = off;
  off += align256(int64_t(cfg.max_partial_rows) * cfg.head_dim * 4);
  ctx->off_part_lse = off;
  off += align256(int64_t(cfg.max_partial_rows) * 4);
  ctx->off_counters = off;
  off += align256(int64_t(cfg.max_tiles) * 4);
  ctx->ws_bytes = off;

  bool ok = true;
  for (int s = 0; s < 2 && ok; ++s) {
    ok = cudaMallocHost(&ctx->host_slot[s], size_t(image_bytes)) == cudaSuccess &&
         cudaEventCreateWithFlags(&ctx->slot_event[s], cudaEventDisableTiming) == cudaSuccess;
  }
  ok = ok && cudaMallocHost(&ctx->host_write, size_t(write_bytes)) == cudaSuccess &&
       cudaEventCreateWithFlags(&ctx->write_event, cudaEventDisableTiming) == cudaSuccess;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  ok = ok && cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
       q == cudaDriverEntryPointSuccess && fn;
  if (!ok) {
    rae_destroy(ctx);
    return RAE_ERR_CUDA;
  }
  ctx->encode = reinterpret_cast<EncodeTiledFn>(fn);
  *out = ctx;
  return RAE_OK;
}

int rae_destroy(rae_ctx* ctx) {
  if (!ctx) return RAE_ERR_INVALID_ARG;
  for (int s = 0; s < 2; ++s) {
    if (ctx->slot_event[s]) {
      cudaEventSynchronize(ctx->slot_event[s]);
      cudaEventDestroy(ctx->slot_event[s]);
    }
    if (ctx->host_slot[s]) cudaFreeHost(ctx->host_slot[s]);
  }
  if (ctx->write_event) {
    cudaEventSynchronize(ctx->write_event);
    cudaEventDestroy(ctx->write_event);
  }
  if (ctx->host_write) cudaFreeHost(ctx->host_write);
  for (cudaEvent_t ev : ctx->timing_events) cudaEventDestroy(ev);
  delete ctx;
  return RAE_OK;
}

const char* rae_last_error(const rae_ctx* ctx) {
  if (!ctx) return rae::noalloc_last_error();
  return ctx->last_error.c_str();
}

size_t rae_workspace_bytes(const rae_ctx* ctx) { return ctx ? size_t(ctx->ws_bytes) : 0; }

size_t rae_plan_image_bytes(const rae_ctx* ctx) {
  return ctx ? size_t(ctx->image_words) * sizeof(int32_t) : 0;
}

size_t rae_plan_image_bytes_for(const rae_config* cfg) {
  if (!cfg) return 0;
  std::string msg;
  if (check_config(*cfg, &msg)) return 0;
  return size_t(image_words_for(*cfg)) * sizeof(int32_t);
}

int rae_set_wait_timeout_ns(rae_ctx* ctx, int64_t timeout_ns) {
  if (!ctx || timeout_ns <= 0) return RAE_ERR_INVALID_ARG;
  ctx->timeout_ns = timeout_ns;
  return RAE_OK;
}

}  // extern "C"

namespace {

// The context write and the append: the tokens of request b (rows cu_src[b]..cu_src[b+1]-1
// of k_src / v_src) go to sequence positions start[b]... of its pages (start == nullptr: 0).
// Validates a K/V write, lists its page copies and stages them in the workspace on `stream`;
// *dev_items / *num_items describe the staged list (num_items 0: nothing to write).
int stage_write_items(rae_ctx* ctx, const int32_t* cu_src, const int32_t* page_indptr,
                      const int32_t* page_indices, const int32_t* start, int32_t batch,
                      int32_t num_pages, void* workspace, cudaStream_t st,
                      WriteItem** dev_items, int64_t* num_items) {
  int rc = wait_staging(ctx, ctx->write_event, &ctx->write_pending);
  if (rc) return rc;
  std::string msg;
  int64_t n = 0;
  rc = build_write_items(ctx->cfg, cu_src, page_indptr, page_indices, start, batch, num_pages,
                         ctx->host_write, ctx->cfg.max_kv_pages, &n, &msg);
  if (rc) return set_err(ctx, rc, msg);
  *num_items = n;
  *dev_items = reinterpret_cast<WriteItem*>(static_cast<uint8_t*>(workspace) + ctx->off_write);
  if (n == 0) return RAE_OK;
  cudaError_t e = cudaMemcpyAsync(*dev_items, ctx->host_write, size_t(n) * sizeof(WriteItem),
                                  cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_err(ctx, e, "write items copy");
  e = cudaEventRecord(ctx->write_event, st);
  if (e != cudaSuccess) return cuda_err(ctx, e, "cudaEventRecord");
  ctx->write_pending = true;
  return RAE_OK;
}

int write_kv(rae_ctx* ctx, const void* k_src, const void* v_src, const int32_t* cu_src,
             const int32_t* page_indptr, const int32_t* page_indices, const int32_t* start,
             int32_t batch, void* k_pool, void* v_pool, int32_t num_pages, void* workspace,
             void* stream) {
  if (!ctx) return RAE_ERR_INVALID_ARG;
  if (!workspace || !k_pool || !v_pool || ((!k_src || !v_src) && batch > 0 && cu_src && cu_src[batch] > 0))
    return set_err(ctx, RAE_ERR_INVALID_ARG, "NULL device pointer");
  if (!aligned16(k_src) || !aligned16(v_src) || !aligned16(k_pool) || !aligned16(v_pool))
    return set_err(ctx, RAE_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WriteItem* dev_items = nullptr;
  int64_t n = 0;
  int rc = stage_write_items(ctx, cu_src, page_indptr, page_indices, start, batch, num_pages,
                             workspace, st, &dev_items, &n);
  if (rc || n == 0) return rc;
  cudaError_t e = launch_context_write(dev_items, n, k_src, v_src, k_pool, v_pool, geometry(ctx->cfg), st);
  if (e != cudaSuccess) return cuda_err(ctx, e, "context write launch");
  return RAE_OK;
}

}  // namespace

extern "C" {

int rae_write_context(rae_ctx* ctx, const void* k_src, const void* v_src, const int32_t* cu_enc,
                      const int32_t* page_indptr, const int32_t* page_indices, int32_t batch,
                      void* k_pool, void* v_pool, int32_t num_pages, void* workspace,
                      void* stream) {
  return write_kv(ctx, k_src, v_src, cu_enc, page_indptr, page_indices, nullptr, batch, k_pool,
                  v_pool, num_pages, workspace, stream);
}

int rae_project_write_context(rae_ctx* ctx, const void* hidden, int32_t hidden_dim,
                              const void* w_k, const void* b_k, const void* w_v, const void* b_v,
                              const int32_t* cu_enc, const int32_t* page_indptr,
                              const int32_t* page_indices, int32_t batch, void* k_pool,
                              void* v_pool, int32_t num_pages, void* workspace, void* stream) {
  if (!ctx) return RAE_ERR_INVALID_ARG;
  const rae_config& c = ctx->cfg;
  const int32_t n_half = c.num_kv_heads * c.head_dim;
  if (hidden_dim <= 0 || hidden_dim % 64 != 0 || n_half % 128 != 0)
    return set_err(ctx, RAE_ERR_UNSUPPORTED,
                   "projection needs hidden_dim % 64 == 0 and num_kv_heads * head_dim % 128 == 0");
  if (!workspace || !k_pool || !v_pool || !w_k || !w_v)
    return set_err(ctx, RAE_ERR_INVALID_ARG, "NULL device pointer");
  if (!aligned16(hidden) || !aligned16(w_k) || !aligned16(w_v) || !aligned16(b_k) ||
      !aligned16(b_v) || !aligned16(k_pool) || !aligned16(v_pool))
    return set_err(ctx, RAE_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  if (batch < 0 || (batch > 0 && !cu_enc)) return set_err(ctx, RAE_ERR_INVALID_ARG, "bad cu_enc");
  const int64_t m = batch > 0 ? cu_enc[batch] : 0;
  if (m > int64_t(65535) * 128) return set_err(ctx, RAE_ERR_CAPACITY, "more than 8388480 tokens");
  if (m > 0 && !hidden) return set_err(ctx, RAE_ERR_INVALID_ARG, "NULL hidden states");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WriteItem* dev_items = nullptr;
  int64_t n = 0;
  int rc = stage_write_items(ctx, cu_enc, page_indptr, page_indices, nullptr, batch, num_pages,
                             workspace, st, &dev_items, &n);
  if (rc || n == 0) return rc;
  ProjectWriteArgs a;
  {
    const cuuint64_t dims[2] = {cuuint64_t(hidden_dim), cuuint64_t(m)};
    const cuuint64_t strides[1] = {cuuint64_t(hidden_dim) * 2};
    const cuuint32_t box[2] = {64, 128};
    if ((rc = make_map(ctx, &a.maps[0], hidden, 2, dims, strides, box))) return rc;
  }
  for (int w = 0; w < 2; ++w) {
    const cuuint64_t dims[2] = {cuuint64_t(hidden_dim), cuuint64_t(n_half)};
    const cuuint64_t strides[1] = {cuuint64_t(hidden_dim) * 2};
    const cuuint32_t box[2] = {64, cuuint32_t(project_write_tile_cols(n_half))};
    if ((rc = make_map(ctx, &a.maps[1 + w], w ? w_v : w_k, 2, dims, strides, box))) return rc;
  }
  a.bias_k = b_k;
  a.bias_v = b_v;
  a.items = dev_items;
  a.num_items = n;
  a.k_pool = k_pool;
  a.v_pool = v_pool;
  a.err = reinterpret_cast<int*>(workspace);
  a.timeout_ns = ctx->timeout_ns;
  a.m = int32_t(m);
  a.hidden = hidden_dim;
  a.geo = geometry(c);
  cudaError_t e = launch_project_write(a, st);
  if (e != cudaSuccess) return cuda_err(ctx, e, "projection kernel launch");
  return RAE_OK;
}

int rae_o_proj_partial(rae_ctx* ctx, const void* attn, int32_t m, int32_t k, const void* w_o,
                       int32_t n, const void* bias, void* out, void* workspace, void* stream) {
  if (!ctx) return RAE_ERR_INVALID_ARG;
  if (m < 0 || k <= 0 || n <= 0) return set_err(ctx, RAE_ERR_INVALID_ARG, "bad o_proj sizes");
  if (k % 64 != 0 || n % o_proj_tile_cols() != 0)
    return set_err(ctx, RAE_ERR_UNSUPPORTED, "o_proj needs k % 64 == 0 and n % 128 == 0");
  if (m > int64_t(65535) * 128) return set_err(ctx, RAE_ERR_CAPACITY, "more than 8388480 rows");
  if (m == 0) return RAE_OK;
  if (!attn || !w_o || !out || !workspace)
    return set_err(ctx, RAE_ERR_INVALID_ARG, "NULL device pointer");
  if (!aligned16(attn) || !aligned16(w_o) || !aligned16(bias) || !aligned16(out))
    return set_err(ctx, RAE_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  OProjArgs a;
  int rc;
  {
    const cuuint64_t dims[2] = {cuuint64_t(k), cuuint64_t(m)};
    const cuuint64_t strides[1] = {cuuint64_t(k) * 2};
    const cuuint32_t box[2] = {64, 128};
    if ((rc = make_map(ctx, &a.maps[0], attn, 2, dims, strides, box))) return rc;
  }
  {
    const cuuint64_t dims[2] = {cuuint64_t(k), cuuint64_t(n)};
    const cuuint64_t strides[1] = {cuuint64_t(k) * 2};
    const cuuint32_t box[2] = {64, cuuint32_t(o_proj_tile_cols())};
    if ((rc = make_map(ctx, &a.maps[1], w_o, 2, dims, strides, box))) return rc;
  }
  a.bias = bias;
  a.out = out;
  a.err = reinterpret_cast<int*>(workspace);
  a.timeout_ns = ctx->timeout_ns;
  a.m = m;
  a.n = n;
  a.k = k;
  cudaError_t e = launch_o_proj(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_err(ctx, e, "o_proj kernel launch");
  return RAE_OK;
}

int rae_append_kv(rae_ctx* ctx, const void* k_new, const void* v_new,
                  const int32_t* append_indptr, const int32_t* kv_page_indptr,
                  const int32_t* kv_page_indices, const int32_t* kv_len, int32_t batch,
                  void* k_pool, void* v_pool, int32_t num_pages, void* workspace, void* stream) {
  if (!ctx) return RAE_ERR_INVALID_ARG;
  if (batch < 0) return set_err(ctx, RAE_ERR_INVALID_ARG, "batch < 0");
  if (batch > ctx->cfg.max_batch) return set_err(ctx, RAE_ERR_CAPACITY, "batch > max_batch");
  if (batch > 0 && (!append_indptr || !kv_len))
    return set_err(ctx, RAE_ERR_INVALID_ARG, "append_indptr or kv_len is NULL");
  std::vector<int32_t> start(size_t(batch > 0 ? batch : 0));
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t n = append_indptr[b + 1] - append_indptr[b];
    if (n < 0) return set_err(ctx, RAE_ERR_INVALID_ARG, "append_indptr decreases");
    if (n > kv_len[b])
      return set_err(ctx, RAE_ERR_INVALID_ARG,
                     "request " + std::to_string(b) + " appends more tokens than kv_len holds");
    start[size_t(b)] = kv_len[b] - n;
  }
  return write_kv(ctx, k_new, v_new, append_indptr, kv_page_indptr, kv_page_indices,
                  start.data(), batch, k_pool, v_pool, num_pages, workspace, stream);
}

int rae_plan_paged(rae_ctx* ctx, int32_t slot, const int32_t* qo_indptr,
                   const int32_t* kv_page_indptr, const int32_t* kv_page_indices,
                   const int32_t* kv_len, int32_t batch, int32_t num_pages, void* workspace,
                   void* stream, rae_plan* out) {
  if (!ctx) return RAE_ERR_INVALID_ARG;
  if (slot != 0 && slot != 1) return set_err(ctx, RAE_ERR_INVALID_ARG, "slot must be 0 or 1");
  if (!workspace || !out) return set_err(ctx, RAE_ERR_INVALID_ARG, "NULL workspace or out");
  int rc = wait_staging(ctx, ctx->slot_event[slot], &ctx->slot_pending[slot]);
  if (rc) return rc;
  std::string msg;
  rae_plan plan{};
  rc = build_paged_plan(ctx->cfg, qo_indptr, kv_page_indptr, kv_page_indices, kv_len, batch,
                        num_pages, ctx->host_slot[slot], ctx->image_words, &plan, &msg);
  if (rc) return set_err(ctx, rc, msg);
  rc = stage_plan(ctx, slot, workspace, stream, &plan, rc);
  if (rc) return rc;
  *out = plan;
  return RAE_OK;
}

int rae_plan_paged_causal(rae_ctx* ctx, int32_t slot, const int32_t* qo_indptr,
                          const int32_t* kv_page_indptr, const int32_t* kv_page_indices,
                          const int32_t* kv_len, int32_t batch, int32_t num_pages,
                          void* workspace, void* stream, rae_plan* out) {
  if (!ctx) return RAE_ERR_INVALID_ARG;
  if (slot != 0 && slot != 1) return set_err(ctx, RAE_ERR_INVALID_ARG, "slot must be 0 or 1");
  if (!workspace || !out) return set_err(ctx, RAE_ERR_INVALID_ARG, "NULL workspace or out");
  int rc = wait_staging(ctx, ctx->slot_event[slot], &ctx->slot_pending[slot]);
  if (rc) return rc;
  std::string msg;
  rae_plan plan{};
  rc = build_paged_plan(ctx->cfg, qo_indptr, kv_page_indptr, kv_page_indices, kv_len, batch,
                        num_pages, ctx->host_slot[slot], ctx->image_words, &plan, &msg, true);
  if (rc) return set_err(ctx, rc, msg);
  rc = stage_plan(ctx, slot, workspace, stream, &plan, rc);
  if (rc) return rc;
  *out = plan;
  return RAE_OK;
}

int rae_plan_ragged(rae_ctx* ctx, int32_t slot, const int32_t* cu_q, const int32_t* cu_kv,
                    int32_t num_spans, int32_t block_size, void* workspace, void* stream,
                    rae_plan* out) {
  if (!ctx) return RAE_ERR_INVALID_ARG;
  if (slot != 0 && slot != 1) return set_err(ctx, RAE_ERR_INVALID_ARG, "slot must be 0 or 1");
  if (!workspace || !out) return set_err(ctx, RAE_ERR_INVALID_ARG, "NULL workspace or out");
  int rc = wait_staging(ctx, ctx->slot_event[slot], &ctx->slot_pending[slot]);
  if (rc) return rc;
  std::string msg;
  rae_plan plan{};
  rc = build_ragged_plan(ctx->cfg, cu_q, cu_kv, num_spans, block_size, ctx->host_slot[slot],
                         ctx->image_words, &plan, &msg);
  if (rc) return set_err(ctx, rc, msg);
  rc = stage_plan(ctx, slot, workspace, stream, &plan, rc);
  if (rc) return rc;
  *out = plan;
  return RAE_OK;
}

int rae_run_paged(rae_ctx* ctx, const rae_plan* plan, const void* q, const void* k_pool,
                  const void* v_pool, int32_t num_pages, void* out, float sm_scale,
                  void* workspace, void* stream) {
  if (!ctx) return RAE_ERR_INVALID_ARG;
  int rc = check_plan(ctx, plan, true);
  if (rc) return rc;
  if (plan->total_q == 0 || plan->num_ctas == 0) return RAE_OK;
  if (!q || !k_pool || !v_pool || !out || !workspace)
    return set_err(ctx, RAE_ERR_INVALID_ARG, "NULL device pointer");
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out))
    return set_err(ctx, RAE_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  if (num_pages <= 0) return set_err(ctx, RAE_ERR_INVALID_ARG, "num_pages must be positive");
  if (num_pages < plan->kv_extent)
    return set_err(ctx, RAE_ERR_INVALID_ARG,
                   "the plan lists page " + std::to_string(plan->kv_extent - 1) + " but the pools hold " +
                       std::to_string(num_pages) + " pages");
  const rae_config& c = ctx->cfg;
  const Geometry geo = geometry(c);
  const DevPlan dp = dev_plan(ctx, plan, workspace);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* part_o = reinterpret_cast<float*>(ws + ctx->off_part_o);
  float* part_lse = reinterpret_cast<float*>(ws + ctx->off_part_lse);
  int* err = reinterpret_cast<int*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float sl2 = scale_log2_of(ctx, sm_scale);
  cudaError_t e;
  if (plan->kind == kKindDecodeSimt) {
    record(timing_event(ctx, 0), st);
    e = launch_decode_simt(dp, geo, q, k_pool, v_pool, out, part_o, part_lse, err, sl2,
                           ctx->timeout_ns, plan->rows_max, st);
    if (e != cudaSuccess) return cuda_err(ctx, e, "decode kernel launch");
  } else if (plan->kind == kKindTcPagedSwap) {
    TcTensors maps;
    const int n_rows = plan->rows_max;
    const int64_t rows = int64_t(num_pages) * c.num_kv_heads * c.page_size;
    if ((rc = map_3d(ctx, &maps.q, q, c.head_dim, c.num_qo_heads, plan->total_q, geo.g, n_rows / geo.g))) return rc;
    if ((rc = map_pool(ctx, &maps.k, k_pool, c.head_dim, rows, c.page_size))) return rc;
    if ((rc = map_pool(ctx, &maps.v, v_pool, c.head_dim, rows, c.page_size))) return rc;
    record(timing_event(ctx, 0), st);
    e = launch_attn_swapab(dp, geo, n_rows, maps, out, part_o, part_lse, err, sl2, ctx->timeout_ns, st);
    if (e != cudaSuccess) return cuda_err(ctx, e, "attention kernel launch");
  } else {
    TcTensors maps;
    const int tpt = kTcRows / geo.g;
    const int64_t rows = int64_t(num_pages) * c.num_kv_heads * c.page_size;
    if ((rc = map_3d(ctx, &maps.q, q, c.head_dim, c.num_qo_heads, plan->total_q, geo.g, tpt))) return rc;
    if ((rc = map_pool(ctx, &maps.k, k_pool, c.head_dim, rows, c.page_size))) return rc;
    if ((rc = map_pool(ctx, &maps.v, v_pool, c.head_dim, rows, c.page_size))) return rc;
    record(timing_event(ctx, 0), st);
    e = launch_attn_tc(dp, geo, true, maps, out, part_o, part_lse, err, sl2, ctx->timeout_ns, st);
    if (e != cudaSuccess) return cuda_err(ctx, e, "attention kernel launch");
  }
  return finish_run(ctx, st);
}

int rae_run_ragged(rae_ctx* ctx, const rae_plan* plan, const void* q, const void* k,
                   const void* v, int32_t total_kv, void* out, float sm_scale, void* workspace,
                   void* stream) {
  if (!ctx) return RAE_ERR_INVALID_ARG;
  int rc = check_plan(ctx, plan, false);
  if (rc) return rc;
  if (plan->total_q == 0 || plan->num_ctas == 0) return RAE_OK;
  if (!q || !k || !v || !out || !workspace)
    return set_err(ctx, RAE_ERR_INVALID_ARG, "NULL device pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return set_err(ctx, RAE_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  if (total_kv < plan->kv_extent)
    return set_err(ctx, RAE_ERR_INVALID_ARG,
                   "the plan reads " + std::to_string(plan->kv_extent) + " key tokens but k and v hold " +
                       std::to_string(total_kv));
  const rae_config& c = ctx->cfg;
  const Geometry geo = geometry(c);
  const DevPlan dp = dev_plan(ctx, plan, workspace);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* part_o = reinterpret_cast<float*>(ws + ctx->off_part_o);
  float* part_lse = reinterpret_cast<float*>(ws + ctx->off_part_lse);
  int* err = reinterpret_cast<int*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  TcTensors maps;
  const int tpt = kTcRows / geo.g;
  if ((rc = map_3d(ctx, &maps.q, q, c.head_dim, c.num_qo_heads, plan->total_q, geo.g, tpt))) return rc;
  if ((rc = map_3d(ctx, &maps.k, k, c.head_dim, c.num_kv_heads, total_kv, 1, kTcRows))) return rc;
  if ((rc = map_3d(ctx, &maps.v, v, c.head_dim, c.num_kv_heads, total_kv, 1, kTcRows))) return rc;
  record(timing_event(ctx, 0), st);
  cudaError_t e = launch_attn_tc(dp, geo, false, maps, out, part_o, part_lse, err,
                                 scale_log2_of(ctx, sm_scale), ctx->timeout_ns, st);
  if (e != cudaSuccess) return cuda_err(ctx, e, "attention kernel launch");
  return finish_run(ctx, st);
}

int rae_check_device_status(rae_ctx* ctx, void* workspace, void* stream) {
  if (!ctx || !workspace) return RAE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_err(ctx, e, "status read");
  if (word != 0) {
    // A kernel that gave up may have left split arrival counters behind: clear them too.
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    e = cudaMemsetAsync(ws, 0, sizeof(int), st);
    if (e == cudaSuccess)
      e = cudaMemsetAsync(ws + ctx->off_counters, 0, size_t(ctx->cfg.max_tiles) * 4, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_err(ctx, e, "status clear");
    return set_err(ctx, RAE_ERR_DEVICE_TIMEOUT,
                   "a kernel gave up a bounded wait (site " + std::to_string(word) + ")");
  }
  return RAE_OK;
}

int rae_enable_kernel_timing(rae_ctx* ctx, int32_t max_records) {
  if (!ctx || max_records < 0) return RAE_ERR_INVALID_ARG;
  for (cudaEvent_t ev : ctx->timing_events) cudaEventDestroy(ev);
  ctx->timing_events.clear();
  ctx->timing_max = 0;
  ctx->timing_count = 0;
  ctx->timing_events.resize(size_t(max_records) * 4, nullptr);
  for (auto& ev : ctx->timing_events) {
    cudaError_t e = cudaEventCreate(&ev);
    if (e != cudaSuccess) return cuda_err(ctx, e, "cudaEventCreate");
  }
  ctx->timing_has_merge.assign(size_t(max_records), 0);
  ctx->timing_max = max_records;
  return RAE_OK;
}

int rae_read_kernel_timing(rae_ctx* ctx, float* attn_ms, float* merge_ms, int32_t max,
                           int32_t* count) {
  if (!ctx || !count || max < 0) return RAE_ERR_INVALID_ARG;
  const int32_t n = std::min(ctx->timing_count, max);
  for (int32_t i = 0; i < n; ++i) {
    cudaEvent_t* ev = &ctx->timing_events[size_t(i) * 4];
    cudaError_t e = cudaEventSynchronize(ev[1]);
    float a = 0.f, m = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&a, ev[0], ev[1]);
    if (e == cudaSuccess && ctx->timing_has_merge[size_t(i)]) {
      e = cudaEventSynchronize(ev[3]);
      if (e == cudaSuccess) e = cudaEventElapsedTime(&m, ev[2], ev[3]);
    }
    if (e != cudaSuccess) return cuda_err(ctx, e, "kernel timing");
    if (attn_ms) attn_ms[i] = a;
    if (merge_ms) merge_ms[i] = m;
  }
  *count = n;
  ctx->timing_count = 0;
  return RAE_OK;
}

int rae_plan_paged_host(const rae_config* cfg, const int32_t* qo_indptr,
                        const int32_t* kv_page_indptr, const int32_t* kv_page_indices,
                        const int32_t* kv_len, int32_t batch, int32_t num_pages, void* image,
                        size_t image_bytes, rae_plan* out, char* err, size_t err_len) {
  if (!cfg || !out) return RAE_ERR_INVALID_ARG;
  std::string msg;
  rae_plan plan{};
  int rc = build_paged_plan(*cfg, qo_indptr, kv_page_indptr, kv_page_indices, kv_len, batch,
                            num_pages, static_cast<int32_t*>(image), int64_t(image_bytes / 4),
                            &plan, &msg);
  if (rc) {
    if (err && err_len) std::snprintf(err, err_len, "%s", msg.c_str());
    return rc;
  }
  *out = plan;
  return RAE_OK;
}

int rae_plan_paged_causal_host(const rae_config* cfg, const int32_t* qo_indptr,
                               const int32_t* kv_page_indptr, const int32_t* kv_page_indices,
                               const int32_t* kv_len, int32_t batch, int32_t num_pages,
                               void* image, size_t image_bytes, rae_plan* out, char* err,
                               size_t err_len) {
  if (!cfg || !out) return RAE_ERR_INVALID_ARG;
  std::string msg;
  rae_plan plan{};
  int rc = build_paged_plan(*cfg, qo_indptr, kv_page_indptr, kv_page_indices, kv_len, batch,
                            num_pages, static_cast<int32_t*>(image), int64_t(image_bytes / 4),
                            &plan, &msg, true);
  if (rc) {
    if (err && err_len) std::snprintf(err, err_len, "%s", msg.c_str());
    return rc;
  }
  *out = plan;
  return RAE_OK;
}

int rae_plan_ragged_host(const rae_config* cfg, const int32_t* cu_q, const int32_t* cu_kv,
                         int32_t num_spans, int32_t block_size, void* image, size_t image_bytes,
                         rae_plan* out, char* err, size_t err_len) {
  if (!cfg || !out) return RAE_ERR_INVALID_ARG;
  std::string msg;
  rae_plan plan{};
  int rc = build_ragged_plan(*cfg, cu_q, cu_kv, num_spans, block_size,
                             static_cast<int32_t*>(image), int64_t(image_bytes / 4), &plan, &msg);
  if (rc) {
    if (err && err_len) std::snprintf(err, err_len, "%s", msg.c_str());
    return rc;
  }
  *out = plan;
  return RAE_OK;
}

}  // extern "C"
