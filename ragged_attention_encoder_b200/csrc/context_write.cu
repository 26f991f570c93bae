// Context write: scatters packed encoder K/V [sum_enc, Hkv, d] into the paged pools
// [num_pages, Hkv, P, d] (M* page "mstar.engine.resources.attn.cross": the encode step writes
// the context once as an ordinary KV stream; later steps only read it).
//
// One CTA copies one page's worth of tokens for K and for V.  The source rows of a page are
// one contiguous block of ntok * Hkv * d elements, the destination is the page's Hkv runs of
// ntok * d elements, so both sides move in whole 16-byte vectors with coalesced accesses.
// Each thread issues four iterations' loads before their stores (eight 16-byte loads in
// flight), and both sides stream past L2 (neither is read again soon).
// HBM bound: algorithmic bytes = 2 (K and V) x 2 (read + write) x tokens x Hkv x d x 2 B.
#include <mutex>
#include <string>

#include "kernels.h"
#include "rae.h"

namespace rae {
namespace {

__global__ void __launch_bounds__(256) context_write_kernel(const WriteItem* __restrict__ items,
                                                            const uint4* __restrict__ k_src,
                                                            const uint4* __restrict__ v_src,
                                                            uint4* __restrict__ k_pool,
                                                            uint4* __restrict__ v_pool,
                                                            int32_t hkv, int32_t vec_per_row,
                                                            int32_t page_size) {
  const WriteItem it = items[blockIdx.x];
  const int32_t per_tok = hkv * vec_per_row;          // 16-byte vectors per token (all heads)
  const int32_t n = it.ntok * per_tok;
  const int64_t src0 = int64_t(it.src_row) * per_tok;
  const int64_t page0 = int64_t(it.page) * hkv * page_size * vec_per_row;
  constexpr int U = 4;
  for (int32_t e0 = threadIdx.x; e0 < n; e0 += U * blockDim.x) {
    uint4 kv[U], vv[U];
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const int32_t e = e0 + i * int32_t(blockDim.x);
      if (e < n) {
        kv[i] = __ldcs(k_src + src0 + e);
        vv[i] = __ldcs(v_src + src0 + e);
      }
    }
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const int32_t e = e0 + i * int32_t(blockDim.x);
      if (e < n) {
        const int32_t slot = e / per_tok;
        const int32_t rem = e - slot * per_tok;
        const int32_t h = rem / vec_per_row;
        const int32_t u = rem - h * vec_per_row;
        const int64_t dst = page0 + (int64_t(h) * page_size + it.slot0 + slot) * vec_per_row + u;
        __stcs(k_pool + dst, kv[i]);
        __stcs(v_pool + dst, vv[i]);
      }
    }
  }
}

}  // namespace

cudaError_t launch_context_write(const WriteItem* items, int64_t num_items, const void* k_src,
                                 const void* v_src, void* k_pool, void* v_pool,
                                 const Geometry& geo, cudaStream_t stream) {
  if (num_items == 0) return cudaSuccess;
  context_write_kernel<<<dim3(uint32_t(num_items)), 256, 0, stream>>>(
      items, static_cast<const uint4*>(k_src), static_cast<const uint4*>(v_src),
      static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), geo.hkv, geo.d / 8,
      geo.page_size);
  return cudaGetLastError();
}

}  // namespace rae

// ---------------------------------------------------------------------------------------
// Context write without a caller workspace (rae_write_context_noalloc).
//
// The ordinary call stages its page-copy list in the caller's workspace.  Some callers have
// no way to provide one: a serving engine whose device memory is owned entirely by its own
// pool allocator, or code that must not call cudaMalloc at all (because an allocation would
// stall a latency-critical loop or fall outside the memory budget it was given).  For them
// the list lives in this file-scope device array instead.  Every GPU that loads the library
// holds the array (1 MiB) until the process exits.
namespace rae {
namespace {

constexpr int64_t kNoAllocMaxPages = 65536;   // page copies per call (16 B each)
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) WriteItem g_noalloc_items[kNoAllocMaxPages];

WriteItem g_noalloc_host[kNoAllocMaxPages];            // host-side build of the list
WriteItem* g_noalloc_dev[kNoAllocMaxDevices] = {};     // device address of the array, per GPU
std::mutex g_noalloc_mutex;

}  // namespace
}  // namespace rae

namespace rae {
// Message of the calling thread's last failing rae_write_context_noalloc call (the call has
// no context to keep it in); rae_last_error(NULL) returns it.
thread_local std::string g_noalloc_msg;

const char* noalloc_last_error() {
  return g_noalloc_msg.empty() ? "no context" : g_noalloc_msg.c_str();
}

namespace {
int noalloc_fail(int code, const std::string& msg) {
  g_noalloc_msg = "rae_write_context_noalloc: " + msg;
  return code;
}
}  // namespace
}  // namespace rae

extern "C" int rae_write_context_noalloc(const void* k_src, const void* v_src,
                                         const int32_t* cu_enc, const int32_t* page_indptr,
                                         const int32_t* page_indices, int32_t batch,
                                         void* k_pool, void* v_pool, int32_t num_pages,
                                         int32_t num_kv_heads, int32_t head_dim,
                                         int32_t page_size, void* stream) {
  using namespace rae;
  if (!k_pool || !v_pool) return noalloc_fail(RAE_ERR_INVALID_ARG, "k_pool or v_pool is NULL");
  const uintptr_t mis = reinterpret_cast<uintptr_t>(k_src) | reinterpret_cast<uintptr_t>(v_src) |
                        reinterpret_cast<uintptr_t>(k_pool) | reinterpret_cast<uintptr_t>(v_pool);
  if (mis & 15) return noalloc_fail(RAE_ERR_INVALID_ARG, "a device buffer is not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The page list is copied from one host array that the next call rewrites.  A copy
  // recorded into a graph would read that array when the graph is launched, i.e. a later
  // call's list, so the call refuses to be recorded.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess)
    return noalloc_fail(RAE_ERR_CUDA, "cudaStreamIsCapturing failed");
  if (cap != cudaStreamCaptureStatusNone)
    return noalloc_fail(RAE_ERR_UNSUPPORTED,
                        "the stream is capturing; the page list comes from a host array that "
                        "the next call rewrites");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return noalloc_fail(RAE_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return noalloc_fail(RAE_ERR_UNSUPPORTED, "device ordinal above " + std::to_string(kNoAllocMaxDevices - 1));

  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_dev[dev]) {
    // Once per device, with that device current: the host-side name of the array is only a
    // stand-in, the kernel needs the address the runtime gives for this device.
    void* addr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_items);
    if (e != cudaSuccess || !addr)
      return noalloc_fail(RAE_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    g_noalloc_dev[dev] = static_cast<WriteItem*>(addr);
  }

  rae_config cfg{};
  cfg.num_qo_heads = num_kv_heads;
  cfg.num_kv_heads = num_kv_heads;
  cfg.head_dim = head_dim;
  cfg.page_size = page_size;
  cfg.max_batch = batch > 0 ? batch : 1;
  cfg.max_q_tokens = 1;
  cfg.max_kv_pages = int32_t(kNoAllocMaxPages);
  cfg.max_tiles = 1;
  cfg.max_partial_rows = 0;
  cfg.num_sms = 1;
  int64_t n = 0;
  std::string msg;
  // Sizes beyond kNoAllocMaxPages page copies come back as RAE_ERR_CAPACITY, before any
  // device work.
  int rc = build_write_items(cfg, cu_enc, page_indptr, page_indices, nullptr, batch, num_pages,
                             g_noalloc_host, kNoAllocMaxPages, &n, &msg);
  if (rc) {
    if (rc == RAE_ERR_CAPACITY)
      msg += " (at most " + std::to_string(kNoAllocMaxPages) + " page copies per call)";
    return noalloc_fail(rc, msg);
  }
  if (n == 0) return RAE_OK;
  if (!k_src || !v_src) return noalloc_fail(RAE_ERR_INVALID_ARG, "k_src or v_src is NULL");
  // From pageable host memory: the call returns once the list has been staged, so the host
  // array may be rebuilt by the next call.
  cudaError_t e = cudaMemcpyAsync(g_noalloc_dev[dev], g_noalloc_host,
                                  size_t(n) * sizeof(WriteItem), cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess)
    return noalloc_fail(RAE_ERR_CUDA, std::string("cudaMemcpyAsync: ") + cudaGetErrorString(e));
  Geometry geo;
  geo.hq = num_kv_heads;
  geo.hkv = num_kv_heads;
  geo.g = 1;
  geo.d = head_dim;
  geo.page_size = page_size;
  e = launch_context_write(g_noalloc_dev[dev], n, k_src, v_src, k_pool, v_pool, geo, st);
  if (e != cudaSuccess)
    return noalloc_fail(RAE_ERR_CUDA, std::string("launch: ") + cudaGetErrorString(e));
  return RAE_OK;
}
