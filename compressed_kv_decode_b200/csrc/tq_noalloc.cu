// tq_decode_attention_noalloc: the decode attention call for callers that may
// not allocate device memory (and so cannot hand in a workspace).  Its
// scratch is a fixed array in device memory owned by the library; the call
// forwards to tq_decode_attention with that array as the workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "tq_internal.h"

namespace {

constexpr size_t kScratchBytes = TQ_NOALLOC_SCRATCH_BYTES;

// Device-side scratch shared by every call.  In host code this name is only a
// stand-in for the symbol, not a device address: the address comes from
// cudaGetSymbolAddress, once per device, below.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Per device: the context the address was looked up in, and the address.  A
// device reset (or any teardown of the primary context) loads the module
// again, possibly at another address, so a cached address is reused only
// while the current context is the one it came from.
void* g_scratch_ctx[kMaxDevices] = {};
void* g_scratch_addr[kMaxDevices] = {};

// cuCtxGetCurrent from the driver, reached through the runtime (no link to
// the driver library); null if the driver does not provide it.
using CtxGetCurrent = int (*)(void**);
CtxGetCurrent ctx_get_current() {
  static const CtxGetCurrent fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetCurrent>(nullptr);
    return reinterpret_cast<CtxGetCurrent>(f);
  }();
  return fn;
}

// Device address of the scratch array on the current device, looked up with
// that device current on the first call and again whenever the current
// context is not the one of the cached lookup (or cannot be told).
tq_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_UNSUPPORTED;
  void* cur = nullptr;
  const CtxGetCurrent get = ctx_get_current();
  const bool known = get != nullptr && get(&cur) == 0 && cur != nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr || !known || g_scratch_ctx[dev] != cur) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return TQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = known ? cur : nullptr;
  }
  *out = g_scratch_addr[dev];
  return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_decode_attention_noalloc(const tq_ctx* ctx, const void* q,
                                                 tq_dtype q_dtype, int B, int Hq, int Hkv,
                                                 float scale, const void* k_hot,
                                                 const void* v_hot, int W_max,
                                                 const int32_t* hot_len,
                                                 const uint8_t* page_pool, int64_t pool_pages,
                                                 const int32_t* page_table, int max_pages,
                                                 const int32_t* cold_len, float* out,
                                                 void* stream) {
  if (!ctx) return TQ_ERR_INVALID_ARG;
  const size_t need = tq_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max);
  if (need == 0) return TQ_ERR_INVALID_ARG;
  if (need > kScratchBytes) return TQ_ERR_CAPACITY;  // the fixed scratch is too small
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
  if (dev != ctx->device) return TQ_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const tq_status st = scratch_address(&scratch);
  if (st != TQ_OK) return st;
  return tq_decode_attention(ctx, q, q_dtype, B, Hq, Hkv, scale, k_hot, v_hot, W_max, hot_len,
                             page_pool, pool_pages, page_table, max_pages, cold_len, out, scratch,
                             kScratchBytes, stream);
}
