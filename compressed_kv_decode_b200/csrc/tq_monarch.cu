// One decode step of Monarch's hot/cold cache ("Monarch v3: NES-inspiriertes
// KV-Paging", openclawradar.com, sections "Wie es funktioniert" and
// "Vereinfachte Decode-Schleife"): the step's token joins the hot window,
// attention scores the hot tokens and reads the cold pages only where the
// largest raw hot score is below the threshold, and the oldest hot tokens are
// compressed into the cold pages once the window holds window + E of them.
//
// Launches, all on the caller's stream:
//   append      one CTA per sequence: the new K, V rows of every kv head into
//               the ring slot (hot_start + hot_len) mod W_max; hot_len + 1
//   decode      the gated decode (gate, prep, split-K attention, combine)
//   gather      one CTA per (sequence, kv head): the E oldest hot rows of a
//               sequence due for eviction into a contiguous staging tile;
//               per-sequence counts (E or 0)
//   compress    the tensor-core compress/append on the staging tiles, with
//               the per-sequence counts (sequences with 0 write nothing; CTAs
//               without a tile leave at once)
//   finish      cold_len += n, hot_len -= n, hot_start += n (mod W_max)
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace mon {

__global__ void __launch_bounds__(256) append_kernel(const uint4* __restrict__ k_new,
                                                     const uint4* __restrict__ v_new,
                                                     uint4* k_hot, uint4* v_hot, int Hkv,
                                                     int row_chunks, int W_max,
                                                     const int32_t* hot_start, int32_t* hot_len,
                                                     int* err) {
  const int b = blockIdx.x;
  const int len = hot_len[b], start = hot_start[b];
  if (len < 0 || len >= W_max || start < 0 || start >= W_max) {
    if (threadIdx.x == 0) report(err, TQ_ERR_CAPACITY);  // the window is full: token dropped
    return;
  }
  int slot = start + len;
  if (slot >= W_max) slot -= W_max;
  const int per = Hkv * row_chunks;  // 16-byte chunks of one sequence's new K (or V)
  for (int i = threadIdx.x; i < 2 * per; i += blockDim.x) {
    const int isv = i >= per, c = isv ? i - per : i;
    const int h = c / row_chunks, ch = c % row_chunks;
    const size_t src = (static_cast<size_t>(b) * Hkv + h) * row_chunks + ch;
    const size_t dst = ((static_cast<size_t>(b) * Hkv + h) * W_max + slot) * row_chunks + ch;
    if (isv) v_hot[dst] = v_new[src];
    else k_hot[dst] = k_new[src];
  }
  __syncthreads();  // every thread has read hot_len
  if (threadIdx.x == 0) hot_len[b] = len + 1;
}

__global__ void __launch_bounds__(256) gather_kernel(const uint4* __restrict__ k_hot,
                                                     const uint4* __restrict__ v_hot,
                                                     uint4* k_stage, uint4* v_stage, int Hkv,
                                                     int row_chunks, int W_max, int window, int E,
                                                     const int32_t* hot_start,
                                                     const int32_t* hot_len, int32_t* n_evict) {
  const int bh = blockIdx.x, b = bh / Hkv;
  const int len = hot_len[b];
  int start = hot_start[b];
  if (start < 0 || start >= W_max) start = 0;  // reported by the attention step
  const bool ev = len >= window + E && len <= W_max;
  if (threadIdx.x == 0 && bh % Hkv == 0) n_evict[b] = ev ? E : 0;
  if (!ev) return;
  const int per = E * row_chunks;
  for (int i = threadIdx.x; i < 2 * per; i += blockDim.x) {
    const int isv = i >= per, c = isv ? i - per : i;
    const int r = c / row_chunks, ch = c % row_chunks;
    int slot = start + r;
    if (slot >= W_max) slot -= W_max;
    const size_t src = (static_cast<size_t>(bh) * W_max + slot) * row_chunks + ch;
    const size_t dst = (static_cast<size_t>(bh) * E + r) * row_chunks + ch;
    if (isv) v_stage[dst] = v_hot[src];
    else k_stage[dst] = k_hot[src];
  }
}

__global__ void finish_kernel(int B, int W_max, const int32_t* n_evict, int32_t* hot_start,
                              int32_t* hot_len, int32_t* cold_len) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x) {
    const int n = n_evict[b];
    if (n == 0) continue;
    cold_len[b] += n;
    hot_len[b] -= n;
    int s = hot_start[b];
    s = (s >= 0 && s < W_max) ? s + n : n;
    hot_start[b] = s >= W_max ? s - W_max : s;
  }
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace mon

size_t monarch_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_pages,
                               int W_max, int evict_block) {
  const size_t dec = decode_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max);
  if (dec == 0 || evict_block <= 0) return 0;
  const size_t stage = static_cast<size_t>(B) * Hkv * evict_block * ctx->cfg.head_dim * 2;
  return mon::align256(dec) + 2 * mon::align256(stage) + mon::align256(sizeof(int32_t) * B);
}

int launch_monarch_step(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq, int Hkv,
                        float scale, const void* k_new, const void* v_new, void* k_hot,
                        void* v_hot, int W_max, int32_t* hot_start, int32_t* hot_len,
                        uint8_t* pool, int64_t pool_pages, const int32_t* page_table,
                        int max_pages, int32_t* cold_len, float threshold, int window,
                        int evict_block, int32_t* cold_used, float* out, void* ws,
                        size_t ws_bytes, void* stream) {
  const int d = ctx->cfg.head_dim;
  const int E = evict_block;
  const size_t dec = decode_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max);
  const size_t stage = static_cast<size_t>(B) * Hkv * E * d * 2;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* k_stage = base + mon::align256(dec);
  uint8_t* v_stage = k_stage + mon::align256(stage);
  int32_t* n_evict = reinterpret_cast<int32_t*>(v_stage + mon::align256(stage));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int row_chunks = d / 8;
  if (k_new) {
    mon::append_kernel<<<B, 256, 0, st>>>(static_cast<const uint4*>(k_new),
                                          static_cast<const uint4*>(v_new),
                                          static_cast<uint4*>(k_hot), static_cast<uint4*>(v_hot),
                                          Hkv, row_chunks, W_max, hot_start, hot_len,
                                          ctx->dev.err);
    if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  }
  const DecodeGate gate{threshold, cold_used};
  int rc = launch_decode(ctx, q, q_dtype, B, Hq, Hkv, scale, k_hot, v_hot, W_max, hot_start,
                         hot_len, pool, pool_pages, page_table, max_pages, cold_len, &gate, out,
                         ws, dec, stream);
  if (rc != TQ_OK) return rc;
  mon::gather_kernel<<<B * Hkv, 256, 0, st>>>(
      static_cast<const uint4*>(k_hot), static_cast<const uint4*>(v_hot),
      reinterpret_cast<uint4*>(k_stage), reinterpret_cast<uint4*>(v_stage), Hkv, row_chunks, W_max,
      window, E, hot_start, hot_len, n_evict);
  if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  rc = launch_compress_tc(ctx, k_stage, v_stage, false, B, Hkv, E, pool, pool_pages, page_table,
                          max_pages, cold_len, stream, n_evict);
  if (rc != TQ_OK) return rc;
  mon::finish_kernel<<<(B + 127) / 128, 128, 0, st>>>(B, W_max, n_evict, hot_start, hot_len,
                                                     cold_len);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace tq
