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
//   promote     (with promotion) one CTA per sequence: per cold position the
//               largest attention weight over the query heads that read the
//               cold tier, from the attention's logits and the combine's
//               log-sum-exp; consecutive counts; positions that reach the
//               sticky count are masked and their decompressed records
//               (n Pi^T c_hat for K, n_v Pi^T c_hat_v for V, fp16) appended to
//               the ring of every kv head
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

constexpr int PROMO_THREADS = 256;
constexpr int PROMO_MAX = TQ_PROMOTE_MAX_PER_STEP;

struct PromoParams {
  int Hq, Hkv, W_max, max_pages;
  float thr;
  int sticky, max_per_step;
  const float* logits;  // [B][Hq][cap]
  const float* lse;     // [B][Hq]
  uint32_t* mask;       // [B][cap / 32]
  uint8_t* counts;      // [B][cap]
  const uint8_t* pool;
  long long pool_pages, page_bytes;
  int blk, off_h, off_l, off_vc, off_nk, off_vn;
  const int32_t* page_table;
  const int32_t* cold_len;
  const int32_t* hot_start;
  int32_t* hot_len;
  __half* k_hot;
  __half* v_hot;
  const float* rot;  // Pi [D][D], row-major (x_rot = Pi x)
  float kc0, kc1;
  float vc[8];
  int* err;
};

// Promotion (see the launch list above), one CTA per sequence.
template <int D>
__global__ void __launch_bounds__(PROMO_THREADS) promote_kernel(PromoParams p) {
  const int b = blockIdx.x, tid = threadIdx.x;
  const int cap = p.max_pages * TQ_PAGE_TOKENS;
  __shared__ int chosen[PROMO_MAX];
  __shared__ int s_count, s_hl;
  __shared__ int wsum[PROMO_THREADS / 32];
  __shared__ float ck[D], cv[D];
  const int cl = min(max(p.cold_len[b], 0), cap);
  const int hl = p.hot_len[b];
  if (tid == 0) {
    s_count = 0;
    s_hl = hl;
  }
  __syncthreads();
  const int limit = min(p.max_per_step, max(0, p.W_max - 1 - hl));
  uint32_t* mask = p.mask + static_cast<size_t>(b) * (cap / 32);
  uint8_t* counts = p.counts + static_cast<size_t>(b) * cap;
  const float* lse = p.lse + static_cast<size_t>(b) * p.Hq;
  for (int base = 0; base < cl; base += PROMO_THREADS) {
    const int pos = base + tid;
    bool cand = false;
    if (pos < cl && !((mask[pos >> 5] >> (pos & 31)) & 1u)) {
      float w = 0.0f;
      for (int h = 0; h < p.Hq; ++h) {
        const float L = lse[h];
        if (L < __builtin_huge_valf())  // the head read the cold tier
          w = fmaxf(w, exp2f(p.logits[(static_cast<size_t>(b) * p.Hq + h) * cap + pos] - L));
      }
      const int c = w >= p.thr ? min(counts[pos] + 1, 255) : 0;
      counts[pos] = static_cast<uint8_t>(c);
      cand = c >= p.sticky;
    }
    // rank of this position among the block's candidates, in position order
    const uint32_t bal = __ballot_sync(0xffffffffu, cand);
    const int lane = tid & 31, warp = tid >> 5;
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < PROMO_THREADS / 32; ++w) {
      if (w < warp) before += wsum[w];
      total += wsum[w];
    }
    const int rank = s_count + before + __popc(bal & ((1u << lane) - 1u));
    if (cand && rank < limit) {
      chosen[rank] = pos;
      counts[pos] = 0;
      atomicOr(&mask[pos >> 5], 1u << (pos & 31));
    }
    __syncthreads();
    if (tid == 0) s_count = min(limit, s_count + total);
    __syncthreads();
  }
  const int n = s_count;
  int start = p.hot_start[b];
  if (start < 0 || start >= p.W_max) start = 0;
  // decompress each moved position into the ring of every kv head
  for (int i = 0; i < n; ++i) {
    const int pos = chosen[i];
    int slot = start + hl + i;
    while (slot >= p.W_max) slot -= p.W_max;
    for (int kvh = 0; kvh < p.Hkv; ++kvh) {
      const int bh = b * p.Hkv + kvh;
      const int page = p.page_table[static_cast<size_t>(bh) * p.max_pages + pos / TQ_PAGE_TOKENS];
      const bool ok = page >= 0 && page < p.pool_pages;
      if (!ok && tid == 0) report(p.err, TQ_ERR_CAPACITY);
      const int s16 = pos % TQ_PAGE_TOKENS, t = s16 & 15;
      const uint8_t* bk = p.pool + static_cast<size_t>(ok ? page : 0) * p.page_bytes + (s16 >> 4) * p.blk;
      for (int j = tid; j < D; j += PROMO_THREADS) {
        const int byte = plane_byte(j, t);
        const int hb = (bk[p.off_h + byte] >> (t & 7)) & 1, lb = (bk[p.off_l + byte] >> (t & 7)) & 1;
        // level index 2H + L of (-c1, -c0, +c0, +c1)
        const float lev = hb ? (lb ? p.kc1 : p.kc0) : (lb ? -p.kc0 : -p.kc1);
        ck[j] = ok ? lev : 0.0f;
        const int vb = bk[p.off_vc + (vc_pos<D>(j, t >> 1) & (8 * D - 1))];
        const int code = (t & 1) ? (vb >> 4) : (vb & 15);
        cv[j] = ok ? ((code & 8) ? -p.vc[code & 7] : p.vc[code & 7]) : 0.0f;
      }
      __syncthreads();
      const __half2 nn = *reinterpret_cast<const __half2*>(bk + p.off_nk + 4 * t);
      const float nk = ok ? __low2float(nn) : 0.0f;
      const float nv = ok ? __half2float(*reinterpret_cast<const __half*>(bk + p.off_vn + 2 * t)) : 0.0f;
      for (int o = tid; o < 2 * D; o += PROMO_THREADS) {
        const int isv = o >= D, oo = isv ? o - D : o;
        const float* cc = isv ? cv : ck;
        float acc = 0.0f;
        for (int j = 0; j < D; ++j) acc = fmaf(p.rot[j * D + oo], cc[j], acc);  // (Pi^T c)[oo]
        const size_t dst = (static_cast<size_t>(bh) * p.W_max + slot) * D + oo;
        if (isv) p.v_hot[dst] = __float2half_rn(nv * acc);
        else p.k_hot[dst] = __float2half_rn(nk * acc);
      }
      __syncthreads();
    }
  }
  if (tid == 0) p.hot_len[b] = s_hl + n;
}

}  // namespace mon

size_t monarch_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_pages,
                               int W_max, int evict_block) {
  const size_t dec = decode_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max);
  if (dec == 0 || evict_block <= 0) return 0;
  const size_t stage = static_cast<size_t>(B) * Hkv * evict_block * ctx->cfg.head_dim * 2;
  return mon::align256(dec) + 2 * mon::align256(stage) + mon::align256(sizeof(int32_t) * B) +
         mon::align256(sizeof(float) * B * Hq);  // per-head log-sum-exp (promotion)
}

int launch_monarch_step(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq, int Hkv,
                        float scale, const void* k_new, const void* v_new, void* k_hot,
                        void* v_hot, int W_max, int32_t* hot_start, int32_t* hot_len,
                        uint8_t* pool, int64_t pool_pages, const int32_t* page_table,
                        int max_pages, int32_t* cold_len, float threshold, int window,
                        int evict_block, const tq_promotion* promo, int32_t* cold_used,
                        float* out, void* ws, size_t ws_bytes, void* stream) {
  const int d = ctx->cfg.head_dim;
  const int E = evict_block;
  const size_t dec = decode_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max);
  const size_t stage = static_cast<size_t>(B) * Hkv * E * d * 2;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* k_stage = base + mon::align256(dec);
  uint8_t* v_stage = k_stage + mon::align256(stage);
  int32_t* n_evict = reinterpret_cast<int32_t*>(v_stage + mon::align256(stage));
  float* lse = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(n_evict) +
                                        mon::align256(sizeof(int32_t) * B));
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
  DecodePromo dp{};
  if (promo) {
    dp.cold_mask = promo->cold_mask;
    dp.logits = promo->logits;
    dp.lse = lse;
  }
  int rc = launch_decode(ctx, q, q_dtype, B, Hq, Hkv, scale, k_hot, v_hot, W_max, hot_start,
                         hot_len, pool, pool_pages, page_table, max_pages, cold_len, &gate, out,
                         ws, dec, stream, nullptr, promo ? &dp : nullptr);
  if (rc != TQ_OK) return rc;
  if (promo) {
    const PageLayout L = page_layout(d, ctx->cfg.qjl_dim, true);
    mon::PromoParams pp{};
    pp.Hq = Hq;
    pp.Hkv = Hkv;
    pp.W_max = W_max;
    pp.max_pages = max_pages;
    pp.thr = promo->threshold;
    pp.sticky = promo->sticky;
    pp.max_per_step = promo->max_per_step;
    pp.logits = promo->logits;
    pp.lse = lse;
    pp.mask = promo->cold_mask;
    pp.counts = promo->counts;
    pp.pool = pool;
    pp.pool_pages = pool_pages;
    pp.page_bytes = static_cast<long long>(L.bytes);
    pp.blk = static_cast<int>(L.block);
    pp.off_h = static_cast<int>(L.kc);
    pp.off_l = static_cast<int>(L.kl);
    pp.off_vc = static_cast<int>(L.vc);
    pp.off_nk = static_cast<int>(L.kn);
    pp.off_vn = static_cast<int>(L.vn);
    pp.page_table = page_table;
    pp.cold_len = cold_len;
    pp.hot_start = hot_start;
    pp.hot_len = hot_len;
    pp.k_hot = static_cast<__half*>(k_hot);
    pp.v_hot = static_cast<__half*>(v_hot);
    pp.rot = ctx->dev.rot;
    pp.kc0 = ctx->cb.key_c[0];
    pp.kc1 = ctx->cb.key_c[1];
    for (int i = 0; i < 8; ++i) pp.vc[i] = ctx->cb.val_c[i];
    pp.err = ctx->dev.err;
    if (d == 128)
      mon::promote_kernel<128><<<B, mon::PROMO_THREADS, 0, st>>>(pp);
    else
      mon::promote_kernel<64><<<B, mon::PROMO_THREADS, 0, st>>>(pp);
    if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  }
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
