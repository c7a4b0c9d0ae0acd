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
//   weights     (with promotion) one thread per cold position: its largest
//               attention weight over the query heads that read the cold
//               tier, from the attention's logits and the combine's
//               log-sum-exp; consecutive counts; candidate bits
//   promote     (with promotion) one CTA per sequence: the first candidates
//               in position order are masked and their decompressed records
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
  if (!TQ_IN_RANGE(err, slot, W_max)) return;  // (the whole block)
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
  uint32_t* cand;       // [B][cap / 32] workspace: positions whose count reached sticky
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

// Weights and counts, one thread per cold position (grid: position blocks x
// sequences): the position's weight is its largest softmax probability over
// the query heads that read the cold tier (logit and log-sum-exp in base 2;
// a head that kept off the cold tier has log-sum-exp +inf); a weight at or
// above the threshold counts the step, a lower one resets the count.  Bit
// (pos mod 32) of cand word pos / 32: the count reached the sticky value.
__global__ void __launch_bounds__(PROMO_THREADS) weights_kernel(PromoParams p) {
  const int b = blockIdx.y, pos = blockIdx.x * PROMO_THREADS + threadIdx.x;
  const int cap = p.max_pages * TQ_PAGE_TOKENS;
  extern __shared__ float s_lse[];  // [Hq]
  for (int h = threadIdx.x; h < p.Hq; h += PROMO_THREADS)
    s_lse[h] = p.lse[static_cast<size_t>(b) * p.Hq + h];
  __syncthreads();
  const int cl = min(max(p.cold_len[b], 0), cap);
  bool cand = false;
  if (pos < cl) {
    uint32_t* mask = p.mask + static_cast<size_t>(b) * (cap / 32);
    if (!((mask[pos >> 5] >> (pos & 31)) & 1u)) {
      const float* lg = p.logits + static_cast<size_t>(b) * p.Hq * cap + pos;
      float w = 0.0f;
#pragma unroll 8
      for (int h = 0; h < p.Hq; ++h) {
        const float L = s_lse[h];
        const float x = __ldg(lg + static_cast<size_t>(h) * cap);
        if (L < __builtin_huge_valf()) w = fmaxf(w, exp2f(x - L));
      }
      uint8_t* counts = p.counts + static_cast<size_t>(b) * cap;
      const int c = w >= p.thr ? min(counts[pos] + 1, 255) : 0;
      counts[pos] = static_cast<uint8_t>(c);
      cand = c >= p.sticky;
    }
  }
  const uint32_t bal = __ballot_sync(0xffffffffu, cand);
  if ((threadIdx.x & 31) == 0 && pos < cap)
    p.cand[static_cast<size_t>(b) * (cap / 32) + (pos >> 5)] = bal;
}

// Promotion of one sequence (one CTA): the first `limit` candidates in
// position order (limit = min(max_per_step, W_max - 1 - hot_len)) are masked,
// their counts reset, and their decompressed records, n Pi^T c_hat (K) and
// n_v Pi^T c_hat_v (V) rounded to fp16, appended to the ring of every kv head;
// hot_len grows by their number.  Pi is staged in shared memory, and the
// (position, kv head) pairs are decompressed in batches, every thread taking
// outputs of every pair of the batch.
template <int D>
__global__ void __launch_bounds__(PROMO_THREADS) promote_kernel(PromoParams p) {
  constexpr int PB = 8;  // (position, kv head) pairs per batch
  const int b = blockIdx.x, tid = threadIdx.x;
  const int cap = p.max_pages * TQ_PAGE_TOKENS;
  extern __shared__ float s_rot[];  // [D][D]
  __shared__ int chosen[PROMO_MAX];
  __shared__ int wsum[PROMO_THREADS / 32];
  __shared__ float lev[PB][2][D];   // key and value levels of the batch's pairs
  __shared__ float nrm[PB][2];
  __shared__ int s_count;
  const int cl = min(max(p.cold_len[b], 0), cap);
  const int hl = p.hot_len[b];
  const int limit = min(p.max_per_step, max(0, p.W_max - 1 - hl));
  if (tid == 0) s_count = 0;
  __syncthreads();
  // the first `limit` candidates, in position order (one word per thread)
  const uint32_t* cw = p.cand + static_cast<size_t>(b) * (cap / 32);
  const int nwords = (cl + 31) / 32;
  for (int w0 = 0; w0 < nwords && s_count < limit; w0 += PROMO_THREADS) {
    const int w = w0 + tid;
    uint32_t bits = 0u;
    if (w < nwords) {
      bits = cw[w];
      if (32 * w + 32 > cl) bits &= (cl - 32 * w >= 32) ? ~0u : ((1u << (cl - 32 * w)) - 1u);
    }
    const int n = __popc(bits);
    // exclusive prefix of n over the block's threads
    int incl = n;
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = s_count;
    for (int q = 0; q < warp; ++q) before += wsum[q];
    before += incl - n;
    while (bits && before < limit) {
      const int j = __ffs(static_cast<int>(bits)) - 1;
      bits &= bits - 1u;
      chosen[before++] = 32 * w + j;
    }
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int q = 0; q < PROMO_THREADS / 32; ++q) tot += wsum[q];
      s_count = min(limit, s_count + tot);
    }
    __syncthreads();
  }
  const int n = s_count;
  if (n == 0) return;
  uint32_t* mask = p.mask + static_cast<size_t>(b) * (cap / 32);
  uint8_t* counts = p.counts + static_cast<size_t>(b) * cap;
  for (int i = tid; i < n; i += PROMO_THREADS) {
    const int pos = chosen[i];
    counts[pos] = 0;
    atomicOr(&mask[pos >> 5], 1u << (pos & 31));
  }
  for (int i = tid; i < D * D; i += PROMO_THREADS) s_rot[i] = p.rot[i];
  int start = p.hot_start[b];
  if (start < 0 || start >= p.W_max) start = 0;
  const int npair = n * p.Hkv;
  for (int pb0 = 0; pb0 < npair; pb0 += PB) {
    const int nb = min(PB, npair - pb0);
    __syncthreads();  // s_rot staged; the previous batch's levels consumed
    // levels of the batch's pairs: pair = i * Hkv + kvh
    for (int e = tid; e < nb * D; e += PROMO_THREADS) {
      const int q = e / D, j = e % D;
      const int pr = pb0 + q, i = pr / p.Hkv, kvh = pr % p.Hkv;
      const int pos = TQ_IN_RANGE(p.err, chosen[i], cap) ? chosen[i] : 0;
      const int bh = b * p.Hkv + kvh;
      const int page = p.page_table[static_cast<size_t>(bh) * p.max_pages + pos / TQ_PAGE_TOKENS];
      const bool ok = page >= 0 && page < p.pool_pages;
      if (!ok && j == 0) report(p.err, TQ_ERR_CAPACITY);
      const int s16 = pos % TQ_PAGE_TOKENS, t = s16 & 15;
      const uint8_t* bk = p.pool + static_cast<size_t>(ok ? page : 0) * p.page_bytes + (s16 >> 4) * p.blk;
      const int byte = plane_byte(j, t);
      const int hb = (bk[p.off_h + byte] >> (t & 7)) & 1, lb = (bk[p.off_l + byte] >> (t & 7)) & 1;
      // level index 2H + L of (-c1, -c0, +c0, +c1)
      lev[q][0][j] = ok ? (hb ? (lb ? p.kc1 : p.kc0) : (lb ? -p.kc0 : -p.kc1)) : 0.0f;
      const int vb = bk[p.off_vc + (vc_pos<D>(j, t >> 1) & (8 * D - 1))];
      const int code = (t & 1) ? (vb >> 4) : (vb & 15);
      lev[q][1][j] = ok ? ((code & 8) ? -p.vc[code & 7] : p.vc[code & 7]) : 0.0f;
      if (j == 0) {
        nrm[q][0] = ok ? __low2float(*reinterpret_cast<const __half2*>(bk + p.off_nk + 4 * t)) : 0.0f;
        nrm[q][1] = ok ? __half2float(*reinterpret_cast<const __half*>(bk + p.off_vn + 2 * t)) : 0.0f;
      }
    }
    __syncthreads();
    // outputs (Pi^T c)[o] = sum_j Pi[j][o] c[j]: thread = output coordinate
    // and K / V, over every pair of the batch
    for (int e = tid; e < 2 * D; e += PROMO_THREADS) {
      const int isv = e >= D, o = isv ? e - D : e;
      float acc[PB];
#pragma unroll
      for (int q = 0; q < PB; ++q) acc[q] = 0.0f;
      for (int j = 0; j < D; ++j) {
        const float r = s_rot[j * D + o];
#pragma unroll
        for (int q = 0; q < PB; ++q) acc[q] = fmaf(r, lev[q][isv][j], acc[q]);
      }
      for (int q = 0; q < nb; ++q) {
        const int pr = pb0 + q, i = pr / p.Hkv, kvh = pr % p.Hkv;
        int slot = start + hl + i;
        while (slot >= p.W_max) slot -= p.W_max;
        const size_t dst = ((static_cast<size_t>(b) * p.Hkv + kvh) * p.W_max + slot) * D + o;
        const __half hv = __float2half_rn(nrm[q][isv] * acc[q]);
        if (!TQ_IN_RANGE(p.err, i, PROMO_MAX)) continue;
        if (isv) p.v_hot[dst] = hv;
        else p.k_hot[dst] = hv;
      }
    }
  }
  if (tid == 0) p.hot_len[b] = hl + n;
}

}  // namespace mon

size_t monarch_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_pages,
                               int W_max, int evict_block) {
  const size_t dec = decode_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max);
  if (dec == 0 || evict_block <= 0) return 0;
  const size_t stage = static_cast<size_t>(B) * Hkv * evict_block * ctx->cfg.head_dim * 2;
  return mon::align256(dec) + 2 * mon::align256(stage) + mon::align256(sizeof(int32_t) * B) +
         mon::align256(sizeof(float) * B * Hq) +  // per-head log-sum-exp (promotion)
         mon::align256(sizeof(uint32_t) * B * max_pages * (TQ_PAGE_TOKENS / 32));  // candidates
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
  uint32_t* cand = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(lse) +
                                               mon::align256(sizeof(float) * B * Hq));
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
    pp.cand = cand;
    const int cap = max_pages * TQ_PAGE_TOKENS;
    mon::weights_kernel<<<dim3((cap + mon::PROMO_THREADS - 1) / mon::PROMO_THREADS, B),
                          mon::PROMO_THREADS, sizeof(float) * Hq, st>>>(pp);
    if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
    const int rot_bytes = static_cast<int>(sizeof(float)) * d * d;
    static SmemAttr promo_attr;
    if (d == 128) {
      if (!raise_smem_limit(mon::promote_kernel<128>, rot_bytes, promo_attr)) return TQ_ERR_CUDA;
      mon::promote_kernel<128><<<B, mon::PROMO_THREADS, rot_bytes, st>>>(pp);
    } else {
      mon::promote_kernel<64><<<B, mon::PROMO_THREADS, rot_bytes, st>>>(pp);
    }
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
