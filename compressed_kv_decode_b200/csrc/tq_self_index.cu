// Self-Indexing KV cache ("Self-Indexing KVCache", section "Methodologie:
// Self-Indexing KVCache", items 1-4): keys are centred by their channel
// mean, cut into 4-dimensional subvectors whose sign pattern is a 4-bit
// index, and a codebook of 16 centroids per group is built in one pass; a
// query scores every token by a table of its dot products with the centroids
// (lookup and add), keeps the best tokens after the 64 full-precision sinks,
// and attends over the sinks and those tokens only.
//
//  build   one CTA per (batch, kv head): channel mean (fp32), then every
//          (token, group) index (one byte each, pattern in the low nibble)
//          with the centred subvector summed into its centroid in shared
//          memory; centroids = sums / counts (zero for an unused index).
//  scores  one CTA per (batch, query head): the d/4 x 16 table in shared
//          memory, then one token per thread: 4 x 16-byte loads of its d/4
//          indices and d/4 table lookups.
//  select  one CTA per (batch, query head): radix select of the top k
//          scores, ties to the lower position, output in position order.
//  attend  one CTA per (batch, query head): exact softmax attention over the
//          sinks and the selected tokens' stored fp16 keys and values.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace six {

template <int D>
__global__ void __launch_bounds__(256) build_kernel(const __half* __restrict__ k, int T,
                                                    float* __restrict__ mu,
                                                    uint8_t* __restrict__ codes,
                                                    float* __restrict__ cent) {
  constexpr int NG = D / 4;      // groups
  constexpr int PH = 256 / D;    // token phases of the mean
  constexpr int GP = 256 / NG;   // token phases of the index pass
  const int bh = blockIdx.x, tid = threadIdx.x;
  const __half* kb = k + static_cast<size_t>(bh) * T * D;
  __shared__ float part[PH][D];
  __shared__ float smu[D];
  __shared__ float csum[NG][16][4];
  __shared__ int ccnt[NG][16];
  // channel mean
  {
    const int j = tid % D, ph = tid / D;
    float s = 0.0f;
    for (int t = ph; t < T; t += PH) s += __half2float(kb[static_cast<size_t>(t) * D + j]);
    part[ph][j] = s;
  }
  for (int i = tid; i < NG * 16 * 4; i += blockDim.x) (&csum[0][0][0])[i] = 0.0f;
  for (int i = tid; i < NG * 16; i += blockDim.x) (&ccnt[0][0])[i] = 0;
  __syncthreads();
  if (tid < D) {
    float s = 0.0f;
#pragma unroll
    for (int p = 0; p < PH; ++p) s += part[p][tid];
    const float m = T > 0 ? s / static_cast<float>(T) : 0.0f;
    smu[tid] = m;
    mu[static_cast<size_t>(bh) * D + tid] = m;
  }
  __syncthreads();
  // indices and centroid sums: thread = (group g, token phase)
  {
    const int g = tid % NG, ph = tid / NG;
    const float m0 = smu[4 * g], m1 = smu[4 * g + 1], m2 = smu[4 * g + 2], m3 = smu[4 * g + 3];
    for (int t = ph; t < T; t += GP) {
      const uint2 raw = *reinterpret_cast<const uint2*>(kb + static_cast<size_t>(t) * D + 4 * g);
      const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
      const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
      const float c0 = a.x - m0, c1 = a.y - m1, c2 = b.x - m2, c3 = b.y - m3;
      const int p = (c0 > 0.0f ? 1 : 0) | (c1 > 0.0f ? 2 : 0) | (c2 > 0.0f ? 4 : 0) |
                    (c3 > 0.0f ? 8 : 0);
      codes[(static_cast<size_t>(bh) * T + t) * NG + g] = static_cast<uint8_t>(p);
      atomicAdd(&csum[g][p][0], c0);
      atomicAdd(&csum[g][p][1], c1);
      atomicAdd(&csum[g][p][2], c2);
      atomicAdd(&csum[g][p][3], c3);
      atomicAdd(&ccnt[g][p], 1);
    }
  }
  __syncthreads();
  for (int i = tid; i < NG * 16 * 4; i += blockDim.x) {
    const int gp = i / 4;
    const int n = (&ccnt[0][0])[gp];
    cent[static_cast<size_t>(bh) * NG * 64 + i] = n > 0 ? (&csum[0][0][0])[i] / static_cast<float>(n) : 0.0f;
  }
}

template <int D>
__global__ void __launch_bounds__(256) scores_kernel(const void* q, int q_dtype, int Hq, int Hkv,
                                                     int T, const uint8_t* __restrict__ codes,
                                                     const float* __restrict__ cent,
                                                     float* __restrict__ scores) {
  constexpr int NG = D / 4;
  const int bq = blockIdx.x, b = bq / Hq, hq = bq % Hq, kvh = hq / (Hq / Hkv);
  const int bh = b * Hkv + kvh;
  __shared__ float sq[D];
  __shared__ float lut[NG][16];
  for (int i = threadIdx.x; i < D; i += blockDim.x)
    sq[i] = load_as_float(q, static_cast<size_t>(bq) * D + i, static_cast<tq_dtype>(q_dtype));
  __syncthreads();
  const float* cb = cent + static_cast<size_t>(bh) * NG * 64;
  for (int i = threadIdx.x; i < NG * 16; i += blockDim.x) {
    const int g = i / 16;
    const float* c = cb + 4 * i;
    lut[g][i % 16] = fmaf(sq[4 * g], c[0], fmaf(sq[4 * g + 1], c[1],
                          fmaf(sq[4 * g + 2], c[2], sq[4 * g + 3] * c[3])));
  }
  __syncthreads();
  const uint8_t* cbase = codes + static_cast<size_t>(bh) * T * NG;
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    const uint4* row = reinterpret_cast<const uint4*>(cbase + static_cast<size_t>(t) * NG);
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < NG / 16; ++w) {
      const uint4 v = row[w];
      const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int g = 16 * w + e;
        s += lut[g][(words[e >> 2] >> (8 * (e & 3))) & 0xFu];
      }
    }
    scores[static_cast<size_t>(bq) * T + t] = s;
  }
}

// Ordered key of a score: a larger float gives a larger unsigned key; -0.0
// and +0.0 share one key (they compare equal); every NaN gets key 0, below
// -inf, so NaN scores are picked last (ties among them to the lower position).
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;
  const uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Rank of this thread's flag among the block's set flags in thread order, and
// the block's count.  Every thread of the block calls it.
template <int NT>
__device__ __forceinline__ int block_rank(bool f, int& total, int* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t bal = __ballot_sync(0xffffffffu, f);
  const int r = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) wsum[warp] = __popc(bal);
  __syncthreads();
  int off = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const int c = wsum[w];
    off += w < warp ? c : 0;
    tot += c;
  }
  __syncthreads();
  total = tot;
  return off + r;
}

// Top-k of one row of scores over the positions [lo, T): a radix select on
// the ordered 32-bit keys (four 8-bit digits, most significant first) finds
// the k-th largest key K* and how many tokens with key K* are taken; one pass
// in position order then writes every token above K* and the first of those
// equal to K*, so ties go to the lower position and the output is sorted.
template <int NT>
__global__ void __launch_bounds__(NT) select_kernel(const float* __restrict__ scores, int T,
                                                    int lo, int k_eff, int k_cap,
                                                    int32_t* __restrict__ picked) {
  const int tid = threadIdx.x;
  const float* s = scores + static_cast<size_t>(blockIdx.x) * T;
  int32_t* out = picked + static_cast<size_t>(blockIdx.x) * k_cap;
  __shared__ int hist[256];
  __shared__ int wsum[NT / 32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;
  for (int i = k_eff + tid; i < k_cap; i += NT) out[i] = -1;
  if (k_eff <= 0) return;
  uint32_t prefix = 0;
  int need = k_eff;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t hi = pass == 0 ? 0u : (0xffffffffu << (shift + 8));
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
    for (int t = lo + tid; t < T; t += NT) {
      const uint32_t key = order_key(s[t]);
      if ((key & hi) == (prefix & hi)) atomicAdd(&hist[(key >> shift) & 0xffu], 1);
    }
    __syncthreads();
    if (tid == 0) {
      int cum = 0, bin = 255;
      for (; bin > 0; --bin) {
        if (cum + hist[bin] >= need) break;
        cum += hist[bin];
      }
      s_prefix = prefix | (static_cast<uint32_t>(bin) << shift);
      s_need = need - cum;
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
  }
  // in position order: every key above K*, then the first `need` equal to it
  int taken = 0, ties = 0;
  for (int c0 = lo; c0 < T && taken < k_eff; c0 += NT) {
    const int t = c0 + tid;
    const uint32_t key = t < T ? order_key(s[t]) : 0u;
    const bool eq = t < T && key == prefix;
    int n_eq;
    const int tie_rank = ties + block_rank<NT>(eq, n_eq, wsum);
    const bool sel = (t < T && key > prefix) || (eq && tie_rank < need);
    int n_sel;
    const int slot = taken + block_rank<NT>(sel, n_sel, wsum);
    if (sel && slot < k_eff) out[slot] = t;
    ties += n_eq;
    taken += n_sel;
  }
}

// Exact softmax attention of one query head over the sinks [0, n_s) and its
// selected positions, with the stored fp16 keys and values.  A warp takes
// every eighth token: a lane holds D/32 coordinates, the dot product is a
// shuffle reduction, and the warp keeps a running maximum, sum and weighted
// value; the eight warps are merged at the end.
template <int D>
__global__ void __launch_bounds__(256) attend_kernel(const void* q, int q_dtype, int Hq, int Hkv,
                                                     int T, const __half* __restrict__ keys,
                                                     const __half* __restrict__ values,
                                                     const int32_t* __restrict__ picked,
                                                     int k_cap, int k_eff, int n_s, float scale,
                                                     float* __restrict__ out, int* err) {
  constexpr int PL = D / 32;
  const int row = blockIdx.x, b = row / Hq, hq = row % Hq, kvh = hq / (Hq / Hkv);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t base = static_cast<size_t>(b * Hkv + kvh) * T * D;
  __shared__ float sm[8], sl[8];
  __shared__ float sacc[8][D];
  float qv[PL], acc[PL];
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    qv[i] = load_as_float(q, static_cast<size_t>(row) * D + lane * PL + i,
                          static_cast<tq_dtype>(q_dtype)) * scale;
    acc[i] = 0.0f;
  }
  float m = -INFINITY, l = 0.0f;
  const int n = n_s + k_eff;
  for (int j = warp; j < n; j += 8) {
    const int pos = j < n_s ? j : picked[static_cast<size_t>(row) * k_cap + (j - n_s)];
    if (pos < 0 || pos >= T) {
      if (lane == 0) report(err, TQ_ERR_INVALID_ARG);
      continue;
    }
    const size_t off = base + static_cast<size_t>(pos) * D + lane * PL;
    float kf[PL], vf[PL];
    if constexpr (PL == 4) {
      const uint2 kr = *reinterpret_cast<const uint2*>(keys + off);
      const uint2 vr = *reinterpret_cast<const uint2*>(values + off);
      const float2 k0 = __half22float2(*reinterpret_cast<const __half2*>(&kr.x));
      const float2 k1 = __half22float2(*reinterpret_cast<const __half2*>(&kr.y));
      const float2 v0 = __half22float2(*reinterpret_cast<const __half2*>(&vr.x));
      const float2 v1 = __half22float2(*reinterpret_cast<const __half2*>(&vr.y));
      kf[0] = k0.x; kf[1] = k0.y; kf[2] = k1.x; kf[3] = k1.y;
      vf[0] = v0.x; vf[1] = v0.y; vf[2] = v1.x; vf[3] = v1.y;
    } else {
      const float2 k0 = __half22float2(*reinterpret_cast<const __half2*>(keys + off));
      const float2 v0 = __half22float2(*reinterpret_cast<const __half2*>(values + off));
      kf[0] = k0.x; kf[1] = k0.y;
      vf[0] = v0.x; vf[1] = v0.y;
    }
    float dot = 0.0f;
#pragma unroll
    for (int i = 0; i < PL; ++i) dot = fmaf(kf[i], qv[i], dot);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    const float mn = fmaxf(m, dot);
    const float corr = expf(m - mn), p = expf(dot - mn);
    l = fmaf(l, corr, p);
#pragma unroll
    for (int i = 0; i < PL; ++i) acc[i] = fmaf(acc[i], corr, p * vf[i]);
    m = mn;
  }
#pragma unroll
  for (int i = 0; i < PL; ++i) sacc[warp][lane * PL + i] = acc[i];
  if (lane == 0) {
    sm[warp] = m;
    sl[warp] = l;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) M = fmaxf(M, sm[w]);
    float L = 0.0f, o = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float f = expf(sm[w] - M);
        L = fmaf(sl[w], f, L);
        o = fmaf(sacc[w][c], f, o);
      }
    }
    out[static_cast<size_t>(row) * D + c] = L > 0.0f ? o / L : 0.0f;
  }
}

}  // namespace six

int launch_self_index_build(const tq_ctx* ctx, const void* k, int B, int Hkv, int T, float* mu,
                            uint8_t* codes, float* cent, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const __half* kh = static_cast<const __half*>(k);
  if (ctx->cfg.head_dim == 128)
    six::build_kernel<128><<<B * Hkv, 256, 0, st>>>(kh, T, mu, codes, cent);
  else
    six::build_kernel<64><<<B * Hkv, 256, 0, st>>>(kh, T, mu, codes, cent);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

int launch_self_index_scores(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                             int Hkv, int T, const uint8_t* codes, const float* cent,
                             float* scores, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int qd = static_cast<int>(q_dtype);
  if (ctx->cfg.head_dim == 128)
    six::scores_kernel<128><<<B * Hq, 256, 0, st>>>(q, qd, Hq, Hkv, T, codes, cent, scores);
  else
    six::scores_kernel<64><<<B * Hq, 256, 0, st>>>(q, qd, Hq, Hkv, T, codes, cent, scores);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

int launch_self_index_select(const float* scores, int rows, int T, int lo, int k_eff, int k_cap,
                             int32_t* picked, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  six::select_kernel<512><<<rows, 512, 0, st>>>(scores, T, lo, k_eff, k_cap, picked);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

int launch_self_index_attend(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                             int Hkv, int T, const void* keys, const void* values,
                             const int32_t* picked, int k_cap, int k_eff, int n_s, float scale,
                             float* out, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int qd = static_cast<int>(q_dtype);
  const __half* kh = static_cast<const __half*>(keys);
  const __half* vh = static_cast<const __half*>(values);
  if (ctx->cfg.head_dim == 128)
    six::attend_kernel<128><<<B * Hq, 256, 0, st>>>(q, qd, Hq, Hkv, T, kh, vh, picked, k_cap,
                                                    k_eff, n_s, scale, out, ctx->dev.err);
  else
    six::attend_kernel<64><<<B * Hq, 256, 0, st>>>(q, qd, Hq, Hkv, T, kh, vh, picked, k_cap,
                                                   k_eff, n_s, scale, out, ctx->dev.err);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace tq
