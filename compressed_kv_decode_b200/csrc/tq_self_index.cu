// Self-Indexing KV cache, index build and compressed-domain scores ("Self-
// Indexing KVCache", page 2, section "Methodologie: Self-Indexing KVCache",
// items 1-3): keys are centred by their channel mean, cut into 4-dimensional
// subvectors whose sign pattern is a 4-bit index, and a codebook of 16
// centroids per group is built in one pass; a query scores every token by a
// table of its dot products with the centroids (lookup and add).
//
//  build   one CTA per (batch, kv head): channel mean (fp32), then every
//          (token, group) index (one byte each, pattern in the low nibble)
//          with the centred subvector summed into its centroid in shared
//          memory; centroids = sums / counts (zero for an unused index).
//  scores  one CTA per (batch, query head): the d/4 x 16 table in shared
//          memory, then one token per thread: 4 x 16-byte loads of its d/4
//          indices and d/4 table lookups.
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

}  // namespace tq
