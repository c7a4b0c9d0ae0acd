// One decode step of Tensor Cache's two-level state ("Tensor Cache:
// Eviction-conditioned Associative Memory for Transformers", gist.science,
// section "Methodik: Tensor Cache (TC)"): an fp16 ring of the last W tokens
// read with exact softmax attention (L1), and a d x d outer-product matrix A
// per kv head written only by the ring's evictions (L2),
//   A <- lambda A + eta (k (x) v),   r = q A,   y = y_local + sigmoid(g) r.
//
// Launches, all on the caller's stream:
//   update   D / 32 CTAs per (sequence, kv head), each 32 columns of A:
//            when the ring is full the token the step's token will overwrite
//            is written into A; then r = q A (the updated A) for the group's
//            query heads.  One pass over A: read, update, write, and the
//            products of the read.  The new ring start and length go to the
//            workspace (the caller's arrays are read by every CTA).
//   decode   the split-K attention over the ring alone (prep, attention,
//            combine), with the ring start and length of this step: prep
//            writes the step's token into its slot (after every update CTA
//            has read the token it replaces), the combine's epilogue adds
//            sigmoid(g) r and writes the new ring start and length back
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace tcache {

// Columns of A per update CTA: a (sequence, kv head) takes D / UPD_COLS CTAs,
// each the whole read r_j = sum_i q_i A[i][j] of its columns (no reduction
// across CTAs).
constexpr int UPD_COLS = 32;

template <int D, int G>
__global__ void __launch_bounds__(256) update_kernel(const void* q, int q_dtype, int Hq, int Hkv,
                                                     const __half* k_ring, const __half* v_ring,
                                                     int W, const int32_t* ring_start,
                                                     const int32_t* ring_len, float* A,
                                                     const float* lambda, const float* eta,
                                                     float* r_out, int32_t* new_start,
                                                     int32_t* new_len, int* err) {
  constexpr int NSPLIT = D / UPD_COLS;
  constexpr int NR = 256 / UPD_COLS;  // row phases
  constexpr int RPT = D / NR;         // rows per thread
  const int bh = blockIdx.x / NSPLIT, cs = blockIdx.x % NSPLIT;
  const int b = bh / Hkv, kvh = bh % Hkv;
  const int tid = threadIdx.x, jl = tid % UPD_COLS, rp = tid / UPD_COLS;
  const int j = cs * UPD_COLS + jl;
  __shared__ float sk[D];
  __shared__ float sq[G][D];
  __shared__ float part[NR][G][UPD_COLS];
  const int len = ring_len[b], start = ring_start[b];
  const bool ok = len >= 0 && len <= W && start >= 0 && start < W;
  const bool lead = cs == 0 && kvh == 0 && tid == 0;  // one writer of the sequence's ring state
  if (!ok) {
    if (tid == 0) report(err, TQ_ERR_CAPACITY);
    if (lead) {
      new_start[b] = 0;
      new_len[b] = 0;
    }
    if (tid < G * UPD_COLS)
      r_out[(static_cast<size_t>(b) * Hq + kvh * G + tid / UPD_COLS) * D + cs * UPD_COLS +
            tid % UPD_COLS] = 0.0f;
    return;
  }
  // a full ring evicts its oldest token, whose slot the step's token takes
  // (written by the decode's prep launch, after this one)
  const bool evict = len == W;
  const size_t row = (static_cast<size_t>(bh) * W + (TQ_IN_RANGE(err, start, W) ? start : 0)) * D;
  if (tid < D) sk[tid] = evict ? __half2float(k_ring[row + tid]) : 0.0f;
  for (int i = tid; i < G * D; i += blockDim.x)
    sq[i / D][i % D] = load_as_float(q, (static_cast<size_t>(b) * Hq + kvh * G) * D + i,
                                     static_cast<tq_dtype>(q_dtype));
  if (lead) {
    new_start[b] = evict ? (start + 1 == W ? 0 : start + 1) : start;
    new_len[b] = evict ? W : len + 1;
  }
  const float lam = lambda[kvh], et = eta[kvh];
  const float evj = evict ? et * __half2float(v_ring[row + j]) : 0.0f;
  // A[i][j], i = key coordinate: this thread takes column j, rows rp, rp + NR,
  // ...; all of its values are loaded before any arithmetic
  float* Ab = A + static_cast<size_t>(bh) * D * D;
  float av[RPT];
#pragma unroll
  for (int m = 0; m < RPT; ++m) av[m] = Ab[static_cast<size_t>(rp + NR * m) * D + j];
  // (the barrier also keeps the compiler from sinking the loads past the stores below)
  __syncthreads();
  float acc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g] = 0.0f;
#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    const int i = rp + NR * m;
    float a = av[m];
    if (evict) {
      a = fmaf(lam, a, evj * sk[i]);
      Ab[static_cast<size_t>(i) * D + j] = a;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g] = fmaf(sq[g][i], a, acc[g]);
  }
#pragma unroll
  for (int g = 0; g < G; ++g) part[rp][g][jl] = acc[g];
  __syncthreads();
  for (int i = tid; i < G * UPD_COLS; i += blockDim.x) {
    const int g = i / UPD_COLS, jj = i % UPD_COLS;
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < NR; ++k) s += part[k][g][jj];
    r_out[(static_cast<size_t>(b) * Hq + kvh * G + g) * D + cs * UPD_COLS + jj] = s;
  }
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace tcache

size_t tensor_cache_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int W) {
  const size_t dec = decode_workspace_bytes(ctx, B, Hq, Hkv, 0, W);
  if (dec == 0) return 0;
  return tcache::align256(dec) +
         tcache::align256(sizeof(float) * static_cast<size_t>(B) * Hq * ctx->cfg.head_dim) +
         2 * tcache::align256(sizeof(int32_t) * B);
}

int launch_tensor_cache_step(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                             int Hkv, float scale, const void* k_new, const void* v_new,
                             void* k_ring, void* v_ring, int W, int32_t* ring_start,
                             int32_t* ring_len, float* A, const float* lambda, const float* eta,
                             const float* gate, float* out, void* ws, size_t ws_bytes,
                             void* stream) {
  (void)ws_bytes;
  const int d = ctx->cfg.head_dim;
  const int G = Hq / Hkv;
  const size_t dec = decode_workspace_bytes(ctx, B, Hq, Hkv, 0, W);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* r = reinterpret_cast<float*>(base + tcache::align256(dec));
  int32_t* ns = reinterpret_cast<int32_t*>(
      reinterpret_cast<uint8_t*>(r) + tcache::align256(sizeof(float) * static_cast<size_t>(B) * Hq * d));
  int32_t* nl = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(ns) +
                                           tcache::align256(sizeof(int32_t) * B));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const __half* kr = static_cast<const __half*>(k_ring);
  const __half* vr = static_cast<const __half*>(v_ring);
  const int qd = static_cast<int>(q_dtype);
#define TQ_TC_LAUNCH(DD, GG)                                                                      \
  tcache::update_kernel<DD, GG><<<B * Hkv * (DD / tcache::UPD_COLS), 256, 0, st>>>(               \
      q, qd, Hq, Hkv, kr, vr, W, ring_start, ring_len, A, lambda, eta, r, ns, nl, ctx->dev.err)
  if (d == 128) {
    switch (G) {
      case 1: TQ_TC_LAUNCH(128, 1); break;
      case 2: TQ_TC_LAUNCH(128, 2); break;
      case 4: TQ_TC_LAUNCH(128, 4); break;
      case 8: TQ_TC_LAUNCH(128, 8); break;
      default: return TQ_ERR_UNSUPPORTED;
    }
  } else if (d == 64) {
    switch (G) {
      case 1: TQ_TC_LAUNCH(64, 1); break;
      case 2: TQ_TC_LAUNCH(64, 2); break;
      case 4: TQ_TC_LAUNCH(64, 4); break;
      case 8: TQ_TC_LAUNCH(64, 8); break;
      default: return TQ_ERR_UNSUPPORTED;
    }
  } else {
    return TQ_ERR_UNSUPPORTED;
  }
#undef TQ_TC_LAUNCH
  if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  // prep writes the step's token into the ring; the combine adds sigmoid(g) r
  // and writes the ring start and length back
  const DecodeFuse fz{r, gate, ns, nl, ring_start, ring_len, k_new, v_new, k_ring, v_ring};
  return launch_decode(ctx, q, q_dtype, B, Hq, Hkv, scale, k_ring, v_ring, W, ns, nl, nullptr, 0,
                       nullptr, 0, nullptr, nullptr, out, ws, dec, stream, &fz);
}

}  // namespace tq
