// Self-Indexing KV cache ("Self-Indexing KVCache", section "Methodologie:
// Self-Indexing KVCache", items 1-4): keys are centred by their channel
// mean, cut into 4-dimensional subvectors whose sign pattern is a 4-bit
// index, and a codebook of 16 centroids per group is built in one pass; a
// query scores every token by a table of its dot products with the centroids
// (lookup and add), keeps the best tokens after the 64 full-precision sinks,
// and attends over the sinks and those tokens only.
//
//  build   one cluster of 16 (or 8) CTAs per (batch, kv head), each CTA a
//          slice of the tokens: channel mean (fp32, the CTAs' partial sums
//          added in rank order through distributed shared memory), then
//          every (token, group) index (one byte each, pattern in the low
//          nibble) with the centred subvector summed into per-CTA centroid
//          sums, reduced across the cluster; centroids = sums / counts (zero
//          for an unused index).
//  scores  one CTA per (batch, query head): the d/4 x 16 table in shared
//          memory, then one token per thread: 4 x 16-byte loads of its d/4
//          indices and d/4 table lookups.
//  select  one CTA per SM, persistent over the (batch, query head) rows:
//          the row's ordered keys staged in shared memory, radix select of
//          the top k over three digits, ties to the lower position, output
//          in position order.
//  attend  one CTA per (batch, query head): exact softmax attention over the
//          sinks and the selected tokens' stored fp16 keys and values, a
//          token per D/8 lanes, several tokens in flight per warp.
#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace six {

constexpr int BUILD_THREADS = 512;
// Dynamic shared memory of the build kernel: the private centroid tables
// (one per lane group of NG lanes: 16 float4 sums + 16 counts per group),
// 160 KB at either head dimension.  One CTA per SM: the clusters then cover
// few kv heads at a time, and a head's keys stay in L2 between the mean pass
// and the index pass.
constexpr int BUILD_SMEM = 160 * 1024;

// Index build for one (batch, kv head) per cluster of CS CTAs, CTA r taking
// the tokens [T r / CS, T (r + 1) / CS):
//   1. per-channel partial sums of its tokens (16-byte loads, 8 channels per
//      thread, sixteen rows in flight, then a fixed-order reduction over the
//      token phases);
//   2. cluster barrier; every CTA adds the CS partials in rank order from
//      distributed shared memory, so all CTAs hold the same fp32 mean;
//   3. its tokens' (token, group) sign patterns, written as bytes; lane g of
//      a lane group takes group g and adds the subvector to its own table
//      entry (no atomics: every entry has one writer); the mean is taken off
//      the sums once per entry at the end;
//   4. the CTA's tables added entry by entry in a fixed order; cluster
//      barrier; CTA r reduces a slice of the (group, pattern) entries over
//      the CS CTAs in rank order and writes the centroids.
// Every sum is taken in a fixed order: the results do not vary from run to
// run.
template <int D>
__global__ void __launch_bounds__(BUILD_THREADS, 1) build_kernel(const __half* __restrict__ k, int T,
                                                                 float* __restrict__ mu,
                                                                 uint8_t* __restrict__ codes,
                                                                 float* __restrict__ cent) {
  namespace cg = cooperative_groups;
  constexpr int NG = D / 4;                         // groups
  constexpr int C8 = D / 8;                         // 16-byte chunks of a key row
  constexpr int PH = BUILD_THREADS / C8;            // token phases of the mean pass
  constexpr int TPW = 32 / NG;                      // tokens per warp in the index pass
  constexpr int NWARP = BUILD_THREADS / 32;
  constexpr int NCOPY = NWARP * TPW;                // private tables
  constexpr int TSTEP = NCOPY;                      // tokens per CTA per index round
  constexpr int U = 16;                             // rows in flight per thread
  constexpr int NE = 16 * NG;                       // (pattern, group) entries
  static_assert(NCOPY * NE * 20 <= BUILD_SMEM, "tables");
  static_assert(PH * D * 4 <= BUILD_SMEM, "mean partials");
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = static_cast<int>(cluster.num_blocks());
  const int r = static_cast<int>(cluster.block_rank());
  const int bh = blockIdx.x / CS, tid = threadIdx.x;
  const int t0 = static_cast<int>(static_cast<long long>(T) * r / CS);
  const int t1 = static_cast<int>(static_cast<long long>(T) * (r + 1) / CS);
  const __half* kb = k + static_cast<size_t>(bh) * T * D;
  extern __shared__ __align__(16) float dyn[];
  float* red = dyn;                                             // [PH][D] (mean pass)
  float4* csum = reinterpret_cast<float4*>(dyn);                // [NCOPY][16][NG]
  float* ccnt = dyn + 4 * NCOPY * NE;                           // [NCOPY][16][NG]
  __shared__ float part[D];  // this CTA's channel sums
  __shared__ float smu[D];
  // 1. channel sums of this CTA's tokens
  {
    const int c = tid % C8, ph = tid / C8;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
    for (int t = t0 + ph; t < t1; t += U * PH) {
      uint4 raw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tt = t + u * PH;
        raw[u] = tt < t1 ? *reinterpret_cast<const uint4*>(kb + static_cast<size_t>(tt) * D + 8 * c)
                         : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
          acc[2 * e] += f.x;
          acc[2 * e + 1] += f.y;
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[ph * D + 8 * c + e] = acc[e];
  }
  __syncthreads();
  if (tid < D) {
    float s = 0.0f;
    for (int q = 0; q < PH; ++q) s += red[q * D + tid];
    part[tid] = s;
  }
  __syncthreads();  // red is read: the tables may overwrite it
  for (int i = tid; i < NCOPY * NE; i += BUILD_THREADS) {
    csum[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    ccnt[i] = 0.0f;
  }
  // 2. the mean from every CTA's sums, in rank order
  cluster.sync();
  if (tid < D) {
    float s = 0.0f;
    for (int q = 0; q < CS; ++q) s += *cluster.map_shared_rank(&part[tid], q);
    const float m = s / static_cast<float>(T);
    smu[tid] = m;
    if (r == 0) mu[static_cast<size_t>(bh) * D + tid] = m;
  }
  __syncthreads();
  // 3. sign patterns and the lane's table: lane = (token of the warp, group g).
  // The pattern compares the raw key with the mean (the sign of the fp32
  // difference is that of the exact one); the table sums the raw subvectors,
  // and n mu is taken off once per entry at the end.
  {
    const int warp = tid >> 5, lane = tid & 31;
    const int sub = lane / NG, g = lane % NG;
    const int copy = warp * TPW + sub;
    float4* my_sum = csum + static_cast<size_t>(copy) * NE + g;  // + 16-entry stride NG
    float* my_cnt = ccnt + static_cast<size_t>(copy) * NE + g;
    const float m0 = smu[4 * g], m1 = smu[4 * g + 1], m2 = smu[4 * g + 2], m3 = smu[4 * g + 3];
    const int t_first = t0 + copy;
    uint8_t* cbp = codes + (static_cast<size_t>(bh) * T + t_first) * NG + g;
    const __half* kp = kb + static_cast<size_t>(t_first) * D + 4 * g;
    for (int t = t_first; t < t1; t += U * TSTEP, cbp += U * TSTEP * NG, kp += U * TSTEP * D) {
      uint2 raw[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        raw[u] = t + u * TSTEP < t1 ? *reinterpret_cast<const uint2*>(kp + u * TSTEP * D)
                                    : make_uint2(0u, 0u);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (t + u * TSTEP >= t1) break;
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw[u].x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw[u].y));
        const int pt = (a.x > m0 ? 1 : 0) | (a.y > m1 ? 2 : 0) | (b.x > m2 ? 4 : 0) |
                       (b.y > m3 ? 8 : 0);
        cbp[u * TSTEP * NG] = static_cast<uint8_t>(pt);
        float4 sv = my_sum[pt * NG];
        sv.x += a.x;
        sv.y += a.y;
        sv.z += b.x;
        sv.w += b.y;
        my_sum[pt * NG] = sv;
        my_cnt[pt * NG] += 1.0f;
      }
    }
  }
  __syncthreads();
  // 4. the CTA's tables entry by entry (into table 0), then the cluster's
  for (int e = tid; e < NE; e += BUILD_THREADS) {
    float4 sv = csum[e];
    float n = ccnt[e];
    for (int q = 1; q < NCOPY; ++q) {
      const float4 o = csum[static_cast<size_t>(q) * NE + e];
      sv.x += o.x;
      sv.y += o.y;
      sv.z += o.z;
      sv.w += o.w;
      n += ccnt[static_cast<size_t>(q) * NE + e];
    }
    csum[e] = sv;
    ccnt[e] = n;
  }
  cluster.sync();
  {
    const int e0 = NE * r / CS, e1 = NE * (r + 1) / CS;
    for (int e = e0 + tid; e < e1; e += BUILD_THREADS) {
      float n = 0.0f;
      float4 sv = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      for (int q = 0; q < CS; ++q) {
        n += *cluster.map_shared_rank(&ccnt[e], q);
        const float4 o = *cluster.map_shared_rank(&csum[e], q);
        sv.x += o.x;
        sv.y += o.y;
        sv.z += o.z;
        sv.w += o.w;
      }
      // entry e = (pattern pt, group g); centroids are stored [group][pattern][4]
      // (the tables hold raw sums: the centred mean is sum / n - mu)
      const int pt = e / NG, g = e % NG;
      float* out = cent + ((static_cast<size_t>(bh) * NG + g) * 16 + pt) * 4;
      out[0] = n > 0.0f ? sv.x / n - smu[4 * g] : 0.0f;
      out[1] = n > 0.0f ? sv.y / n - smu[4 * g + 1] : 0.0f;
      out[2] = n > 0.0f ? sv.z / n - smu[4 * g + 2] : 0.0f;
      out[3] = n > 0.0f ? sv.w / n - smu[4 * g + 3] : 0.0f;
    }
  }
  cluster.sync();  // no CTA leaves while another still reads its shared memory
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

constexpr int SEL_THREADS = 1024;
constexpr int SEL_SMEM = 200 * 1024;  // staged keys: rows of up to 51200 positions
constexpr int SEL_RUN = 32;  // consecutive positions per thread in the ordered pass
constexpr int SEL_LOADS = 8; // row loads in flight per thread

// Exclusive prefix sums over the block's threads (in thread order) of two
// counts, and their block totals.  Every thread of the block calls it.
__device__ __forceinline__ int2 block_scan2(int a, int b, int2& total, int2* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int xa = __shfl_up_sync(0xffffffffu, ia, o), xb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) {
      ia += xa;
      ib += xb;
    }
  }
  if (lane == 31) wsum[warp] = make_int2(ia, ib);
  __syncthreads();
  if (warp == 0) {
    int2 w = lane < SEL_THREADS / 32 ? wsum[lane] : make_int2(0, 0);
    int sa = w.x, sb = w.y;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int xa = __shfl_up_sync(0xffffffffu, sa, o), xb = __shfl_up_sync(0xffffffffu, sb, o);
      if (lane >= o) {
        sa += xa;
        sb += xb;
      }
    }
    if (lane < SEL_THREADS / 32) wsum[lane] = make_int2(sa - w.x, sb - w.y);  // exclusive
    if (lane == SEL_THREADS / 32 - 1) wsum[SEL_THREADS / 32] = make_int2(sa, sb);
  }
  __syncthreads();
  const int2 base = wsum[warp];
  total = wsum[SEL_THREADS / 32];
  __syncthreads();  // wsum is reused by the next call
  return make_int2(base.x + ia - a, base.y + ib - b);
}

// The bin of a histogram (counted from the top bin down) in which the
// running count reaches `need`; writes the bin and the count still wanted
// inside it.  NB bins, NB / SEL_THREADS per thread.  Every thread calls it.
template <int NB>
__device__ __forceinline__ void find_bin(const int* hist, int need, int* s_bin, int* s_need,
                                         int2* wsum) {
  constexpr int PER = NB / SEL_THREADS;
  const int top = NB - 1 - PER * static_cast<int>(threadIdx.x);  // this thread's bins: top, top-1, ...
  int c[PER], local = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    c[i] = hist[top - i];
    local += c[i];
  }
  int2 tot;
  const int before = block_scan2(local, 0, tot, wsum).x;
  if (before < need && before + local >= need) {
    int cum = before;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      if (cum + c[i] >= need) {
        *s_bin = top - i;
        *s_need = need - cum;
        break;
      }
      cum += c[i];
    }
  }
  __syncthreads();
}

// Top-k of each row of scores over the positions [lo, T), one row at a time
// per CTA (persistent over the rows).  The row's ordered keys are staged in
// shared memory when they fit (else re-read from global memory); a radix
// select over three digits (11, 11 and 10 bits, most significant first) finds
// the k-th largest key K* and how many keys equal to K* are taken; one
// ordered pass then writes every position with a key above K* and the first
// of those equal to K*: ties go to the lower position and the output is
// sorted.  Thread i of the ordered pass owns SEL_RUN consecutive positions:
// it keeps their comparisons as bit masks, and two block scans give its tie
// rank and its output slot.
__global__ void __launch_bounds__(SEL_THREADS, 1) select_kernel(const float* __restrict__ scores,
                                                                int rows, int T, int lo, int k_eff,
                                                                int k_cap, int cap_keys,
                                                                int32_t* __restrict__ picked) {
  extern __shared__ uint32_t skey[];  // [cap_keys]
  __shared__ int hist[2048];
  __shared__ int2 wsum[SEL_THREADS / 32 + 1];
  __shared__ int s_bin, s_need;
  const int tid = threadIdx.x;
  const int L = T - lo;
  const bool staged = L <= cap_keys;
  for (int row = blockIdx.x; row < rows; row += gridDim.x) {
    const float* s = scores + static_cast<size_t>(row) * T + lo;
    int32_t* out = picked + static_cast<size_t>(row) * k_cap;
    for (int i = k_eff + tid; i < k_cap; i += SEL_THREADS) out[i] = -1;
    if (k_eff <= 0 || L <= 0) continue;
    if (tid == 0 && row + static_cast<int>(gridDim.x) < rows) {
      // the CTA's next row into L2 while this one is worked on (16-byte
      // aligned interior of the row only)
      const char* nb = reinterpret_cast<const char*>(s + static_cast<size_t>(gridDim.x) * T);
      const uintptr_t b0 = (reinterpret_cast<uintptr_t>(nb) + 15) & ~static_cast<uintptr_t>(15);
      const uintptr_t b1 = (reinterpret_cast<uintptr_t>(nb) + 4ull * L) & ~static_cast<uintptr_t>(15);
      if (b1 > b0)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(b0),
                     "r"(static_cast<uint32_t>(b1 - b0))
                     : "memory");
    }
    // digit 1: bits 31..21
    for (int i = tid; i < 2048; i += SEL_THREADS) hist[i] = 0;
    __syncthreads();
    for (int i0 = tid; i0 < L; i0 += SEL_LOADS * SEL_THREADS) {
      float v[SEL_LOADS];  // all loads of the round in flight before the updates
#pragma unroll
      for (int j = 0; j < SEL_LOADS; ++j) {
        const int i = i0 + j * SEL_THREADS;
        v[j] = i < L ? s[i] : 0.0f;
      }
#pragma unroll
      for (int j = 0; j < SEL_LOADS; ++j) {
        const int i = i0 + j * SEL_THREADS;
        if (i < L) {
          const uint32_t key = order_key(v[j]);
          if (staged) skey[i] = key;
          atomicAdd(&hist[key >> 21], 1);
        }
      }
    }
    __syncthreads();
    find_bin<2048>(hist, k_eff, &s_bin, &s_need, wsum);
    uint32_t prefix = static_cast<uint32_t>(s_bin) << 21;
    int need = s_need;
    // digit 2: bits 20..10 of the keys under the prefix
    for (int i = tid; i < 2048; i += SEL_THREADS) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < L; i += SEL_THREADS) {
      const uint32_t key = staged ? skey[i] : order_key(s[i]);
      if ((key >> 21) == (prefix >> 21)) atomicAdd(&hist[(key >> 10) & 2047u], 1);
    }
    __syncthreads();
    find_bin<2048>(hist, need, &s_bin, &s_need, wsum);
    prefix |= static_cast<uint32_t>(s_bin) << 10;
    need = s_need;
    // digit 3: bits 9..0
    for (int i = tid; i < 1024; i += SEL_THREADS) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < L; i += SEL_THREADS) {
      const uint32_t key = staged ? skey[i] : order_key(s[i]);
      if ((key >> 10) == (prefix >> 10)) atomicAdd(&hist[key & 1023u], 1);
    }
    __syncthreads();
    find_bin<1024>(hist, need, &s_bin, &s_need, wsum);
    prefix |= static_cast<uint32_t>(s_bin);
    need = s_need;
    // ordered pass over runs of SEL_RUN positions
    int taken = 0, ties = 0;
    const int lane_rot = tid & (SEL_RUN - 1);
    for (int c0 = 0; c0 < L && taken < k_eff; c0 += SEL_THREADS * SEL_RUN) {
      const int p0 = c0 + tid * SEL_RUN;
      uint32_t gt = 0u, eq = 0u;
#pragma unroll 8
      for (int j = 0; j < SEL_RUN; ++j) {
        const int jj = (j + lane_rot) & (SEL_RUN - 1);  // rotated: no bank conflicts
        const int pos = p0 + jj;
        if (pos < L) {
          const uint32_t key = staged ? skey[pos] : order_key(s[pos]);
          gt |= (key > prefix ? 1u : 0u) << jj;
          eq |= (key == prefix ? 1u : 0u) << jj;
        }
      }
      int2 tot;
      const int n_eq = __popc(eq);
      const int tie0 = ties + block_scan2(n_eq, 0, tot, wsum).x;
      const int take = max(0, min(n_eq, need - tie0));
      uint32_t sel = gt, e = eq;
      for (int i = 0; i < take; ++i) {  // the first `take` ties, lowest positions first
        sel |= e & (~e + 1u);
        e &= e - 1u;
      }
      ties += tot.x;
      const int slot0 = taken + block_scan2(__popc(sel), 0, tot, wsum).x;
      int slot = slot0;
      while (sel) {
        const int j = __ffs(static_cast<int>(sel)) - 1;
        sel &= sel - 1u;
        if (slot < k_eff) out[slot] = lo + p0 + j;
        ++slot;
      }
      taken += tot.x;
    }
    __syncthreads();  // hist, skey and the shared words are reused by the next row
  }
}

// Exact softmax attention of one query head over the sinks [0, n_s) and its
// selected positions, with the stored fp16 keys and values.  A token is read
// by LPT = D / 8 lanes (16 bytes of its key and of its value each), so a warp
// reads 32 / LPT tokens per round and keeps AT_U rounds in flight; the
// positions of the next rounds are loaded one step ahead.  Every lane group
// keeps its own running maximum, sum and weighted value (base-2 softmax with
// the scale folded into the query); the groups and warps are merged at the
// end.  A picked position outside [0, T) is skipped and reported.
constexpr int AT_WARPS = 8;
constexpr int AT_U = 2;

template <int D>
__global__ void __launch_bounds__(AT_WARPS * 32) attend_kernel(const void* q, int q_dtype, int Hq,
                                                               int Hkv, int T,
                                                               const __half* __restrict__ keys,
                                                               const __half* __restrict__ values,
                                                               const int32_t* __restrict__ picked,
                                                               int k_cap, int k_eff, int n_s,
                                                               float scale, float* __restrict__ out,
                                                               int* err) {
  constexpr int LPT = D / 8;        // lanes per token
  constexpr int NSUB = 32 / LPT;    // tokens per warp per round
  constexpr int NPART = AT_WARPS * NSUB;
  constexpr int STEP = AT_WARPS * NSUB * AT_U;  // tokens per CTA per step
  const int row = blockIdx.x, b = row / Hq, hq = row % Hq, kvh = hq / (Hq / Hkv);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPT, sl = lane % LPT;
  const size_t base = static_cast<size_t>(b * Hkv + kvh) * T * D + sl * 8;
  const int32_t* prow = picked + static_cast<size_t>(row) * k_cap;
  __shared__ float sm[NPART], sls[NPART];
  __shared__ float sacc[NPART][D];
  const float sl2 = scale * 1.4426950408889634f;  // softmax in base 2
  float qv[8], acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    qv[i] = load_as_float(q, static_cast<size_t>(row) * D + sl * 8 + i,
                          static_cast<tq_dtype>(q_dtype)) * sl2;
    acc[i] = 0.0f;
  }
  float m = -INFINITY, l = 0.0f;
  const int n = n_s + k_eff;
  const int first = (warp * AT_U) * NSUB + sub;  // this lane group's token of round 0
  auto pos_of = [&](int j) -> int {
    if (j >= n) return -2;  // past the end: no token
    return j < n_s ? j : __ldg(prow + (j - n_s));
  };
  int pos[AT_U];
#pragma unroll
  for (int u = 0; u < AT_U; ++u) pos[u] = pos_of(first + u * NSUB);
  for (int j0 = 0; j0 < n; j0 += STEP) {
    uint4 kr[AT_U], vr[AT_U];
    bool ok[AT_U];
#pragma unroll
    for (int u = 0; u < AT_U; ++u) {
      ok[u] = pos[u] >= 0 && pos[u] < T;
      if (pos[u] != -2 && !ok[u] && sl == 0) report(err, TQ_ERR_INVALID_ARG);
      const size_t off = base + static_cast<size_t>(ok[u] ? pos[u] : 0) * D;
      kr[u] = ok[u] ? *reinterpret_cast<const uint4*>(keys + off) : make_uint4(0u, 0u, 0u, 0u);
      vr[u] = ok[u] ? *reinterpret_cast<const uint4*>(values + off) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < AT_U; ++u) pos[u] = pos_of(first + j0 + STEP + u * NSUB);
#pragma unroll
    for (int u = 0; u < AT_U; ++u) {
      const uint32_t kw[4] = {kr[u].x, kr[u].y, kr[u].z, kr[u].w};
      float dot = 0.0f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&kw[e]));
        dot = fmaf(f.x, qv[2 * e], fmaf(f.y, qv[2 * e + 1], dot));
      }
#pragma unroll
      for (int o = LPT / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (!ok[u]) continue;
      const float mn = fmaxf(m, dot);
      const float corr = exp2f(m - mn), pr = exp2f(dot - mn);
      l = fmaf(l, corr, pr);
      const uint32_t vw[4] = {vr[u].x, vr[u].y, vr[u].z, vr[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&vw[e]));
        acc[2 * e] = fmaf(acc[2 * e], corr, pr * f.x);
        acc[2 * e + 1] = fmaf(acc[2 * e + 1], corr, pr * f.y);
      }
      m = mn;
    }
  }
  const int part = warp * NSUB + sub;
#pragma unroll
  for (int i = 0; i < 8; ++i) sacc[part][sl * 8 + i] = acc[i];
  if (sl == 0) {
    sm[part] = m;
    sls[part] = l;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float M = -INFINITY;
    for (int w = 0; w < NPART; ++w) M = fmaxf(M, sm[w]);
    float L = 0.0f, o = 0.0f;
    if (M != -INFINITY) {
      for (int w = 0; w < NPART; ++w) {
        const float f = exp2f(sm[w] - M);
        L = fmaf(sls[w], f, L);
        o = fmaf(sacc[w][c], f, o);
      }
    }
    out[static_cast<size_t>(row) * D + c] = L > 0.0f ? o / L : 0.0f;
  }
}

}  // namespace six

// Cluster size of the index build: 16 CTAs per kv head where the device can
// co-schedule such clusters (non-portable size), else 8; found once per
// device and head dimension.
template <int D>
static int build_cluster(cudaLaunchConfig_t cfg, cudaLaunchAttribute attr) {
  static std::mutex mu;
  static int known[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (known[dev]) return known[dev];
  auto kern = six::build_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           six::BUILD_SMEM) != cudaSuccess)
    return 0;
  const bool wide = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                    cudaSuccess;
  cudaGetLastError();
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  for (int cs : {16, 8}) {
    if (cs > 8 && !wide) continue;
    attr.val.clusterDim.x = cs;
    cfg.gridDim = dim3(cs);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) {
      known[dev] = cs;
      return cs;
    }
    cudaGetLastError();
  }
  return 0;
}

int launch_self_index_build(const tq_ctx* ctx, const void* k, int B, int Hkv, int T, float* mu,
                            uint8_t* codes, float* cent, void* stream) {
  const __half* kh = static_cast<const __half*>(k);
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr{};
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 1;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.blockDim = dim3(six::BUILD_THREADS);
  cfg.dynamicSmemBytes = six::BUILD_SMEM;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  const bool d128 = ctx->cfg.head_dim == 128;
  const int cs = d128 ? build_cluster<128>(cfg, attr) : build_cluster<64>(cfg, attr);
  if (cs == 0) return TQ_ERR_CUDA;
  attr.val.clusterDim.x = cs;
  cfg.gridDim = dim3(static_cast<unsigned>(B * Hkv * cs));
  const cudaError_t e = d128 ? cudaLaunchKernelEx(&cfg, six::build_kernel<128>, kh, T, mu, codes, cent)
                             : cudaLaunchKernelEx(&cfg, six::build_kernel<64>, kh, T, mu, codes, cent);
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
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

int launch_self_index_select(const tq_ctx* ctx, const float* scores, int rows, int T, int lo,
                            int k_eff, int k_cap, int32_t* picked, void* stream) {
  (void)ctx;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  static std::mutex mu;
  static int sms[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TQ_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!sms[dev]) {
      if (cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
          cudaFuncSetAttribute(six::select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               six::SEL_SMEM) != cudaSuccess)
        return TQ_ERR_CUDA;
    }
  }
  const int L = T - lo;
  const int cap_keys = six::SEL_SMEM / 4;
  const size_t smem = L > 0 && L <= cap_keys ? static_cast<size_t>(L) * 4 : 0;
  const int grid = rows < sms[dev] ? rows : sms[dev];
  six::select_kernel<<<grid, six::SEL_THREADS, smem, st>>>(scores, rows, T, lo, k_eff, k_cap,
                                                           cap_keys, picked);
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
    six::attend_kernel<128><<<B * Hq, six::AT_WARPS * 32, 0, st>>>(q, qd, Hq, Hkv, T, kh, vh, picked, k_cap,
                                                    k_eff, n_s, scale, out, ctx->dev.err);
  else
    six::attend_kernel<64><<<B * Hq, six::AT_WARPS * 32, 0, st>>>(q, qd, Hq, Hkv, T, kh, vh, picked, k_cap,
                                                   k_eff, n_s, scale, out, ctx->dev.err);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace tq
