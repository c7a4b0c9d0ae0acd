// Compressed inner-product search ("TurboQuant" summary, de.news.hada.io
// topic 27867, section "Leistung bei der Vektorsuche"): the estimated inner
// product of each query with every keys-only database record,
//   n * ( <Pi q, c_hat> + sqrt(pi/2)/m * gamma * <S Pi q, 1 - 2 bits> ),
// then the k best per query (ties to the lower id).
//
// Launches:
//  1. qprep   per query: q_rot, q_s, estimator constants folded in, per-query
//             power-of-two prescale, fp16 hi/lo split, stored as the B matrix
//             of the tensor-core contraction in MMA k-index order.
//  2. score   persistent CTAs over (query tile of 32, database slice) items.
//             Each warp unpacks 32 database records at a time straight from
//             global memory (L2-resident) into exact {0, +-1, +-2^-7, +-gamma}
//             fp16 fragments and contracts them with the query tile held in
//             shared memory (m16n8k16 MMAs, fp32 accumulate); a threshold filter
//             feeds rare insertions into per-warp top-k lists in shared memory.
//  3. merge   per query: the best k of all per-warp lists.
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace tk {

constexpr int NWARP = 8;
constexpr int QT = 32;  // queries per tile (64 B columns: hi, lo)
constexpr float NEG_INF = -__builtin_huge_valf();

template <int D>
struct Cfg {
  static constexpr int KS = D / 16;
  static constexpr int KTOT = 3 * D;          // k extent: sign plane, magnitude plane, QJL plane
  static constexpr int RB = 2 * KTOT + 16;    // padded B row bytes
  static constexpr int NTQ = 2 * QT / 8;      // n-tiles per query tile
  static constexpr int SMEM_B = 2 * QT * RB;  // B tile
};

struct Params {
  const float* queries;
  int Q;
  const uint8_t* db;
  long long N;
  int k;
  long long page_bytes;
  int off_kc, off_qs, off_kn, off_kg;
  const float* rot;
  const float* qjl;
  float kc0, kc1, alpha;
  uint16_t* bmat;    // [Q * 2][KTOT] fp16 bits (rows: query hi, query lo)
  float* desc;       // [Q] descale
  float* cand_s;     // [items][NWARP][QT][k]
  int* cand_i;
  int n_slices;
  long long pages;
  int* err;
};

// coordinate fed by MMA k-index kk (0..15) of key k-step s for lane column c
template <int D>
__device__ __forceinline__ int key_coord(int s, int kk) {
  const int c = (kk & 7) >> 1, e = kk & 1, reg = kk >> 3;
  const int P = c * (D / 8) + 2 * s + reg;
  return 16 * (P >> 3) + (P & 7) + 8 * e;
}

template <int D>
__device__ __forceinline__ int qjl_index(int s, int kk) {
  const int c = (kk & 7) >> 1, e = kk & 1, reg = kk >> 3;
  const int P = c * (D / 8) + 2 * s + reg;
  return 32 * (P >> 4) + (P & 15) + 16 * e;
}

// y[r] = sum_k M[r][k] x[k]: one warp per row, float4 per lane, shuffle reduce
template <int D>
__device__ __forceinline__ void warp_matvec(const float* __restrict__ M, const float* x, float* y) {
  constexpr int LANES = D / 4, RPP = 32 / LANES, NW = 4, PASSES = D / (NW * RPP);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, sub = lane / LANES, l4 = lane % LANES;
  float4 m[PASSES];
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps)
    m[ps] = __ldg(reinterpret_cast<const float4*>(M + static_cast<size_t>((ps * NW + warp) * RPP + sub) * D) + l4);
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    float a = m[ps].x * x[4 * l4] + m[ps].y * x[4 * l4 + 1] + m[ps].z * x[4 * l4 + 2] + m[ps].w * x[4 * l4 + 3];
#pragma unroll
    for (int o = LANES / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (l4 == 0) y[(ps * NW + warp) * RPP + sub] = a;
  }
}

template <int D>
__global__ void __launch_bounds__(128) qprep_kernel(Params p) {
  using C = Cfg<D>;
  const int q = blockIdx.x;
  __shared__ float sq[D], sr[D], ss[D];
  __shared__ unsigned smax;
  __shared__ float sfac;
  const int tid = threadIdx.x;
  if (tid == 0) smax = 0u;
  for (int j = tid; j < D; j += blockDim.x) sq[j] = p.queries[static_cast<size_t>(q) * D + j];
  __syncthreads();
  warp_matvec<D>(p.rot, sq, sr);
  __syncthreads();
  warp_matvec<D>(p.qjl, sr, ss);
  __syncthreads();
  const float w1 = p.kc0, w2 = 128.0f * (p.kc1 - p.kc0), w3 = p.alpha;
  for (int j = tid; j < D; j += blockDim.x) {
    const float m = fmaxf(fmaxf(fabsf(w1 * sr[j]), fabsf(w2 * sr[j])), fabsf(w3 * ss[j]));
    atomicMax(&smax, __float_as_uint(m));
  }
  __syncthreads();
  if (tid == 0) {
    const float mx = __uint_as_float(smax);
    float f = 1.0f;
    if (mx > 0.0f && isfinite(mx)) {
      int e;
      frexpf(mx, &e);
      f = ldexpf(1.0f, 8 - e);
    }
    sfac = f;
    p.desc[q] = 1.0f / f;
  }
  __syncthreads();
  const float f = sfac;
  for (int kk = tid; kk < C::KTOT; kk += blockDim.x) {
    const int plane = kk / D, s = (kk % D) / 16, ki = kk % 16;
    float w;
    if (plane == 0) w = w1 * sr[key_coord<D>(s, ki)];
    else if (plane == 1) w = w2 * sr[key_coord<D>(s, ki)];
    else w = w3 * ss[qjl_index<D>(s, ki)];
    uint16_t hi, lo;
    split_f16(f * w, hi, lo);
    p.bmat[(static_cast<size_t>(q) * 2) * C::KTOT + kk] = hi;
    p.bmat[(static_cast<size_t>(q) * 2 + 1) * C::KTOT + kk] = lo;
  }
}

__device__ __forceinline__ bool better(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

// insert (s, id) into a sorted (best first) list of k entries
__device__ __forceinline__ void list_insert(float* ls, int* li, int k, float s, int id) {
  if (!better(s, id, ls[k - 1], li[k - 1])) return;
  int pos = k - 1;
  while (pos > 0 && better(s, id, ls[pos - 1], li[pos - 1])) {
    ls[pos] = ls[pos - 1];
    li[pos] = li[pos - 1];
    --pos;
  }
  ls[pos] = s;
  li[pos] = id;
}

template <int D>
__global__ void __launch_bounds__(NWARP * 32, 1) score_kernel(Params p) {
  using C = Cfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  uint8_t* bt = smem;
  float* ls_all = reinterpret_cast<float*>(smem + C::SMEM_B);
  int* li_all = reinterpret_cast<int*>(smem + C::SMEM_B + NWARP * QT * p.k * 4);
  float* ls = ls_all + warp * QT * p.k;
  int* li = li_all + warp * QT * p.k;

  const int n_qt = (p.Q + QT - 1) / QT;
  const int items = n_qt * p.n_slices;
  const int qword = (c * (D / 8)) >> 4, qsb = (c * (D / 8)) & 15;
  const uint32_t b_base = smem_u32(bt) + ((lane & 7) + ((lane >> 4) & 1) * 8) * C::RB + ((lane >> 3) & 1) * 16;

  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int qt = item % n_qt, sl = item / n_qt;
    const int q0 = qt * QT;
    // query tile: rows 2*i (hi) and 2*i+1 (lo) of the B matrix
    __syncthreads();
    for (int i = tid; i < 2 * QT * (C::KTOT / 8); i += blockDim.x) {
      const int row = i / (C::KTOT / 8), ch = i % (C::KTOT / 8);
      const int qq = q0 + row / 2;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (qq < p.Q)
        v = reinterpret_cast<const uint4*>(p.bmat + (static_cast<size_t>(q0) * 2 + row) * C::KTOT)[ch];
      reinterpret_cast<uint4*>(bt + row * C::RB)[ch] = v;
    }
    for (int i = lane; i < QT * p.k; i += 32) {
      ls[i] = NEG_INF;
      li[i] = 0x7fffffff;
    }
    __syncthreads();
    // thresholds and descales of this lane's queries (n-tile t -> query 4t + c)
    float thr_s[C::NTQ];
    int thr_i[C::NTQ];
    float dq[C::NTQ];
#pragma unroll
    for (int t = 0; t < C::NTQ; ++t) {
      thr_s[t] = NEG_INF;
      thr_i[t] = 0x7fffffff;
      const int qq = q0 + 4 * t + c;
      dq[t] = (qq < p.Q) ? p.desc[qq] : 0.0f;
    }
    const long long pg0 = p.pages * sl / p.n_slices, pg1 = p.pages * (sl + 1) / p.n_slices;
    // the 32 records of step grp; the next step's words are requested before
    // the current step's contraction so the L2 latency overlaps it
    uint32_t kw_n[2][2][D / 64], qw_n[2][2];
    uint16_t gg_n[2][2], nn_n[2][2];
    auto fetch = [&](long long grp) {
      const long long page = grp >> 2;
      const int slot0 = static_cast<int>(grp & 3) * 32;
      const uint8_t* pgp = p.db + page * p.page_bytes;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int slot = slot0 + 16 * mt + g + 8 * r;
#pragma unroll
          for (int w = 0; w < D / 64; ++w)
            kw_n[mt][r][w] = __ldg(reinterpret_cast<const uint32_t*>(pgp + p.off_kc + slot * (D / 4)) + c * (D / 64) + w);
          qw_n[mt][r] = __ldg(reinterpret_cast<const uint32_t*>(pgp + p.off_qs + slot * (D / 8)) + qword);
          gg_n[mt][r] = __ldg(reinterpret_cast<const uint16_t*>(pgp + p.off_kg) + slot);
          nn_n[mt][r] = __ldg(reinterpret_cast<const uint16_t*>(pgp + p.off_kn) + slot);
        }
      }
    };
    if (pg0 * 4 + warp < pg1 * 4) fetch(pg0 * 4 + warp);
    for (long long grp = pg0 * 4 + warp; grp < pg1 * 4; grp += NWARP) {
      const long long page = grp >> 2;
      const int slot0 = static_cast<int>(grp & 3) * 32;
      float acc[2][C::NTQ][4];
      uint32_t kw[2][2][D / 64], qw[2][2];
      uint32_t gg[2][2];
      float nn[2][2];
      int ids[2][2];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          ids[mt][r] = static_cast<int>(page * TQ_PAGE_TOKENS + slot0 + 16 * mt + g + 8 * r);
#pragma unroll
          for (int w = 0; w < D / 64; ++w) kw[mt][r][w] = kw_n[mt][r][w];
          qw[mt][r] = qw_n[mt][r];
          gg[mt][r] = static_cast<uint32_t>(gg_n[mt][r]) * 0x10001u;
          nn[mt][r] = __half2float(__ushort_as_half(nn_n[mt][r]));
        }
#pragma unroll
        for (int t = 0; t < C::NTQ; ++t) acc[mt][t][0] = acc[mt][t][1] = acc[mt][t][2] = acc[mt][t][3] = 0.0f;
      }
      if (grp + NWARP < pg1 * 4) fetch(grp + NWARP);
      // key planes: k-steps 0..KS-1 (sign) and KS..2KS-1 (magnitude)
#pragma unroll
      for (int s = 0; s < C::KS; ++s) {
        const int w = s >> 2, sh = 4 * (s & 3);
        uint32_t a1[2][4], a2[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const uint32_t x0a = kw[mt][0][w] << sh, x0b = kw[mt][0][w] << (sh + 1);
          const uint32_t x1a = kw[mt][1][w] << sh, x1b = kw[mt][1][w] << (sh + 1);
          a1[mt][0] = (x0a & 0x80008000u) | 0x3C003C00u;
          a1[mt][1] = (x1a & 0x80008000u) | 0x3C003C00u;
          a1[mt][2] = (x0b & 0x80008000u) | 0x3C003C00u;
          a1[mt][3] = (x1b & 0x80008000u) | 0x3C003C00u;
          a2[mt][0] = x0a & 0xA000A000u;
          a2[mt][1] = x1a & 0xA000A000u;
          a2[mt][2] = x0b & 0xA000A000u;
          a2[mt][3] = x1b & 0xA000A000u;
        }
#pragma unroll
        for (int t = 0; t < C::NTQ; t += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(b_base + t * 8 * C::RB + s * 32, b0, b1, b2, b3);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            mma_f16(acc[mt][t], a1[mt][0], a1[mt][1], a1[mt][2], a1[mt][3], b0, b1);
            mma_f16(acc[mt][t + 1], a1[mt][0], a1[mt][1], a1[mt][2], a1[mt][3], b2, b3);
          }
          ldsm_x4(b_base + t * 8 * C::RB + (C::KS + s) * 32, b0, b1, b2, b3);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            mma_f16(acc[mt][t], a2[mt][0], a2[mt][1], a2[mt][2], a2[mt][3], b0, b1);
            mma_f16(acc[mt][t + 1], a2[mt][0], a2[mt][1], a2[mt][2], a2[mt][3], b2, b3);
          }
        }
      }
      // QJL plane: k-steps 2KS .. 3KS-1
#pragma unroll
      for (int s = 0; s < C::KS; ++s) {
        const int sh = qsb + 2 * s;
        uint32_t a3[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          a3[mt][0] = ((qw[mt][0] << sh) & 0x80008000u) | gg[mt][0];
          a3[mt][1] = ((qw[mt][1] << sh) & 0x80008000u) | gg[mt][1];
          a3[mt][2] = ((qw[mt][0] << (sh + 1)) & 0x80008000u) | gg[mt][0];
          a3[mt][3] = ((qw[mt][1] << (sh + 1)) & 0x80008000u) | gg[mt][1];
        }
#pragma unroll
        for (int t = 0; t < C::NTQ; t += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(b_base + t * 8 * C::RB + (2 * C::KS + s) * 32, b0, b1, b2, b3);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            mma_f16(acc[mt][t], a3[mt][0], a3[mt][1], a3[mt][2], a3[mt][3], b0, b1);
            mma_f16(acc[mt][t + 1], a3[mt][0], a3[mt][1], a3[mt][2], a3[mt][3], b2, b3);
          }
        }
      }
      // threshold filter, rare insertions (one candidate at a time per warp)
#pragma unroll
      for (int t = 0; t < C::NTQ; ++t) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float s = (acc[mt][t][2 * r] + acc[mt][t][2 * r + 1]) * dq[t] * nn[mt][r];
            const int id = ids[mt][r];
            const bool valid = id < p.N && (q0 + 4 * t + c) < p.Q;
            const bool cand = valid && better(s, id, thr_s[t], thr_i[t]);
            unsigned mask = __ballot_sync(0xffffffffu, cand);
            while (mask) {
              const int src = __ffs(mask) - 1;
              mask &= mask - 1;
              const int qc = src & 3;  // query 4t + qc of the tile
              if (lane == src) list_insert(ls + (4 * t + qc) * p.k, li + (4 * t + qc) * p.k, p.k, s, id);
              __syncwarp();
              if (c == qc) {
                thr_s[t] = ls[(4 * t + qc) * p.k + p.k - 1];
                thr_i[t] = li[(4 * t + qc) * p.k + p.k - 1];
              }
            }
          }
        }
      }
    }
    __syncwarp();
    // per-warp lists -> global candidates of this item
    const size_t base = (static_cast<size_t>(item) * NWARP + warp) * QT * p.k;
    for (int i = lane; i < QT * p.k; i += 32) {
      p.cand_s[base + i] = ls[i];
      p.cand_i[base + i] = li[i];
    }
  }
}

// per query: the best k among n_slices * NWARP lists of k candidates
__global__ void __launch_bounds__(128) merge_kernel(Params p, int32_t* out_ids, float* out_scores) {
  const int q = blockIdx.x;
  const int qt = q / QT, qi = q % QT;
  const int n_qt = (p.Q + QT - 1) / QT;
  const int lists = p.n_slices * NWARP;
  extern __shared__ uint8_t sm[];
  float* cs = reinterpret_cast<float*>(sm);
  int* ci = reinterpret_cast<int*>(sm + sizeof(float) * lists * p.k);
  __shared__ float rs[4];
  __shared__ int ri[4], rp[4];
  const int total = lists * p.k;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int l = i / p.k, e = i % p.k;
    const int sl = l / NWARP, w = l % NWARP;
    const int item = sl * n_qt + qt;
    const size_t src = ((static_cast<size_t>(item) * NWARP + w) * QT + qi) * p.k + e;
    cs[i] = p.cand_s[src];
    ci[i] = p.cand_i[src];
  }
  __syncthreads();
  for (int r = 0; r < p.k; ++r) {
    float bs = NEG_INF;
    int bi = 0x7fffffff, bp = -1;
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
      if (ci[i] != 0x7fffffff && (bp < 0 || better(cs[i], ci[i], bs, bi))) {
        bs = cs[i];
        bi = ci[i];
        bp = i;
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      const int op = __shfl_xor_sync(0xffffffffu, bp, o);
      if (op >= 0 && (bp < 0 || better(os, oi, bs, bi))) {
        bs = os;
        bi = oi;
        bp = op;
      }
    }
    if ((threadIdx.x & 31) == 0) {
      rs[threadIdx.x >> 5] = bs;
      ri[threadIdx.x >> 5] = bi;
      rp[threadIdx.x >> 5] = bp;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = rs[0];
      int id = ri[0], pos = rp[0];
      for (int w = 1; w < 4; ++w)
        if (rp[w] >= 0 && (pos < 0 || better(rs[w], ri[w], s, id))) {
          s = rs[w];
          id = ri[w];
          pos = rp[w];
        }
      out_scores[static_cast<size_t>(q) * p.k + r] = (pos >= 0) ? s : NEG_INF;
      out_ids[static_cast<size_t>(q) * p.k + r] = (pos >= 0) ? id : -1;
      if (pos >= 0) ci[pos] = 0x7fffffff;  // taken
    }
    __syncthreads();
  }
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Ws {
  size_t bmat, desc, cs, ci, total;
};

inline int n_slices_for(const tq_ctx* ctx, int Q, long long pages) {
  const int n_qt = (Q + QT - 1) / QT;
  // enough items to fill every SM several times, slices of at least a few pages
  long long want = (static_cast<long long>(ctx->num_sms) * 4 + n_qt - 1) / n_qt;
  if (want < 1) want = 1;
  if (want > pages) want = pages;
  return static_cast<int>(want);
}

Ws ws_layout(const tq_ctx* ctx, int Q, long long N, int k) {
  const int d = ctx->cfg.head_dim;
  const long long pages = (N + TQ_PAGE_TOKENS - 1) / TQ_PAGE_TOKENS;
  const int n_qt = (Q + QT - 1) / QT;
  const int ns = n_slices_for(ctx, Q, pages);
  const size_t items = static_cast<size_t>(n_qt) * ns;
  Ws w;
  size_t off = 0;
  w.bmat = off;
  off = align256(off + sizeof(uint16_t) * static_cast<size_t>(n_qt) * QT * 2 * 3 * d);
  w.desc = off;
  off = align256(off + sizeof(float) * static_cast<size_t>(n_qt) * QT);
  w.cs = off;
  off = align256(off + sizeof(float) * items * NWARP * QT * k);
  w.ci = off;
  off = align256(off + sizeof(int) * items * NWARP * QT * k);
  w.total = off;
  return w;
}

}  // namespace tk

size_t topk_workspace_bytes(const tq_ctx* ctx, int Q, int64_t N, int k) {
  return tk::ws_layout(ctx, Q, N, k).total;
}

int launch_topk(const tq_ctx* ctx, const float* queries, int Q, const uint8_t* db, int64_t N,
                int k, int32_t* out_ids, float* out_scores, void* ws, size_t ws_bytes,
                void* stream) {
  const int d = ctx->cfg.head_dim;
  const tk::Ws L = tk::ws_layout(ctx, Q, N, k);
  if (ws_bytes < L.total) return TQ_ERR_INVALID_ARG;
  const PageLayout pl = page_layout(d, ctx->cfg.qjl_dim, false);
  tk::Params p{};
  p.queries = queries;
  p.Q = Q;
  p.db = db;
  p.N = N;
  p.k = k;
  p.page_bytes = static_cast<long long>(pl.bytes);
  p.off_kc = static_cast<int>(pl.kc);
  p.off_qs = static_cast<int>(pl.qs);
  p.off_kn = static_cast<int>(pl.kn);
  p.off_kg = static_cast<int>(pl.kg);
  p.rot = ctx->dev.rot;
  p.qjl = ctx->dev.qjl;
  p.kc0 = ctx->cb.key_c[0];
  p.kc1 = ctx->cb.key_c[1];
  p.alpha = 1.2533141373155001f / static_cast<float>(ctx->cfg.qjl_dim);
  uint8_t* base = static_cast<uint8_t*>(ws);
  p.bmat = reinterpret_cast<uint16_t*>(base + L.bmat);
  p.desc = reinterpret_cast<float*>(base + L.desc);
  p.cand_s = reinterpret_cast<float*>(base + L.cs);
  p.cand_i = reinterpret_cast<int*>(base + L.ci);
  p.pages = (N + TQ_PAGE_TOKENS - 1) / TQ_PAGE_TOKENS;
  p.n_slices = tk::n_slices_for(ctx, Q, p.pages);
  p.err = ctx->dev.err;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int n_qt = (Q + tk::QT - 1) / tk::QT;
  const int items = n_qt * p.n_slices;
  const int grid = items < ctx->num_sms ? items : ctx->num_sms;
  const size_t merge_smem = static_cast<size_t>(p.n_slices) * tk::NWARP * k * 8;
  if (merge_smem > 200 * 1024) return TQ_ERR_UNSUPPORTED;
  // queries of the last partial tile are read as zero rows by the scorer;
  // the B matrix has room for whole tiles
  auto go = [&](auto dtag) -> int {
    constexpr int D = decltype(dtag)::value;
    using C = tk::Cfg<D>;
    const size_t smem = C::SMEM_B + static_cast<size_t>(tk::NWARP) * tk::QT * k * 8;
    static bool set = false;
    if (!set) {
      if (cudaFuncSetAttribute(tk::score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               232448) != cudaSuccess)
        return TQ_ERR_CUDA;
      set = true;
    }
    if (smem > 232448) return TQ_ERR_UNSUPPORTED;
    tk::qprep_kernel<D><<<Q, 128, 0, st>>>(p);
    if (ctx->prof_start) cudaEventRecord(static_cast<cudaEvent_t>(ctx->prof_start), st);
    tk::score_kernel<D><<<grid, tk::NWARP * 32, smem, st>>>(p);
    if (ctx->prof_stop) cudaEventRecord(static_cast<cudaEvent_t>(ctx->prof_stop), st);
    if (merge_smem > 48 * 1024 &&
        cudaFuncSetAttribute(tk::merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(merge_smem)) != cudaSuccess)
      return TQ_ERR_CUDA;
    tk::merge_kernel<<<Q, 128, merge_smem, st>>>(p, out_ids, out_scores);
    return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
  };
  if (d == 128) return go(std::integral_constant<int, 128>{});
  if (d == 64) return go(std::integral_constant<int, 64>{});
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq
