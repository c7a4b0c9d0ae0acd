// Compressed inner-product search ("TurboQuant" summary, de.news.hada.io
// topic 27867, section "Leistung bei der Vektorsuche"): the estimated inner
// product of each query with every keys-only database record,
//   n * ( <Pi q, c_hat> + sqrt(pi/2)/m * gamma * <S Pi q, 1 - 2 bits> ),
// then the k best per query (ties to the lower id).
//
// Launches:
//  1. qprep   per query: q_rot, q_s, estimator constants folded in, per-query
//             power-of-two prescale, fp16 hi/lo split, written into the
//             tensor-core B operand of its query block (K-major, 128-byte
//             swizzle, rows = query x {hi, lo}).
//  2. score   persistent CTAs over items = (query block, slice of database
//             pages), one CTA per SM.  The block's B operand stays in shared
//             memory for the item.  For each 128-record page, eight warps
//             expand the packed codes into fp16 planes in tensor memory (A,
//             lane = record): the key plane +-b / +-a for magnitude index 0 / 1
//             (a / b the fp16 ratio nearest kc1 / kc0; the query side carries
//             kc0 / b), and the QJL plane +-gamma; meanwhile the previous
//             page's product runs.  A control warp issues one tcgen05.mma chain
//             per page (M = 128 records, N = queries x {hi, lo}, K = 2d) into a
//             TMEM accumulator.  The eight warps read the scores back, and a
//             filter against a per-query bound shared by all lists (the best
//             k-th score any list has reached) feeds rare insertions into
//             per-warp top-k lists in shared memory.
//  3. merge   per query: the best k of all per-warp lists.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <type_traits>

#include "tq_device.cuh"
#include "tq_internal.h"
#include "tq_keyplane.h"
#include "tq_tc.cuh"

namespace tq {
namespace tk {

constexpr int NEPI = 8;                    // epilogue warps: (TMEM lane quarter) x (query half)
constexpr int NTHREADS = (NEPI + 1) * 32;  // + the control warp
constexpr int PAGE = TQ_PAGE_TOKENS;       // records per tile
constexpr int SB_LD = 33;                  // score staging row of 32 queries (padded)
constexpr int SB_BYTES = NEPI * 32 * SB_LD * 4;
constexpr int COL_A0 = 0, COL_A1 = 128, COL_D = 256, TMEM_COLS = 512;
constexpr float NEG_INF = -__builtin_huge_valf();

// float <-> unsigned with the same order (for atomicMax on scores)
__device__ __forceinline__ uint32_t ord_bits(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float unord_bits(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
constexpr uint32_t ORD_NEG_INF = 0x007fffffu;

// D: head dimension (= sketch size m); QB: queries per block (64 or 128)
template <int D, int QB>
struct Cfg {
  static constexpr int NROW = 2 * QB;              // B rows = MMA N: query x {hi, lo}
  static constexpr int WQ = QB / 2;                // queries per epilogue warp
  static constexpr int NPASS = WQ / 32;            // 32-query passes per warp and page
  static constexpr int KTOT = 2 * D;               // key plane, QJL plane
  static constexpr int B_BYTES = NROW * KTOT * 2;  // one block's B operand (SW128 image)
  static constexpr int NMMA = KTOT / 16;
  static_assert(KTOT / 2 <= COL_A1 - COL_A0, "A buffer");
  static_assert(NROW <= TMEM_COLS - COL_D, "accumulator");
  // shared memory, from a 1024-byte aligned base: B | lists | score staging | barriers
  static size_t smem_bytes(int k) {
    return 1024 + static_cast<size_t>(B_BYTES) + static_cast<size_t>(NEPI) * WQ * k * 8 + SB_BYTES + 64;
  }
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
  const float* sp;     // S Pi
  float w_key, alpha;  // query weights of the key plane (kc0 / b) and of the QJL plane
  uint32_t key_b2, key_d7;  // fp16 b and fp16(2^7 (a - b)), both halves
  uint16_t* bimg;      // [n_qb][NROW * KTOT] fp16 bits, SW128 image per block
  float* desc;         // [n_qb * QB] descale
  uint32_t* gslots;    // [n_qb * QB][k] per query: slot e holds the best score (ordered bits)
                       // among the scored records with id = e mod k
  float* cand_s;       // [items][NEPI][WQ][k]
  int* cand_i;
  int n_qb, n_slices;
  long long pages;
  int seed_only;  // a seeding pass: raise the slots only, write no lists
  int* err;
};

// K index k of the A operand (and so of B): plane (0 key, 1 QJL) and the
// coordinate or sketch index.  A record's A row holds, per plane, two halves
// of D/4 TMEM columns; column c of a half covers two K elements (low, high
// 16 bits):
//   key plane: c = 8 wl + 2 i + e -> coordinate 16 (half*D/32 + wl) + 2 i + e (+ 8 high)
//   QJL plane: c = 16 wl + r      -> sketch index 32 (half*D/64 + wl) + r (+ 16 high)
template <int D>
__host__ __device__ __forceinline__ void k_index(int k, int& plane, int& idx) {
  const int col = k >> 1, hiword = k & 1;
  plane = col / (D / 2);
  const int c = col % (D / 2);
  const int half = c / (D / 4), l = c % (D / 4);
  if (plane == 0) {
    const int wl = l >> 3, i = (l & 7) >> 1, e = l & 1;
    idx = 16 * (half * (D / 32) + wl) + 2 * i + e + 8 * hiword;
  } else {
    const int wl = l >> 4, r = l & 15;
    idx = 32 * (half * (D / 64) + wl) + r + 16 * hiword;
  }
}

// y1 = M1 x and y2 = M2 x (D x D, one warp per row group, float4 per lane)
template <int D>
__device__ __forceinline__ void warp_matvec2(const float* __restrict__ M1, const float* __restrict__ M2,
                                             const float* x, float* y1, float* y2) {
  constexpr int LANES = D / 4, RPP = 32 / LANES, NW = 4, PASSES = D / (NW * RPP);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, sub = lane / LANES, l4 = lane % LANES;
  float4 m[2][PASSES];
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const size_t r = static_cast<size_t>((ps * NW + warp) * RPP + sub);
    m[0][ps] = __ldg(reinterpret_cast<const float4*>(M1 + r * D) + l4);
    m[1][ps] = __ldg(reinterpret_cast<const float4*>(M2 + r * D) + l4);
  }
#pragma unroll
  for (int w = 0; w < 2; ++w) {
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
      float a = m[w][ps].x * x[4 * l4] + m[w][ps].y * x[4 * l4 + 1] + m[w][ps].z * x[4 * l4 + 2] +
                m[w][ps].w * x[4 * l4 + 3];
#pragma unroll
      for (int o = LANES / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (l4 == 0) (w == 0 ? y1 : y2)[(ps * NW + warp) * RPP + sub] = a;
    }
  }
}

// one CTA per query slot of the padded blocks; slots past Q write zero rows
template <int D, int QB>
__global__ void __launch_bounds__(128) qprep_kernel(Params p) {
  using C = Cfg<D, QB>;
  const int q = blockIdx.x, qb = q / QB, ql = q % QB;
  __shared__ float sq[D], sr[D], ss[D];
  __shared__ unsigned smax;
  __shared__ float sfac;
  const int tid = threadIdx.x;
  uint8_t* img = reinterpret_cast<uint8_t*>(p.bimg + static_cast<size_t>(qb) * (C::B_BYTES / 2));
  if (q >= p.Q) {
    for (int k0 = tid * 8; k0 < C::KTOT; k0 += blockDim.x * 8)
#pragma unroll
      for (int part = 0; part < 2; ++part)
        *reinterpret_cast<uint4*>(img + tc::sw128_offset(2 * ql + part, k0, C::NROW)) = make_uint4(0, 0, 0, 0);
    if (tid == 0) p.desc[q] = 0.0f;
    for (int e = tid; e < p.k; e += blockDim.x) p.gslots[static_cast<size_t>(q) * p.k + e] = ORD_NEG_INF;
    return;
  }
  if (tid == 0) smax = 0u;
  for (int j = tid; j < D; j += blockDim.x) sq[j] = p.queries[static_cast<size_t>(q) * D + j];
  __syncthreads();
  warp_matvec2<D>(p.rot, p.sp, sq, sr, ss);  // q_rot = Pi q, q_s = (S Pi) q
  __syncthreads();
  const float w1 = p.w_key, w3 = p.alpha;
  for (int j = tid; j < D; j += blockDim.x) {
    const float m = fmaxf(fabsf(w1 * sr[j]), fabsf(w3 * ss[j]));
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
  for (int e = tid; e < p.k; e += blockDim.x) p.gslots[static_cast<size_t>(q) * p.k + e] = ORD_NEG_INF;
  __syncthreads();
  const float f = sfac;
  // 16-byte chunks of 8 K elements, hi and lo rows
  for (int k0 = tid * 8; k0 < C::KTOT; k0 += blockDim.x * 8) {
    uint32_t wh[4] = {0u, 0u, 0u, 0u}, wl[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      int plane, idx;
      k_index<D>(k0 + e, plane, idx);
      const float w = plane == 0 ? w1 * sr[idx] : w3 * ss[idx];
      uint16_t hi, lo;
      split_f16(f * w, hi, lo);
      wh[e >> 1] |= static_cast<uint32_t>(hi) << (16 * (e & 1));
      wl[e >> 1] |= static_cast<uint32_t>(lo) << (16 * (e & 1));
    }
    *reinterpret_cast<uint4*>(img + tc::sw128_offset(2 * ql, k0, C::NROW)) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    *reinterpret_cast<uint4*>(img + tc::sw128_offset(2 * ql + 1, k0, C::NROW)) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
  }
}

__device__ __forceinline__ bool better(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}
// Insert (cs, ci) into the sorted (best first) list of k <= 32 entries, the
// whole warp at once: lane e holds entry e, the rank of the candidate is the
// number of entries ahead of it, the entries behind it move down one lane.
// Returns the list's k-th entry afterwards in (ts, ti) (ti < 0x7fffffff once
// the list is full).
__device__ __forceinline__ void warp_insert(float* ls, int* li, int k, float cs, int ci, float& ts, int& ti) {
  const int lane = threadIdx.x & 31;
  const bool in = lane < k;
  const float es = in ? ls[lane] : NEG_INF;
  const int ei = in ? li[lane] : 0x7fffffff;
  const int pos = __popc(__ballot_sync(0xffffffffu, in && better(es, ei, cs, ci)));
  const float us = __shfl_up_sync(0xffffffffu, es, 1);
  const int ui = __shfl_up_sync(0xffffffffu, ei, 1);
  float ns = es;
  int ni = ei;
  if (lane == pos) {
    ns = cs;
    ni = ci;
  } else if (lane > pos) {
    ns = us;
    ni = ui;
  }
  if (in && pos < k) {
    ls[lane] = ns;
    li[lane] = ni;
  }
  ts = __shfl_sync(0xffffffffu, ns, k - 1);
  ti = __shfl_sync(0xffffffffu, ni, k - 1);
  __syncwarp();
}

// compare-exchange with the lane `mask` away: keep the better (or the worse)
// of the two entries
__device__ __forceinline__ void cmpx(float& s, int& i, int mask, bool keep_better) {
  const float os = __shfl_xor_sync(0xffffffffu, s, mask);
  const int oi = __shfl_xor_sync(0xffffffffu, i, mask);
  if (better(os, oi, s, i) == keep_better) {
    s = os;
    i = oi;
  }
}

// Merge a batch of up to 32 candidates (one per lane; (-inf, 0x7fffffff) for
// none) into the sorted list of k <= 32 entries: bitonic sort of the batch,
// elementwise better of the sorted batch and the reversed list (the best 32
// of both, a bitonic sequence), bitonic merge; the first k are the list.
// Returns the list's k-th entry in (ts, ti).
__device__ __forceinline__ void warp_merge_batch(float* ls, int* li, int k, float s, int i, float& ts, int& ti) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1)
      cmpx(s, i, stride, ((lane & stride) == 0) == ((lane & size) == 0));
  const float es = lane < k ? ls[lane] : NEG_INF;
  const int ei = lane < k ? li[lane] : 0x7fffffff;
  const float rs = __shfl_sync(0xffffffffu, es, 31 - lane);
  const int ri = __shfl_sync(0xffffffffu, ei, 31 - lane);
  if (better(rs, ri, s, i)) {
    s = rs;
    i = ri;
  }
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) cmpx(s, i, stride, (lane & stride) == 0);
  if (lane < k) {
    ls[lane] = s;
    li[lane] = i;
  }
  ts = __shfl_sync(0xffffffffu, s, k - 1);
  ti = __shfl_sync(0xffffffffu, i, k - 1);
  __syncwarp();
}

template <int N>
__device__ __forceinline__ void tmem_store(uint32_t taddr, const uint32_t* r) {
  if constexpr (N == 32) tc::st32(taddr, r);
  else if constexpr (N == 16) tc::st16(taddr, r);
  else tc::st8(taddr, r);
}

// A row of one record (this thread's half of the coordinates), from its
// packed words: the key plane (sign, magnitude index -> +-b, +-a) and the QJL
// plane (+-gamma).  Key code word w holds coordinates 16 w + 8 h + 2 i + e
// with the sign bit at 16 h + 15 - 4 i - e and the magnitude bit two below;
// QJL word w holds sketch index 32 w + 16 h + r at bit 16 h + 15 - r.
template <int D>
__device__ __forceinline__ void build_a_row(const uint32_t* kw, const uint32_t* qw, uint32_t gg,
                                            uint32_t base, int half, uint32_t key_b2, uint32_t key_d7) {
  constexpr int NW = D / 32;  // key words of one half
  uint32_t a[D / 4];
#pragma unroll
  for (int wl = 0; wl < NW; ++wl)
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      a[wl * 8 + s] = key_plane_pair(kw[wl] << ((s >> 1) * 4 + (s & 1)), key_d7, key_b2);
    }
  tmem_store<D / 4>(base + half * (D / 4), a);
#pragma unroll
  for (int wl = 0; wl < D / 64; ++wl)
#pragma unroll
    for (int r = 0; r < 16; ++r) a[wl * 16 + r] = ((qw[wl] << r) & 0x80008000u) | gg;
  tmem_store<D / 4>(base + D / 2 + half * (D / 4), a);
}

// the packed words of one record half, gamma and norm
template <int D>
struct Rec {
  uint32_t kw[D / 32];
  uint32_t qw[D / 64];
  uint32_t gg;
  uint32_t n;
};

template <int D>
__device__ __forceinline__ void load_rec(Rec<D>& r, const uint8_t* pg, const Params& p, int slot, int half) {
  const uint8_t* kp = pg + p.off_kc + slot * (D / 4) + half * (D / 8);
  const uint8_t* qp = pg + p.off_qs + slot * (D / 8) + half * (D / 16);
  if constexpr (D == 128) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(kp));
    r.kw[0] = v.x; r.kw[1] = v.y; r.kw[2] = v.z; r.kw[3] = v.w;
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(qp));
    r.qw[0] = u.x; r.qw[1] = u.y;
  } else {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(kp));
    r.kw[0] = v.x; r.kw[1] = v.y;
    r.qw[0] = __ldg(reinterpret_cast<const uint32_t*>(qp));
  }
  r.gg = static_cast<uint32_t>(__ldg(reinterpret_cast<const uint16_t*>(pg + p.off_kg) + slot)) * 0x10001u;
  r.n = __ldg(reinterpret_cast<const uint16_t*>(pg + p.off_kn) + slot);
}

// the pages of slice sl of n_slices over the database
__device__ __forceinline__ void slice_pages(const Params& p, int item, long long& pg0, long long& pg1) {
  const int sl = item / p.n_qb;
  pg0 = p.pages * sl / p.n_slices;
  pg1 = p.pages * (sl + 1) / p.n_slices;
}

// CTA tile sequence: the pages of its items, item after item
struct TileSeq {
  int item;
  long long page, end;
  __device__ __forceinline__ bool start(const Params& p, int items) {
    item = blockIdx.x;
    if (item >= items) return false;
    slice_pages(p, item, page, end);
    return page < end;
  }
  // advance; false at the end of the sequence
  __device__ __forceinline__ bool next(const Params& p, int items) {
    if (++page < end) return true;
    item += gridDim.x;
    if (item >= items) return false;
    slice_pages(p, item, page, end);
    return page < end;
  }
};


template <int D, int QB>
__global__ void __launch_bounds__(NTHREADS, 1) score_kernel(Params p) {
  using C = Cfg<D, QB>;
  constexpr int WQ = C::WQ;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k = p.k;
  float* ls_all = reinterpret_cast<float*>(smem + C::B_BYTES);
  int* li_all = reinterpret_cast<int*>(smem + C::B_BYTES + NEPI * WQ * k * 4);
  float* sbuf = reinterpret_cast<float*>(smem + C::B_BYTES + NEPI * WQ * k * 8);
  uint8_t* bars = smem + C::B_BYTES + NEPI * WQ * k * 8 + SB_BYTES;
  const uint32_t bar_ab = smem_u32(bars), bar_dfull = bar_ab + 16, bar_dfree = bar_ab + 24;
  const uint32_t bar_bfull = bar_ab + 32, bar_bfree = bar_ab + 40, bar_drain = bar_ab + 48;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 56);
  int& s_failed = *reinterpret_cast<int*>(bars + 60);

  const int items = p.n_qb * p.n_slices;
  if (tid == 0) {
    mbar_init(bar_ab, NEPI);
    mbar_init(bar_ab + 8, NEPI);
    mbar_init(bar_dfull, 1);
    mbar_init(bar_dfree, NEPI);
    mbar_init(bar_bfull, 1);
    mbar_init(bar_bfree, 1);
    mbar_init(bar_drain, 1);
    s_failed = 0;
    mbar_init_fence();
  }
  if (warp == NEPI) {
    tc::tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool failed = false;

  if (warp == NEPI) {
    // ---- control: B operand per item, one MMA chain per page ------------------
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_f16(128, C::NROW, false);
      const uint32_t s_b = smem_u32(smem);
      TileSeq ts;
      bool more = ts.start(p, items);
      uint32_t t = 0, nb = 0;
      bool b_pending = false;
      auto load_b = [&](int item) {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(p.bimg) + static_cast<size_t>(item % p.n_qb) * C::B_BYTES;
        mbar_arrive_expect_tx(bar_bfull, C::B_BYTES);
        for (int off = 0; off < C::B_BYTES; off += 16384)
          bulk_g2s(s_b + off, src + off, C::B_BYTES - off < 16384 ? C::B_BYTES - off : 16384, bar_bfull);
        b_pending = true;
      };
      if (more) load_b(ts.item);
      while (more && !failed) {
        const int item = ts.item;
        if (!mbar_wait_bounded(bar_bfull, nb & 1)) { failed = true; break; }
        b_pending = false;
        do {
          if (!mbar_wait_bounded(bar_ab + 8 * (t & 1), (t >> 1) & 1)) { failed = true; break; }
          if (t > 0 && !mbar_wait_bounded(bar_dfree, (t - 1) & 1)) { failed = true; break; }
          tc::fence_after_sync();
          const uint32_t a = tmem + (t & 1 ? COL_A1 : COL_A0);
#pragma unroll
          for (int s = 0; s < C::NMMA; ++s)
            tc::mma_f16_tmem_a(tmem + COL_D, a + 8 * s,
                               tc::sdesc_sw128(s_b + (s >> 2) * (C::NROW * 128) + (s & 3) * 32), idesc, s > 0);
          tc::commit(bar_dfull);
          ++t;
          more = ts.next(p, items);
        } while (more && ts.item == item);
        if (failed) break;
        // the B operand is rewritten once this item's products are done
        tc::commit(bar_bfree);
        if (!mbar_wait_bounded(bar_bfree, nb & 1)) { failed = true; break; }
        ++nb;
        if (more) load_b(ts.item);
      }
      if (failed) {
        // no copy or product may still be in flight when the CTA exits
        if (b_pending) mbar_wait_bounded(bar_bfull, nb & 1);
        tc::commit(bar_drain);
        mbar_wait_bounded(bar_drain, 0);
        s_failed = 1;
      }
    }
    __syncwarp();
  } else {
    // ---- eight warps: A planes, scores, lists --------------------------------
    const int qr = warp & 3, half = warp >> 2;
    const int row = 32 * qr + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(32 * qr) << 16);
    float* ls = ls_all + warp * WQ * k;
    int* li = li_all + warp * WQ * k;
    float* sb = sbuf + warp * 32 * SB_LD;
    // per 32-query pass: valid-query mask, and in lane j a lower bound on
    // query j's k-th best score (ordered bits), below which a record cannot
    // be among the k best: the k-th entry of this warp's list, or the least
    // of the query's k slots (k distinct records' scores).  The slots are
    // read one per page, one page ahead (sf, slot se); their running minimum
    // (cmin) becomes a bound when a round of k slots is complete (slots only
    // grow, so values read at different times still bound the k-th score).
    uint32_t qmask[C::NPASS], bl[C::NPASS], cmin[C::NPASS], sf[C::NPASS];
    int list_item = -1, q0h = 0, se = 0;
    auto flush = [&](int item) {
      if (p.seed_only) return;
      const size_t base = (static_cast<size_t>(item) * NEPI + warp) * WQ * k;
      const float* dq = p.desc + (item % p.n_qb) * QB + WQ * half;
      // lists hold scores before the per-query power-of-two descale (the
      // order is the same); the descale is applied here
      for (int i = lane; i < WQ * k; i += 32) {
        p.cand_s[base + i] = ls[i] * __ldg(dq + i / k);
        p.cand_i[base + i] = li[i];
      }
    };
    auto reset = [&](int item) {
      __syncwarp();
      for (int i = lane; i < WQ * k; i += 32) {
        ls[i] = NEG_INF;
        li[i] = 0x7fffffff;
      }
      q0h = (item % p.n_qb) * QB + WQ * half;
#pragma unroll
      for (int ps = 0; ps < C::NPASS; ++ps) {
        qmask[ps] = __ballot_sync(0xffffffffu, q0h + 32 * ps + lane < p.Q);
        const uint32_t* sl = p.gslots + static_cast<size_t>(q0h + 32 * ps + lane) * k;
        uint32_t mn = 0xffffffffu;
#pragma unroll 4
        for (int e = 0; e < k; ++e) mn = min(mn, __ldcg(sl + e));
        bl[ps] = mn;
        cmin[ps] = 0xffffffffu;
        sf[ps] = __ldcg(sl);
      }
      se = 0;
      __syncwarp();
    };
    // the tile sequence runs one page ahead: tile t+1 is expanded while the
    // product of tile t runs, and tile t+2's words are in flight meanwhile
    TileSeq ts;
    bool have = ts.start(p, items);
    Rec<D> r;
    if (have) load_rec<D>(r, p.db + ts.page * p.page_bytes, p, row, half);
    bool cur = false;
    uint32_t n_cur = 0u;
    long long page_cur = 0;
    int item_cur = 0;
    uint32_t t = 0;
    auto build_next = [&](uint32_t buf) {
      build_a_row<D>(r.kw, r.qw, r.gg, t_lane + (buf ? COL_A1 : COL_A0), half, p.key_b2, p.key_d7);
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_ab + 8 * buf);
    };
    if (have) {
      build_next(0u);
      cur = true;
      n_cur = r.n;
      page_cur = ts.page;
      item_cur = ts.item;
      have = ts.next(p, items);
      if (have) load_rec<D>(r, p.db + ts.page * p.page_bytes, p, row, half);
    }
    while (cur) {
      const bool nxt = have;
      uint32_t n_nxt = 0u;
      long long page_nxt = 0;
      int item_nxt = 0;
      if (nxt) {
        build_next((t + 1) & 1u);
        n_nxt = r.n;
        page_nxt = ts.page;
        item_nxt = ts.item;
        have = ts.next(p, items);
        if (have) load_rec<D>(r, p.db + ts.page * p.page_bytes, p, row, half);
      }
      const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar_dfull, t & 1u));
      if (!ok) {
        failed = true;
        break;
      }
      tc::fence_after_sync();
      if (item_cur != list_item) {
        if (list_item >= 0) flush(list_item);
        reset(item_cur);
        list_item = item_cur;
      }
      const long long id64 = page_cur * PAGE + row;
      const bool valid = id64 < p.N;
      const int id0 = static_cast<int>(page_cur * PAGE + 32 * qr);
      const float nf = __half2float(__ushort_as_half(static_cast<unsigned short>(n_cur)));
      // scores of this warp's queries (32 per pass) x {hi, lo}; the
      // accumulator is released as soon as it is read
      float sc[C::NPASS][32];
#pragma unroll
      for (int ps = 0; ps < C::NPASS; ++ps) {
        uint32_t v0[32], v1[32];
        const uint32_t col = COL_D + 2 * WQ * half + 64 * ps;
        tc::ld32(t_lane + col, v0);
        tc::ld32(t_lane + col + 32, v1);
        tc::wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const uint32_t* v = j < 16 ? v0 : v1;
          const int c = 2 * (j % 16);
          sc[ps][j] = (__uint_as_float(v[c]) + __uint_as_float(v[c + 1])) * nf;
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dfree);
#pragma unroll
      for (int ps = 0; ps < C::NPASS; ++ps) {
        // slot se of this lane's query, read one page ago
        cmin[ps] = min(cmin[ps], sf[ps]);
        if (se == k - 1) {
          bl[ps] = max(bl[ps], cmin[ps]);
          cmin[ps] = 0xffffffffu;
        }
        sf[ps] = __ldcg(p.gslots + static_cast<size_t>(q0h + 32 * ps + lane) * k + (se == k - 1 ? 0 : se + 1));
        const float blf = unord_bits(bl[ps]);
        uint32_t cm = 0u;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (sc[ps][j] >= __shfl_sync(0xffffffffu, blf, j)) cm |= 1u << j;
        cm = valid ? (cm & qmask[ps]) : 0u;
        const uint32_t anyq = __reduce_or_sync(0xffffffffu, cm);
        if (anyq) {
          // rare: the scores go through shared memory so that the insertions
          // run as a rolled loop over (query, record) candidates
#pragma unroll
          for (int j = 0; j < 32; ++j) sb[lane * SB_LD + j] = sc[ps][j];
          __syncwarp();
          uint32_t rem = anyq;
          while (rem) {
            const int j = __ffs(rem) - 1;
            rem &= rem - 1;
            const int jq = 32 * ps + j;
            const bool mine = (cm >> j) & 1u;
            unsigned m = __ballot_sync(0xffffffffu, mine);
            // every candidate raises its slot
            if (mine)
              atomicMax(p.gslots + static_cast<size_t>(q0h + jq) * k + (id0 + lane) % k,
                        ord_bits(sb[lane * SB_LD + j]));
            float ts2 = NEG_INF;
            int ti = 0x7fffffff;
            if (__popc(m) >= 6) {
              warp_merge_batch(ls + jq * k, li + jq * k, k, mine ? sb[lane * SB_LD + j] : NEG_INF,
                               mine ? id0 + lane : 0x7fffffff, ts2, ti);
            } else {
              while (m) {
                const int src = __ffs(m) - 1;
                m &= m - 1;
                warp_insert(ls + jq * k, li + jq * k, k, sb[src * SB_LD + j], id0 + src, ts2, ti);
              }
            }
            if (ti != 0x7fffffff) {
              const uint32_t ob = ord_bits(ts2);
              if (lane == j) bl[ps] = max(bl[ps], ob);
            }
          }
          __syncwarp();
        }
      }
      se = se == k - 1 ? 0 : se + 1;
      ++t;
      cur = nxt;
      n_cur = n_nxt;
      page_cur = page_nxt;
      item_cur = item_nxt;
    }
    if (!failed && list_item >= 0) {
      __syncwarp();
      flush(list_item);
    }
    if (failed && lane == 0) s_failed = 1;
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == NEPI) tc::tmem_dealloc(tmem, TMEM_COLS);
  if (tid == 0 && s_failed) report(p.err, TQ_ERR_TIMEOUT);
}

// per query: the best k among n_slices x 4 lists of k candidates (the four
// warps of its query half, in every slice)
template <int QB>
__global__ void __launch_bounds__(128) merge_kernel(Params p, int32_t* out_ids, float* out_scores) {
  constexpr int WQ = QB / 2;
  const int q = blockIdx.x;
  const int qb = q / QB, ql = q % QB, half = ql / WQ, j = ql % WQ;
  const int lists = p.n_slices * 4;
  extern __shared__ uint8_t sm[];
  float* cs = reinterpret_cast<float*>(sm);
  int* ci = reinterpret_cast<int*>(sm + sizeof(float) * lists * p.k);
  __shared__ float rs[4];
  __shared__ int ri[4], rp[4];
  const int total = lists * p.k;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int l = i / p.k, e = i % p.k;
    const int sl = l >> 2, w = 4 * half + (l & 3);
    const int item = sl * p.n_qb + qb;
    const size_t src = ((static_cast<size_t>(item) * NEPI + w) * WQ + j) * p.k + e;
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

// queries per block: 128 (MMA N = 256) while the per-warp lists of 64
// queries fit in shared memory beside the 2 x 128-row B operand, else 64
inline int qb_for(int k) { return k <= 16 ? 128 : 64; }

struct Ws {
  size_t bimg, desc, gb, cs, ci, total;
};

// slices of the database per query block: at least four items per SM, and
// among the counts up to four times that, the one that loads the SMs most
// evenly (items a multiple of the SM count where one exists); never more
// slices than pages, so that every item has a page
inline int n_slices_for(const tq_ctx* ctx, int Q, int qb, long long pages) {
  const long long n_qb = (Q + qb - 1) / qb, sms = ctx->num_sms > 0 ? ctx->num_sms : 1;
  long long lo = (4 * sms + n_qb - 1) / n_qb;
  if (lo < 1) lo = 1;
  long long best = lo;
  double best_eff = 0.0;
  for (long long ns = lo; ns <= 4 * lo; ++ns) {
    const long long items = n_qb * ns, waves = (items + sms - 1) / sms;
    const double eff = static_cast<double>(items) / static_cast<double>(waves * sms);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = ns;
    }
  }
  if (best > pages) best = pages;
  return static_cast<int>(best < 1 ? 1 : best);
}

Ws ws_layout(const tq_ctx* ctx, int Q, long long N, int k) {
  const int d = ctx->cfg.head_dim, qb = qb_for(k);
  const long long pages = (N + TQ_PAGE_TOKENS - 1) / TQ_PAGE_TOKENS;
  const int n_qb = (Q + qb - 1) / qb;
  const int ns = n_slices_for(ctx, Q, qb, pages);
  const size_t items = static_cast<size_t>(n_qb) * ns;
  Ws w;
  size_t off = 0;
  w.bimg = off;
  off = align256(off + sizeof(uint16_t) * static_cast<size_t>(n_qb) * (2 * qb) * (2 * d));
  w.desc = off;
  off = align256(off + sizeof(float) * static_cast<size_t>(n_qb) * qb);
  w.gb = off;
  off = align256(off + sizeof(uint32_t) * static_cast<size_t>(n_qb) * qb * k);
  w.cs = off;
  off = align256(off + sizeof(float) * items * NEPI * (qb / 2) * k);
  w.ci = off;
  off = align256(off + sizeof(int) * items * NEPI * (qb / 2) * k);
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
  if (ctx->cfg.qjl_dim != d) return TQ_ERR_UNSUPPORTED;
  const tk::Ws L = tk::ws_layout(ctx, Q, N, k);
  if (ws_bytes < L.total) return TQ_ERR_INVALID_ARG;
  const PageLayout pl = page_layout(d, ctx->cfg.qjl_dim, false);
  const int qb = tk::qb_for(k);
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
  p.sp = ctx->dev.sp;
  // the key plane's centroid ratio is carried to better than 2^-19
  KeyPlane kp;
  if (!key_plane(ctx->cb.key_c[0], ctx->cb.key_c[1], kp)) return TQ_ERR_UNSUPPORTED;
  p.w_key = static_cast<float>(ctx->cb.key_c[0] / kp.b);
  p.key_b2 = kp.b2;
  p.key_d7 = kp.d7;
  p.alpha = 1.2533141373155001f / static_cast<float>(ctx->cfg.qjl_dim);
  uint8_t* base = static_cast<uint8_t*>(ws);
  p.bimg = reinterpret_cast<uint16_t*>(base + L.bimg);
  p.desc = reinterpret_cast<float*>(base + L.desc);
  p.gslots = reinterpret_cast<uint32_t*>(base + L.gb);
  p.cand_s = reinterpret_cast<float*>(base + L.cs);
  p.cand_i = reinterpret_cast<int*>(base + L.ci);
  p.pages = (N + TQ_PAGE_TOKENS - 1) / TQ_PAGE_TOKENS;
  p.n_qb = (Q + qb - 1) / qb;
  p.n_slices = tk::n_slices_for(ctx, Q, qb, p.pages);
  p.err = ctx->dev.err;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int items = p.n_qb * p.n_slices;
  const int grid = items < ctx->num_sms ? items : ctx->num_sms;
  const size_t merge_smem = static_cast<size_t>(p.n_slices) * 4 * k * 8;
  if (merge_smem > 200 * 1024) return TQ_ERR_UNSUPPORTED;
  auto go = [&](auto dtag, auto qtag) -> int {
    constexpr int D = decltype(dtag)::value, QB = decltype(qtag)::value;
    using C = tk::Cfg<D, QB>;
    // at least 116 KB, so that one CTA (and one 512-column TMEM allocation)
    // sits on an SM
    size_t smem = C::smem_bytes(k);
    if (smem < 116 * 1024) smem = 116 * 1024;
    if (smem > 232448) return TQ_ERR_UNSUPPORTED;
    static SmemAttr score_attr;  // one per kernel instantiation; grows with k
    if (!raise_smem_limit(tk::score_kernel<D, QB>, static_cast<int>(smem), score_attr))
      return TQ_ERR_CUDA;
    tk::qprep_kernel<D, QB><<<p.n_qb * QB, 128, 0, st>>>(p);
    if (ctx->prof_start) cudaEventRecord(static_cast<cudaEvent_t>(ctx->prof_start), st);
    // seeding pass over the first pages: every query's slots start from the
    // k best of a sample instead of from nothing, which spares the main
    // pass most of its early list insertions
    const long long seed_pages = p.n_slices > 64 ? p.n_slices : 64;
    if (p.pages >= 8 * seed_pages) {
      tk::Params ps = p;
      ps.pages = seed_pages;
      ps.seed_only = 1;
      tk::score_kernel<D, QB><<<grid, tk::NTHREADS, smem, st>>>(ps);
    }
    tk::score_kernel<D, QB><<<grid, tk::NTHREADS, smem, st>>>(p);
    if (ctx->prof_stop) cudaEventRecord(static_cast<cudaEvent_t>(ctx->prof_stop), st);
    static SmemAttr merge_attr;
    if (merge_smem > 48 * 1024 &&
        !raise_smem_limit(tk::merge_kernel<QB>, static_cast<int>(merge_smem), merge_attr))
      return TQ_ERR_CUDA;
    tk::merge_kernel<QB><<<Q, 128, merge_smem, st>>>(p, out_ids, out_scores);
    return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
  };
  using I64 = std::integral_constant<int, 64>;
  using I128 = std::integral_constant<int, 128>;
  if (d == 128) return qb == 128 ? go(I128{}, I128{}) : go(I128{}, I64{});
  if (d == 64) return qb == 128 ? go(I64{}, I128{}) : go(I64{}, I64{});
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq
