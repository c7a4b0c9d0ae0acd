// Compress and append on the 5th-generation tensor cores (tcgen05), for raw
// fp16 / bf16 inputs ("TurboQuant" summary, de.news.hada.io topic 27867,
// section "Funktionsweise von TurboQuant": random rotation, per-coordinate
// quantiser, 1-bit QJL sketch of the residual).
//
// Persistent CTAs of 256 threads, one 128-token page tile at a time:
//   TMA     input tile [128 rows x d] (3-D tensor map over [B*Hkv, n_new, d],
//           128-byte swizzle; rows outside the sequence arrive as zeros),
//           double-buffered (keys, values)
//   MMA     one thread issues tcgen05.mma: x_rot = X (Pi_hi + Pi_lo)^T into
//           TMEM (M = 128, N = d, K = d, f32 accumulate); later p = R S^T
//   epilogue all 8 warps: thread = (row, half of the columns); x_rot from TMEM
//           by tcgen05.ld; norm, codes, residual, sign bits and packing stay
//           in the thread; the residual is written to shared memory in the
//           MMA's operand layout for the sketch; records go straight to the page.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "tq_device.cuh"
#include "tq_internal.h"
#include "tq_tc.cuh"

namespace tq {
namespace tc {

bool encode_map_3d(CUtensorMap* map, bool bf16, const void* base, const uint64_t dims[3],
                   const uint64_t strides_bytes[2], const uint32_t box[3]) {
  using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
      return false;
    fn = reinterpret_cast<EncodeFn>(p);
  }
  const cuuint64_t gdim[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t gstr[2] = {strides_bytes[0], strides_bytes[1]};
  const cuuint32_t bdim[3] = {box[0], box[1], box[2]};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
            const_cast<void*>(base), gdim, gstr, bdim, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

namespace ctc {

constexpr int ROWS = 128;
constexpr int NTHREADS = 256;

template <int D>
struct Cfg {
  static constexpr int HALF = D / 2;          // columns per epilogue thread
  static constexpr int OPB = D * 128;         // bytes of one 64-column block of a D-row operand
  static constexpr int OP = (D / 64) * OPB;   // D x D operand (Pi hi, Pi lo, S)
  static constexpr int XB = ROWS * 128;       // one 64-column block of a 128-row tile
  static constexpr int XT = (D / 64) * XB;    // 128-row tile
  static constexpr int OFF_PH = 0;
  static constexpr int OFF_PL = OFF_PH + OP;
  static constexpr int OFF_S = OFF_PL + OP;
  static constexpr int OFF_X0 = OFF_S + OP;
  static constexpr int OFF_X1 = OFF_X0 + XT;
  static constexpr int OFF_R = OFF_X1 + XT;
  static constexpr int OFF_NK = OFF_R + XT;        // float[2][128] key norm^2 halves
  static constexpr int OFF_NV = OFF_NK + 1024;     // float[2][128] value norm^2 halves
  static constexpr int OFF_G = OFF_NV + 1024;      // float[2][128] residual norm^2 halves
  static constexpr int OFF_VS = OFF_G + 1024;      // value-code section staging (64 D bytes)
  static constexpr int OFF_KM = OFF_VS + D * 64;   // u32 [3][128][D/32] plane masks H, L, QJL
  static constexpr int OFF_N16 = OFF_KM + 3 * ROWS * D / 8;  // fp16 bits [3][128]: n, gamma, n_v
  static constexpr int OFF_BAR = OFF_N16 + 3 * ROWS * 2;     // 5 mbarriers
  static constexpr int OFF_TMEM = OFF_BAR + 64;
  static constexpr int SMEM = OFF_TMEM + 16 + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = (3 * D <= 256) ? 256 : 512;
  static constexpr int COL_RK = 0, COL_SK = D, COL_RV = 2 * D;
};

struct Params {
  int B, Hkv, n_new;
  bool has_v;
  uint8_t* pool;
  long long pool_pages, page_bytes;
  int off_kc, off_qs, off_vc, off_kn, off_kg, off_vn;
  int off_kl, blk;  // pages with values: key plane L, block bytes (block layout)
  const int32_t* page_table;
  int max_pages;
  const int32_t* cold_len;
  const uint16_t* pi_hi;
  const uint16_t* pi_lo;
  const uint16_t* s_h;
  float kc0, kc1, kt0;
  float vt[7];
  int* err;
  int tiles_per_bh;
  const int32_t* n_new_b;  // [B] tokens appended per sequence (eviction), or null: n_new for all
};

struct Tile {
  int bh, lpage, s_lo, s_hi, page, row0;
};

// the next tile of this CTA with active slots, starting at index t (uniform)
__device__ __forceinline__ bool next_tile(const Params& p, int& t, Tile& out) {
  const int total = p.B * p.Hkv * p.tiles_per_bh;
  for (; t < total; t += gridDim.x) {
    const int bh = t / p.tiles_per_bh, ti = t % p.tiles_per_bh;
    const int cl = p.cold_len[bh / p.Hkv];
    const int nn = p.n_new_b ? min(p.n_new_b[bh / p.Hkv], p.n_new) : p.n_new;
    const int lpage = cl / ROWS + ti;
    const int s_lo = max(cl, lpage * ROWS) - lpage * ROWS;
    const int s_hi = min(cl + nn, (lpage + 1) * ROWS) - lpage * ROWS;
    if (s_lo >= s_hi) continue;
    out.bh = bh;
    out.lpage = lpage;
    out.s_lo = s_lo;
    out.s_hi = s_hi;
    out.row0 = lpage * ROWS - cl;
    out.page = (lpage < p.max_pages) ? p.page_table[static_cast<size_t>(bh) * p.max_pages + lpage] : -1;
    return true;
  }
  return false;
}

template <int D>
__device__ __forceinline__ void issue_tile_load(const CUtensorMap* map, uint32_t dst, uint32_t bar,
                                                const Tile& tl) {
  using C = Cfg<D>;
  mbar_arrive_expect_tx(bar, C::XT);
#pragma unroll
  for (int kb = 0; kb < D / 64; ++kb) tc::tma_load_3d(dst + kb * C::XB, map, kb * 64, tl.row0, tl.bh, bar);
}

// x_rot = X (Pi_hi + Pi_lo)^T into TMEM columns [col, col + D)
template <int D, bool BF>
__device__ __forceinline__ void issue_rotation(uint32_t tmem, int col, uint32_t x, uint32_t ph,
                                               uint32_t pl) {
  using C = Cfg<D>;
  constexpr uint32_t idesc = tc::idesc_f16(ROWS, D, BF);
#pragma unroll
  for (int s = 0; s < D / 16; ++s) {
    const int kb = s >> 2, w = (s & 3) * 32;
    const uint64_t a = tc::sdesc_sw128(x + kb * C::XB + w);
    tc::mma_f16(tmem + col, a, tc::sdesc_sw128(ph + kb * C::OPB + w), idesc, s > 0);
    tc::mma_f16(tmem + col, a, tc::sdesc_sw128(pl + kb * C::OPB + w), idesc, true);
  }
}

// sum of squares of this thread's half row of a 16-bit input tile
template <int D, bool BF>
__device__ __forceinline__ float half_row_sumsq(const uint8_t* x, int row, int h) {
  using C = Cfg<D>;
  float ss = 0.0f;
#pragma unroll
  for (int c = 0; c < C::HALF / 8; ++c) {
    const int k = h * C::HALF + 8 * c;
    const uint4 v = *reinterpret_cast<const uint4*>(x + tc::sw128_offset(row, k, ROWS));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a, b;
      if constexpr (BF) {
        a = __uint_as_float(w[i] << 16);
        b = __uint_as_float(w[i] & 0xFFFF0000u);
      } else {
        const __half2 hh = *reinterpret_cast<const __half2*>(&w[i]);
        a = __low2float(hh);
        b = __high2float(hh);
      }
      ss = fmaf(a, a, fmaf(b, b, ss));
    }
  }
  return ss;
}

template <int D>
__device__ __forceinline__ void tmem_load_half(uint32_t taddr, float (&x)[D / 2]) {
#pragma unroll
  for (int c = 0; c < D / 2; c += 32) {
    uint32_t r[32];
    tc::ld32(taddr + c, r);
    tc::wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) x[c + i] = __uint_as_float(r[i]);
  }
}

template <int D, bool BF>
__global__ void __launch_bounds__(NTHREADS, 1)
    compress_tc_kernel(const __grid_constant__ CUtensorMap mapK,
                       const __grid_constant__ CUtensorMap mapV, Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled operand atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = 32 * (warp & 3) + lane;  // TMEM lane quarter of this warp
  const int h = warp >> 2;                 // column half
  const uint32_t s0 = smem_u32(smem);
  const uint32_t bar_full0 = s0 + C::OFF_BAR, bar_full1 = bar_full0 + 8;
  const uint32_t bar_rk = bar_full0 + 16, bar_sk = bar_full0 + 24, bar_rv = bar_full0 + 32;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  float* nk = reinterpret_cast<float*>(smem + C::OFF_NK);
  float* nvp = reinterpret_cast<float*>(smem + C::OFF_NV);
  float* gp = reinterpret_cast<float*>(smem + C::OFF_G);

  {
    // a CTA without a tile leaves before staging the operand tables (calls
    // that append to few sequences, such as evictions, launch many idle CTAs)
    int t0 = blockIdx.x;
    Tile probe;
    if (!next_tile(p, t0, probe)) return;
  }
  // resident operands in the K-major SW128 layout: Pi hi, Pi lo (rows = output
  // coordinate), S (rows = sketch index); 16-byte chunks
  for (int i = tid; i < D * (D / 8); i += NTHREADS) {
    const int r = i / (D / 8), k = (i % (D / 8)) * 8;
    const uint32_t off = tc::sw128_offset(r, k, D);
    *reinterpret_cast<uint4*>(smem + C::OFF_PH + off) =
        *reinterpret_cast<const uint4*>(p.pi_hi + static_cast<size_t>(r) * D + k);
    *reinterpret_cast<uint4*>(smem + C::OFF_PL + off) =
        *reinterpret_cast<const uint4*>(p.pi_lo + static_cast<size_t>(r) * D + k);
    *reinterpret_cast<uint4*>(smem + C::OFF_S + off) =
        *reinterpret_cast<const uint4*>(p.s_h + static_cast<size_t>(r) * D + k);
  }
  if (tid == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(bar_full0 + 8 * i, 1);
    mbar_init_fence();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  fence_proxy_async_smem();  // operand tables visible to the tensor cores
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_lane = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);

  int t = blockIdx.x;
  Tile cur;
  bool have = next_tile(p, t, cur);
  if (have && tid == 0) {
    issue_tile_load<D>(&mapK, s0 + C::OFF_X0, bar_full0, cur);
    if (p.has_v) issue_tile_load<D>(&mapV, s0 + C::OFF_X1, bar_full1, cur);
  }
  bool failed = false;
  for (uint32_t it = 0; have; ++it) {
    const uint32_t par = it & 1u;
    int tn = t + gridDim.x;
    Tile nxt;
    const bool have_next = next_tile(p, tn, nxt);
    const bool page_ok = cur.page >= 0 && cur.page < p.pool_pages;

    // ---- keys: rotation ------------------------------------------------
    if (!mbar_wait_bounded(bar_full0, par)) { failed = true; break; }
    if (tid == 0) {
      tc::fence_after_sync();
      issue_rotation<D, BF>(tmem, C::COL_RK, s0 + C::OFF_X0, s0 + C::OFF_PH, s0 + C::OFF_PL);
      tc::commit(bar_rk);
    }
    nk[h * ROWS + row] = half_row_sumsq<D, BF>(smem + C::OFF_X0, row, h);
    __syncthreads();
    if (!mbar_wait_bounded(bar_rk, par)) { failed = true; break; }
    tc::fence_after_sync();
    if (tid == 0 && have_next) {
      fence_proxy_async_smem();
      issue_tile_load<D>(&mapK, s0 + C::OFF_X0, bar_full0, nxt);
    }
    float x[C::HALF];
    tmem_load_half<D>(t_lane + C::COL_RK + h * C::HALF, x);
    const float nn = sqrtf(nk[row] + nk[ROWS + row]);
    const __half nh = __float2half_rn(nn);
    const float n = __half2float(nh);
    const float T0 = __fmul_rn(n, p.kt0);
    const float inv = n > 0.0f ? 1.0f / n : 0.0f;
    // plane masks of this half row (block layout): H = 1 - sign, L = sign XOR
    // magnitude; bit i % 32 of word i / 32 for column i of the half
    uint32_t hm[C::HALF / 32], lm[C::HALF / 32];
#pragma unroll
    for (int w = 0; w < C::HALF / 32; ++w) hm[w] = lm[w] = 0u;
    float g2 = 0.0f;
#pragma unroll
    for (int c8 = 0; c8 < C::HALF / 8; ++c8) {
      uint32_t rh[4];
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        float rr[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          // computed as for n > 0; a zero vector's row is cleared below
          const int i = 8 * c8 + 2 * e2 + e;  // column within the half
          const float v = x[i];
          const bool neg = v < 0.0f, big = fabsf(v) >= T0;
          const float cp = big ? p.kc1 : p.kc0;
          const float r = fmaf(v, inv, neg ? cp : -cp);
          rr[e] = r;
          g2 = fmaf(r, r, g2);
          if (!neg) hm[i >> 5] |= 1u << (i & 31);
          if (neg != big) lm[i >> 5] |= 1u << (i & 31);
        }
        const __half2 pr = __floats2half2_rn(n > 0.0f ? rr[0] : 0.0f, n > 0.0f ? rr[1] : 0.0f);
        rh[e2] = *reinterpret_cast<const uint32_t*>(&pr);
      }
      *reinterpret_cast<uint4*>(smem + C::OFF_R + tc::sw128_offset(row, h * C::HALF + 8 * c8, ROWS)) =
          make_uint4(rh[0], rh[1], rh[2], rh[3]);
    }
    if (!(n > 0.0f)) {  // zero vector: sign and magnitude 0 (H 1, L 0), residual norm 0
#pragma unroll
      for (int w = 0; w < C::HALF / 32; ++w) {
        hm[w] = 0xFFFFFFFFu;
        lm[w] = 0u;
      }
      g2 = 0.0f;
    }
    gp[h * ROWS + row] = g2;
    uint32_t* km = reinterpret_cast<uint32_t*>(smem + C::OFF_KM);
    uint16_t* n16 = reinterpret_cast<uint16_t*>(smem + C::OFF_N16);
#pragma unroll
    for (int w = 0; w < C::HALF / 32; ++w) {
      km[row * (D / 32) + h * (C::HALF / 32) + w] = hm[w];
      km[(ROWS + row) * (D / 32) + h * (C::HALF / 32) + w] = lm[w];
    }
    fence_proxy_async_smem();  // residual tile visible to the tensor cores
    tc::fence_before_sync();
    __syncthreads();
    // ---- keys: QJL sketch, values: rotation --------------------------------
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t idesc = tc::idesc_f16(ROWS, D, false);
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const int kb = s >> 2, w = (s & 3) * 32;
        tc::mma_f16(tmem + C::COL_SK, tc::sdesc_sw128(s0 + C::OFF_R + kb * C::XB + w),
                    tc::sdesc_sw128(s0 + C::OFF_S + kb * C::OPB + w), idesc, s > 0);
      }
      tc::commit(bar_sk);
    }
    if (p.has_v) {
      if (!mbar_wait_bounded(bar_full1, par)) { failed = true; break; }
      if (tid == 0) {
        tc::fence_after_sync();
        issue_rotation<D, BF>(tmem, C::COL_RV, s0 + C::OFF_X1, s0 + C::OFF_PH, s0 + C::OFF_PL);
        tc::commit(bar_rv);
      }
      nvp[h * ROWS + row] = half_row_sumsq<D, BF>(smem + C::OFF_X1, row, h);
    }
    uint8_t* pg = p.pool + static_cast<size_t>(page_ok ? cur.page : 0) * p.page_bytes;
    if (!mbar_wait_bounded(bar_sk, par)) { failed = true; break; }
    tc::fence_after_sync();
    tmem_load_half<D>(t_lane + C::COL_SK + h * C::HALF, x);
    {
      uint32_t qm[C::HALF / 32];  // QJL plane mask: bit i % 32 of word i / 32
#pragma unroll
      for (int w = 0; w < C::HALF / 32; ++w) qm[w] = 0u;
#pragma unroll
      for (int i = 0; i < C::HALF; ++i)
        if (x[i] < 0.0f) qm[i >> 5] |= 1u << (i & 31);
#pragma unroll
      for (int w = 0; w < C::HALF / 32; ++w)
        km[(2 * ROWS + row) * (D / 32) + h * (C::HALF / 32) + w] = (n > 0.0f) ? qm[w] : 0u;
    }
    __syncthreads();  // residual norm halves and value norm halves complete
    if (h == 0) {
      n16[row] = __half_as_ushort(nh);
      n16[ROWS + row] = __half_as_ushort(__float2half_rn(sqrtf(gp[row] + gp[ROWS + row])));
    }
    // ---- values ------------------------------------------------------------
    if (p.has_v) {
      if (!mbar_wait_bounded(bar_rv, par)) { failed = true; break; }
      tc::fence_after_sync();
      if (tid == 0 && have_next) {
        fence_proxy_async_smem();
        issue_tile_load<D>(&mapV, s0 + C::OFF_X1, bar_full1, nxt);
      }
      tmem_load_half<D>(t_lane + C::COL_RV + h * C::HALF, x);
      const __half vh = __float2half_rn(sqrtf(nvp[row] + nvp[ROWS + row]));
      const float vn = __half2float(vh);
      float T[7];
#pragma unroll
      for (int k = 0; k < 7; ++k) T[k] = __fmul_rn(vn, p.vt[k]);
      // codes of this row, then the pair partner's (adjacent lane) for the bytes
      uint32_t cw[C::HALF / 8];  // 8 nibbles per word, column i in nibble i % 8
#pragma unroll
      for (int w = 0; w < C::HALF / 8; ++w) cw[w] = 0u;
#pragma unroll
      for (int i = 0; i < C::HALF; ++i) {
        uint32_t mg = 0u;
#pragma unroll
        for (int k = 0; k < 7; ++k) mg += (fabsf(x[i]) >= T[k]) ? 1u : 0u;
        const uint32_t code = ((x[i] < 0.0f) ? 8u : 0u) | mg;
        cw[i >> 3] |= code << (4 * (i & 7));
      }
      if (!(vn > 0.0f)) {  // zero vector
#pragma unroll
        for (int w = 0; w < C::HALF / 8; ++w) cw[w] = 0u;
      }
      const bool even = (row & 1) == 0;
      uint32_t ow[C::HALF / 8];
#pragma unroll
      for (int w = 0; w < C::HALF / 8; ++w) ow[w] = __shfl_xor_sync(0xffffffffu, cw[w], 1);
      // even rows place the byte pairs (own code low, partner's high) in the
      // staged section; the whole section then goes out with 16-byte copies
      uint8_t* vs = smem + C::OFF_VS;
      if (even) {
        const int pr = row >> 1;
#pragma unroll
        for (int i = 0; i < C::HALF; ++i) {
          const uint32_t lo = (cw[i >> 3] >> (4 * (i & 7))) & 0xFu;
          const uint32_t hi = (ow[i >> 3] >> (4 * (i & 7))) & 0xFu;
          vs[vc_pos<D>(h * C::HALF + i, pr)] = static_cast<uint8_t>(lo | (hi << 4));
        }
      }
      if (h == 0) reinterpret_cast<uint16_t*>(smem + C::OFF_N16)[2 * ROWS + row] = __half_as_ushort(vh);
    }
    __syncthreads();  // staged planes, norms and value codes complete
    if (page_ok) {
      const uint32_t* kmc = reinterpret_cast<const uint32_t*>(smem + C::OFF_KM);
      const uint16_t* n16c = reinterpret_cast<const uint16_t*>(smem + C::OFF_N16);
      key_planes_out<D>(kmc, kmc + ROWS * (D / 32), kmc + 2 * ROWS * (D / 32), pg, p.blk, p.off_kc,
                        p.off_kl, p.off_qs, cur.s_lo, cur.s_hi, tid, NTHREADS);
      norms_out(n16c, n16c + ROWS, p.has_v ? n16c + 2 * ROWS : nullptr, pg, p.blk, p.off_kn,
                p.off_vn, cur.s_lo, cur.s_hi, tid, NTHREADS);
      if (p.has_v) vc_copy_out<D>(smem + C::OFF_VS, pg, p.blk, p.off_vc, cur.s_lo, cur.s_hi, tid, NTHREADS);
    }
    if (threadIdx.x == 0 && !page_ok) report(p.err, TQ_ERR_CAPACITY);
    tc::fence_before_sync();
    __syncthreads();  // TMEM columns and the residual tile are reused by the next tile
    tc::fence_after_sync();
    cur = nxt;
    t = tn;
    have = have_next;
  }
  if (failed && threadIdx.x == 0) report(p.err, TQ_ERR_TIMEOUT);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, C::TMEM_COLS);
}


// ---------------------------------------------------------------------------
// Keys only (search databases, key-only appends): the same steps, software
// pipelined over tiles and warp-specialised.  One warp issues the copies and
// the tensor-core work (one lane); sixteen warps quantise, a thread owning one
// row and a quarter of its columns.  The rotation of tile t+1 (two TMEM
// accumulators) and the sketch of tile t (its residual kept in TMEM as the
// sketch's A operand, two buffers) run while the sixteen warps quantise;
// input tiles are double-buffered.  Hand-offs go through mbarriers:
//   full[b]     input tile b landed (and its tile record published)
//   rk[b]       rotation of the tile in buffer b done
//   resfull[b]  tile b quantised: residual in TMEM, input and rotation
//               buffers free
//   sk          sketch done;  skfree  sketch accumulator read
// A tile record ring in shared memory carries each tile's page and row range
// from the issuing lane to the quantising warps (bh < 0: no further tile).
// ---------------------------------------------------------------------------
// sum of squares of this thread's part (quarter) of a row of a 16-bit tile
template <int D, bool BF>
__device__ __forceinline__ float part_row_sumsq(const uint8_t* x, int row, int q) {
  constexpr int PART = D / 4;
  float ss = 0.0f;
#pragma unroll
  for (int c = 0; c < PART / 8; ++c) {
    const int k = q * PART + 8 * c;
    const uint4 v = *reinterpret_cast<const uint4*>(x + tc::sw128_offset(row, k, ROWS));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a, b;
      if constexpr (BF) {
        a = __uint_as_float(w[i] << 16);
        b = __uint_as_float(w[i] & 0xFFFF0000u);
      } else {
        const __half2 hh = *reinterpret_cast<const __half2*>(&w[i]);
        a = __low2float(hh);
        b = __high2float(hh);
      }
      ss = fmaf(a, a, fmaf(b, b, ss));
    }
  }
  return ss;
}

template <int N>
__device__ __forceinline__ void tmem_load_part(uint32_t taddr, float (&x)[N]) {
  uint32_t r[N];
  if constexpr (N == 32) tc::ld32(taddr, r);
  else tc::ld16(taddr, r);
  tc::wait_ld();
#pragma unroll
  for (int i = 0; i < N; ++i) x[i] = __uint_as_float(r[i]);
}

constexpr int KEPI = 16;                    // quantising warps
constexpr int KTHREADS = (KEPI + 1) * 32;   // + the issuing warp
constexpr int NPART = 4;                    // column quarters

template <int D>
struct KCfg {
  static constexpr int PART = D / NPART;  // columns per thread
  static constexpr int OPB = D * 128;
  static constexpr int OP = (D / 64) * OPB;
  static constexpr int XB = ROWS * 128;
  static constexpr int XT = (D / 64) * XB;
  static constexpr int OFF_PH = 0;
  static constexpr int OFF_PL = OFF_PH + OP;
  static constexpr int OFF_S = OFF_PL + OP;
  static constexpr int OFF_X = OFF_S + OP;            // two input tiles
  static constexpr int OFF_NK = OFF_X + 2 * XT;       // float[2][4][128] key norm^2 parts
  static constexpr int OFF_G = OFF_NK + 2 * 4 * 512;  // float[2][4][128] residual norm^2 parts
  static constexpr int OFF_RING = OFF_G + 2 * 4 * 512;  // Tile[4]
  static constexpr int OFF_BAR = OFF_RING + 128;      // 9 mbarriers
  static constexpr int OFF_TMEM = OFF_BAR + 128;
  static constexpr int OFF_FAIL = OFF_TMEM + 4;
  static constexpr int SMEM = OFF_TMEM + 16 + 1024;   // + alignment slack
  // TMEM columns: two rotation accumulators, the sketch accumulator, two
  // fp16 residual buffers (A operand: two K elements per 32-bit column)
  static constexpr int COL_RK0 = 0, COL_SK = 2 * D, COL_RES0 = 3 * D;
  static constexpr uint32_t TMEM_COLS = (4 * D <= 256) ? 256 : 512;
  static_assert(COL_RES0 + D <= static_cast<int>(TMEM_COLS), "TMEM columns");
  static_assert(sizeof(Tile) * 4 <= 128, "tile ring");
};

// barrier among the quantising warps (named barrier 1), returning whether any
// of their threads passed `pred`
__device__ __forceinline__ bool epi_sync_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(KEPI * 32)
      : "memory");
  return r != 0;
}

template <int D, bool BF>
__global__ void __maxnreg__(96) compress_keys_kernel(const __grid_constant__ CUtensorMap mapK, Params p) {
  using C = KCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t s0 = smem_u32(smem);
  const uint32_t bar_full = s0 + C::OFF_BAR, bar_rk = bar_full + 16, bar_res = bar_full + 32;
  const uint32_t bar_sk = bar_full + 48, bar_skfree = bar_full + 56, bar_drain = bar_full + 64;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  int* fail_flag = reinterpret_cast<int*>(smem + C::OFF_FAIL);
  float* nk = reinterpret_cast<float*>(smem + C::OFF_NK);
  float* gp = reinterpret_cast<float*>(smem + C::OFF_G);
  Tile* ring = reinterpret_cast<Tile*>(smem + C::OFF_RING);

  for (int i = tid; i < D * (D / 8); i += KTHREADS) {
    const int r = i / (D / 8), k = (i % (D / 8)) * 8;
    const uint32_t off = tc::sw128_offset(r, k, D);
    *reinterpret_cast<uint4*>(smem + C::OFF_PH + off) =
        *reinterpret_cast<const uint4*>(p.pi_hi + static_cast<size_t>(r) * D + k);
    *reinterpret_cast<uint4*>(smem + C::OFF_PL + off) =
        *reinterpret_cast<const uint4*>(p.pi_lo + static_cast<size_t>(r) * D + k);
    *reinterpret_cast<uint4*>(smem + C::OFF_S + off) =
        *reinterpret_cast<const uint4*>(p.s_h + static_cast<size_t>(r) * D + k);
  }
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(bar_full + 8 * i, 1);       // full[2], rk[2]
    for (int i = 0; i < 2; ++i) mbar_init(bar_res + 8 * i, KEPI);     // resfull[2]
    mbar_init(bar_sk, 1);
    mbar_init(bar_skfree, KEPI);
    mbar_init(bar_drain, 1);
    *fail_flag = 0;
    mbar_init_fence();
  }
  if (warp == KEPI) {
    tc::tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  if (warp == KEPI) {
    // ---- copies and tensor-core work, one lane ------------------------------
    if (lane == 0) {
      bool failed = false;
      int tsearch = blockIdx.x;
      uint32_t loads[2] = {0u, 0u}, landed[2] = {0u, 0u};
      // publish the record of tile `idx` of this CTA's sequence and start its
      // copy into buffer `buf`; a missing tile publishes bh = -1
      auto fetch = [&](uint32_t idx, uint32_t buf) -> bool {
        Tile tl;
        const bool ok = next_tile(p, tsearch, tl);
        if (ok) tsearch += gridDim.x;
        else tl.bh = -1;
        ring[idx & 3u] = tl;
        if (ok) {
          fence_proxy_async_smem();
          issue_tile_load<D>(&mapK, s0 + C::OFF_X + buf * C::XT, bar_full + 8 * buf, tl);
          ++loads[buf];
        } else {
          mbar_arrive(bar_full + 8 * buf);  // releases the record
        }
        return ok;
      };
      auto rotate = [&](uint32_t idx) -> bool {
        const uint32_t bb = idx & 1u;
        if (!mbar_wait_bounded(bar_full + 8 * bb, (idx >> 1) & 1u)) return false;
        ++landed[bb];
        tc::fence_after_sync();
        issue_rotation<D, BF>(tmem, C::COL_RK0 + static_cast<int>(bb) * D, s0 + C::OFF_X + bb * C::XT,
                              s0 + C::OFF_PH, s0 + C::OFF_PL);
        tc::commit(bar_rk + 8 * bb);
        return true;
      };
      constexpr uint32_t idesc_sk = tc::idesc_f16(ROWS, D, false);
      bool h_cur = fetch(0, 0);
      bool h_next = h_cur && fetch(1, 1);
      if (h_cur && !rotate(0)) failed = true;
      for (uint32_t it = 0; h_cur && !failed; ++it) {
        const uint32_t b = it & 1u;
        if (h_next && !rotate(it + 1)) { failed = true; break; }
        // tile it quantised: its buffers are free and its residual is ready
        if (!mbar_wait_bounded(bar_res + 8 * b, (it >> 1) & 1u)) { failed = true; break; }
        bool h_next2 = false;
        if (h_next) h_next2 = fetch(it + 2, b);
        if (it > 0 && !mbar_wait_bounded(bar_skfree, (it - 1) & 1u)) { failed = true; break; }
        tc::fence_after_sync();
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          const int kb = s >> 2, w = (s & 3) * 32;
          tc::mma_f16_tmem_a(tmem + C::COL_SK, tmem + C::COL_RES0 + b * (D / 2) + 8 * s,
                             tc::sdesc_sw128(s0 + C::OFF_S + kb * C::OPB + w), idesc_sk, s > 0);
        }
        tc::commit(bar_sk);
        h_cur = h_next;
        h_next = h_next2;
      }
      // no copy or product may still be in flight when the CTA exits
      for (int bb = 0; bb < 2; ++bb)
        for (uint32_t k2 = landed[bb]; k2 < loads[bb]; ++k2) mbar_wait_bounded(bar_full + 8 * bb, k2 & 1u);
      tc::commit(bar_drain);
      mbar_wait_bounded(bar_drain, 0);
      if (failed) *fail_flag = 1;
    }
    __syncwarp();
  } else {
    // ---- sixteen warps: quantise, then the previous tile's sign bits --------
    const int row = 32 * (warp & 3) + lane;  // TMEM lane quarter of this warp
    const int q = warp >> 2;                 // column quarter
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    bool failed = false;
    Tile cur, prev;
    bool have_prev = false;
    float prev_n = 0.0f;
    for (uint32_t it = 0;; ++it) {
      const uint32_t b = it & 1u;
      // the tile's record (released with its copy)
      if (!mbar_wait_bounded(bar_full + 8 * b, (it >> 1) & 1u)) failed = true;
      cur = ring[it & 3u];
      if (epi_sync_or(failed)) {
        failed = true;
        break;
      }
      const bool have = cur.bh >= 0;
      if (!have && !have_prev) break;
      float x[C::PART];
      float n = 0.0f;
      if (have) {
        if (!mbar_wait_bounded(bar_rk + 8 * b, (it >> 1) & 1u)) failed = true;
        tc::fence_after_sync();
        nk[(b * NPART + q) * ROWS + row] = part_row_sumsq<D, BF>(smem + C::OFF_X + b * C::XT, row, q);
        tmem_load_part<C::PART>(t_lane + C::COL_RK0 + b * D + q * C::PART, x);
      }
      if (epi_sync_or(failed)) {  // norm parts complete
        failed = true;
        break;
      }
      if (have) {
        const bool page_ok = cur.page >= 0 && cur.page < p.pool_pages;
        const bool wr = page_ok && row >= cur.s_lo && row < cur.s_hi;
        if (tid == 0 && !page_ok) report(p.err, TQ_ERR_CAPACITY);
        uint8_t* pg = p.pool + static_cast<size_t>(page_ok ? cur.page : 0) * p.page_bytes;
        const float* nkb = nk + b * NPART * ROWS;
        const float nn = sqrtf((nkb[row] + nkb[ROWS + row]) + (nkb[2 * ROWS + row] + nkb[3 * ROWS + row]));
        const __half nh = __float2half_rn(nn);
        n = __half2float(nh);
        const float T0 = __fmul_rn(n, p.kt0);
        const float inv = n > 0.0f ? 1.0f / n : 0.0f;
        // Per coordinate: magnitude index u = [|v| >= n t], residual
        // r = v / n - c_hat (computed as for n > 0; a zero vector's row is
        // cleared below).  Key word w: coordinate 16 w + 8 h + 2 i + e has its
        // sign bit at 16 h + 15 - 4 i - e and its magnitude bit two below, so
        // the coordinates are taken in the words' bit order (h = 1 first) and
        // their bits shifted in from the most significant end, one funnel
        // shift each (the sign bit is the float's).
        uint32_t kw[C::PART / 16];
        uint32_t rh[C::PART / 2];
        float g2 = 0.0f;
#pragma unroll
        for (int w = 0; w < C::PART / 16; ++w) {
          uint32_t acc = 0u;
#pragma unroll
          for (int hh = 1; hh >= 0; --hh)
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
              const int j = 16 * w + 8 * hh + 2 * ii;
              float rr[2];
              uint32_t mb[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const float v = x[j + e];
                const bool big = fabsf(v) >= T0;
                // |r| = |v| / n - c_u, with the sign of v (the level's sign)
                const float m = fmaf(fabsf(v), inv, big ? -p.kc1 : -p.kc0);
                rr[e] = __uint_as_float(__float_as_uint(m) ^ (__float_as_uint(v) & 0x80000000u));
                g2 = fmaf(m, m, g2);
                mb[e] = big ? 0x80000000u : 0u;
              }
              const __half2 pr = __floats2half2_rn(rr[0], rr[1]);
              rh[j / 2] = *reinterpret_cast<const uint32_t*>(&pr);
              acc = __funnelshift_l(__float_as_uint(x[j]), acc, 1);
              acc = __funnelshift_l(__float_as_uint(x[j + 1]), acc, 1);
              acc = __funnelshift_l(mb[0], acc, 1);
              acc = __funnelshift_l(mb[1], acc, 1);
            }
          kw[w] = acc;
        }
        if (!(n > 0.0f)) {  // zero vector: all codes, residual and its norm are 0
#pragma unroll
          for (int w = 0; w < C::PART / 16; ++w) kw[w] = 0u;
#pragma unroll
          for (int i2 = 0; i2 < C::PART / 2; ++i2) rh[i2] = 0u;
          g2 = 0.0f;
        }
        // residual: fp16, coordinates 2c, 2c+1 in TMEM column c of this buffer
        if constexpr (C::PART / 2 == 16)
          tc::st16(t_lane + C::COL_RES0 + b * (D / 2) + q * (C::PART / 2), rh);
        else
          tc::st8(t_lane + C::COL_RES0 + b * (D / 2) + q * (C::PART / 2), rh);
        gp[(b * NPART + q) * ROWS + row] = g2;
        if (wr && TQ_IN_RANGE(p.err, p.off_kc + row * (D / 4) + (q + 1) * (C::PART / 4) - 1,
                              p.page_bytes)) {
          if constexpr (C::PART / 16 == 2)
            *reinterpret_cast<uint2*>(pg + p.off_kc + row * (D / 4) + q * (C::PART / 4)) =
                make_uint2(kw[0], kw[1]);
          else
            *reinterpret_cast<uint32_t*>(pg + p.off_kc + row * (D / 4) + q * (C::PART / 4)) = kw[0];
          if (q == 0) reinterpret_cast<__half*>(pg + p.off_kn)[row] = nh;
        }
        tc::wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_res + 8 * b);
      }
      if (have_prev) {
        if (!mbar_wait_bounded(bar_sk, (it - 1) & 1u)) failed = true;
        tc::fence_after_sync();
        tmem_load_part<C::PART>(t_lane + C::COL_SK + q * C::PART, x);
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_skfree);
        const bool page_ok = prev.page >= 0 && prev.page < p.pool_pages;
        if (!failed && page_ok && row >= prev.s_lo && row < prev.s_hi &&
            TQ_IN_RANGE(p.err, p.off_qs + row * (D / 8) + (q + 1) * (C::PART / 8) - 1, p.page_bytes)) {
          uint8_t* pgp = p.pool + static_cast<size_t>(prev.page) * p.page_bytes;
          // sketch index i of the part sits in its 32-bit word at bit
          // 16 (i / 16 mod 2) + 15 - i mod 16 (a part of 16 fills one half word)
          // (the float's sign bit, shifted in from the most significant end:
          // indices 16..31 of the word first, then 0..15)
          uint32_t qw = 0u;
#pragma unroll
          for (int k2 = 0; k2 < C::PART; ++k2) {
            const int i = C::PART == 32 ? (k2 + 16) & 31 : k2;
            qw = __funnelshift_l(__float_as_uint(x[i]), qw, 1);
          }
          if (!(prev_n > 0.0f)) qw = 0u;  // zero vector
          if constexpr (C::PART == 32)
            *reinterpret_cast<uint32_t*>(pgp + p.off_qs + row * (D / 8) + q * 4) = qw;
          else
            *reinterpret_cast<uint16_t*>(pgp + p.off_qs + row * (D / 8) + q * 2) = static_cast<uint16_t>(qw);
          if (q == 0) {
            const float* gpp = gp + (b ^ 1u) * NPART * ROWS;
            reinterpret_cast<__half*>(pgp + p.off_kg)[row] = __float2half_rn(
                sqrtf((gpp[row] + gpp[ROWS + row]) + (gpp[2 * ROWS + row] + gpp[3 * ROWS + row])));
          }
        }
      }
      prev = cur;
      prev_n = n;
      have_prev = have;
      if (!have) break;  // the last tile's sign bits are out
    }
    if (failed && lane == 0) *fail_flag = 1;
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == KEPI) tc::tmem_dealloc(tmem, C::TMEM_COLS);
  if (tid == 0 && *fail_flag) report(p.err, TQ_ERR_TIMEOUT);
}

}  // namespace ctc

__global__ void advance_cold_len(int32_t* cold_len, int B, int n_new) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) cold_len[b] += n_new;
}

int launch_compress_tc(const tq_ctx* ctx, const void* k, const void* v, bool bf16, int B, int Hkv,
                       int n_new, uint8_t* pool, int64_t pool_pages, const int32_t* page_table,
                       int max_pages, int32_t* cold_len, void* stream, const int32_t* n_new_b) {
  const int d = ctx->cfg.head_dim;
  const PageLayout L = page_layout(d, ctx->cfg.qjl_dim, v != nullptr);
  ctc::Params p{};
  p.B = B;
  p.Hkv = Hkv;
  p.n_new = n_new;
  p.has_v = v != nullptr;
  p.pool = pool;
  p.pool_pages = pool_pages;
  p.page_bytes = static_cast<long long>(L.bytes);
  p.off_kc = static_cast<int>(L.kc);
  p.off_qs = static_cast<int>(L.qs);
  p.off_vc = static_cast<int>(L.vc);
  p.off_kn = static_cast<int>(L.kn);
  p.off_kg = static_cast<int>(L.kg);
  p.off_vn = static_cast<int>(L.vn);
  p.off_kl = static_cast<int>(L.kl);
  p.blk = static_cast<int>(L.block);
  p.page_table = page_table;
  p.max_pages = max_pages;
  p.cold_len = cold_len;
  p.pi_hi = bf16 ? ctx->dev.rot_bf_hi : ctx->dev.rot_h_hi;
  p.pi_lo = bf16 ? ctx->dev.rot_bf_lo : ctx->dev.rot_h_lo;
  p.s_h = ctx->dev.qjl_h;
  p.kc0 = ctx->cb.key_c[0];
  p.kc1 = ctx->cb.key_c[1];
  p.kt0 = ctx->cb.key_t[0];
  for (int i = 0; i < 7; ++i) p.vt[i] = ctx->cb.val_t[i];
  p.err = ctx->dev.err;
  p.tiles_per_bh = (n_new + ctc::ROWS - 1) / ctc::ROWS + 1;
  p.n_new_b = n_new_b;
  CUtensorMap mk, mv;
  const uint64_t dims[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(n_new),
                            static_cast<uint64_t>(B) * Hkv};
  const uint64_t strides[2] = {static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(n_new) * d * 2};
  const uint32_t box[3] = {64, ctc::ROWS, 1};
  if (!tc::encode_map_3d(&mk, bf16, k, dims, strides, box)) return TQ_ERR_CUDA;
  if (v) {
    if (!tc::encode_map_3d(&mv, bf16, v, dims, strides, box)) return TQ_ERR_CUDA;
  } else {
    mv = mk;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long tiles = static_cast<long long>(B) * Hkv * p.tiles_per_bh;
  const int grid = static_cast<int>(tiles < ctx->num_sms ? tiles : ctx->num_sms);
  auto go = [&](auto kern, int smem) -> int {
    // one record per kernel: every instantiation has the same function-pointer
    // type, so they are told apart by head dim and input type
    static SmemAttr attr[4];
    const int slot = (d == 128 ? 2 : 0) + (bf16 ? 1 : 0);
    if (!raise_smem_limit(kern, smem, attr[slot])) return TQ_ERR_CUDA;
    if (ctx->prof_start) cudaEventRecord(static_cast<cudaEvent_t>(ctx->prof_start), st);
    kern<<<grid, ctc::NTHREADS, smem, st>>>(mk, mv, p);
    if (ctx->prof_stop) cudaEventRecord(static_cast<cudaEvent_t>(ctx->prof_stop), st);
    // per-sequence counts: the caller advances the lengths
    if (!n_new_b) advance_cold_len<<<(B + 127) / 128, 128, 0, st>>>(cold_len, B, n_new);
    return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
  };
  if (!v) {
    // keys only: the software-pipelined kernel
    auto gok = [&](auto kern, int smem) -> int {
      static SmemAttr attr[4];  // per head dim and input type, as above
      const int slot = (d == 128 ? 2 : 0) + (bf16 ? 1 : 0);
      if (!raise_smem_limit(kern, smem, attr[slot])) return TQ_ERR_CUDA;
      if (ctx->prof_start) cudaEventRecord(static_cast<cudaEvent_t>(ctx->prof_start), st);
      kern<<<grid, ctc::KTHREADS, smem, st>>>(mk, p);
      if (ctx->prof_stop) cudaEventRecord(static_cast<cudaEvent_t>(ctx->prof_stop), st);
      if (!n_new_b) advance_cold_len<<<(B + 127) / 128, 128, 0, st>>>(cold_len, B, n_new);
      return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
    };
    if (d == 128)
      return bf16 ? gok(ctc::compress_keys_kernel<128, true>, ctc::KCfg<128>::SMEM)
                  : gok(ctc::compress_keys_kernel<128, false>, ctc::KCfg<128>::SMEM);
    return bf16 ? gok(ctc::compress_keys_kernel<64, true>, ctc::KCfg<64>::SMEM)
                : gok(ctc::compress_keys_kernel<64, false>, ctc::KCfg<64>::SMEM);
  }
  if (d == 128)
    return bf16 ? go(ctc::compress_tc_kernel<128, true>, ctc::Cfg<128>::SMEM)
                : go(ctc::compress_tc_kernel<128, false>, ctc::Cfg<128>::SMEM);
  return bf16 ? go(ctc::compress_tc_kernel<64, true>, ctc::Cfg<64>::SMEM)
              : go(ctc::compress_tc_kernel<64, false>, ctc::Cfg<64>::SMEM);
}

}  // namespace tq
