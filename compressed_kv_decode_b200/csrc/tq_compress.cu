// Compress and append ("TurboQuant" summary, de.news.hada.io topic 27867,
// section "Funktionsweise von TurboQuant": random rotation, per-coordinate
// quantiser, 1-bit QJL on the residual; eviction of old tokens into the cold
// region, "Monarch v3", section "Wie es funktioniert").
//
// One CTA tile = the 128 token slots of one destination page of one
// (batch, kv head); 8 warps x 16 rows.  Persistent CTAs keep Pi (fp16 or bf16,
// hi/lo split) and S (fp16) in shared memory.  Per tile:
//   x_rot = Pi x     tensor-core MMA, hi + lo parts of Pi, fp32 accumulate
//   n = fp16(|x|), codes against fp32(n * t_k), residual r = x_rot/n - c_hat
//   p = S r          tensor-core MMA on r rounded to fp16
//   sign bits, gamma = fp16(|r|), bit-plane / nibble packing in registers
//   page assembled in shared memory, stored with 16-byte coalesced stores.
#include <cuda_runtime.h>

#include <cstdint>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace cmp {

constexpr int NWARP = 8;
constexpr int ROWS = 128;

enum { IN_F16 = 0, IN_BF16 = 1, IN_ROT_F32 = 2 };

template <int D>
struct Cfg {
  static constexpr int KS = D / 16;  // k-steps
  static constexpr int NTL = D / 8;  // n-tiles (rotation and sketch, m = D)
  static constexpr int RB = 2 * D + 16;
  static constexpr int WPT = D / 64;  // key code words written per lane per row
  static constexpr int OFF_PH = 0;
  static constexpr int OFF_PL = OFF_PH + D * RB;
  static constexpr int OFF_S = OFF_PL + D * RB;
  static constexpr int OFF_X = OFF_S + D * RB;
  static constexpr int OFF_STG = OFF_X + ROWS * RB;
  static constexpr int STG_KC = 0;
  static constexpr int STG_QS = STG_KC + ROWS * D / 4;
  static constexpr int STG_VC = STG_QS + ROWS * D / 8;
  static constexpr int STG_KN = STG_VC + ROWS / 2 * D;
  static constexpr int STG_KG = STG_KN + 2 * ROWS;
  static constexpr int STG_VN = STG_KG + 2 * ROWS;
  static constexpr int STG_B = STG_VN + 2 * ROWS;
  static constexpr int SMEM = OFF_STG + STG_B;
};

struct Params {
  const void* k;
  const void* v;
  int B, Hkv, n_new;
  uint8_t* pool;
  long long pool_pages, page_bytes;
  int off_kc, off_qs, off_vc, off_kn, off_kg, off_vn;
  int off_kl, blk;  // pages with values: key plane L, block bytes (block layout)
  const int32_t* page_table;
  int max_pages;
  const int32_t* cold_len;
  const uint16_t* pi_hi;  // fp16 or bf16 bits, [D][D]
  const uint16_t* pi_lo;
  const uint16_t* s_h;    // fp16 bits, [D][D]
  float kc0, kc1, kt0;
  float vt[7];
  int* err;
  int tiles_per_bh;
};

template <int IN>
__device__ __forceinline__ void mma_in(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (IN == IN_BF16)
    mma_bf16(d, a0, a1, a2, a3, b0, b1);
  else
    mma_f16(d, a0, a1, a2, a3, b0, b1);
}

__device__ __forceinline__ float in_to_float(uint16_t h, int in) {
  return in == IN_BF16 ? __bfloat162float(__ushort_as_bfloat16(h)) : __half2float(__ushort_as_half(h));
}

// x_rot rows [16 w, 16 w + 16) of the tile: acc[t] = (row g, cols 8t+2c, +1; row g+8, ...)
template <int D, int IN>
__device__ __forceinline__ void rotate_warp(const uint8_t* smem, int warp, int lane,
                                            float (&acc)[Cfg<D>::NTL][4]) {
  using C = Cfg<D>;
#pragma unroll
  for (int t = 0; t < C::NTL; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
  const uint32_t xa = smem_u32(smem + C::OFF_X) + (16 * warp + (lane & 15)) * C::RB + (lane >> 4) * 16;
  const uint32_t pn = ((lane & 7) + ((lane >> 4) & 1) * 8) * C::RB + ((lane >> 3) & 1) * 16;
  const uint32_t ph = smem_u32(smem + C::OFF_PH) + pn, pl = smem_u32(smem + C::OFF_PL) + pn;
#pragma unroll
  for (int s = 0; s < C::KS; ++s) {
    uint32_t a0, a1, a2, a3;
    ldsm_x4(xa + s * 32, a0, a1, a2, a3);
#pragma unroll
    for (int t = 0; t < C::NTL; t += 2) {
      uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
      ldsm_x4(ph + t * 8 * C::RB + s * 32, h0, h1, h2, h3);
      ldsm_x4(pl + t * 8 * C::RB + s * 32, l0, l1, l2, l3);
      mma_in<IN>(acc[t], a0, a1, a2, a3, h0, h1);
      mma_in<IN>(acc[t], a0, a1, a2, a3, l0, l1);
      mma_in<IN>(acc[t + 1], a0, a1, a2, a3, h2, h3);
      mma_in<IN>(acc[t + 1], a0, a1, a2, a3, l2, l3);
    }
  }
}

template <int D, int IN>
__global__ void __launch_bounds__(NWARP * 32, 1) compress_kernel(Params p) {
  using C = Cfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;

  // resident tables: Pi hi/lo and S, rows padded to RB bytes
  for (int i = tid; i < D * (D / 8); i += blockDim.x) {
    const int r = i / (D / 8), ch = i % (D / 8);
    if constexpr (IN != IN_ROT_F32) {
      reinterpret_cast<uint4*>(smem + C::OFF_PH + r * C::RB)[ch] =
          reinterpret_cast<const uint4*>(p.pi_hi + static_cast<size_t>(r) * D)[ch];
      reinterpret_cast<uint4*>(smem + C::OFF_PL + r * C::RB)[ch] =
          reinterpret_cast<const uint4*>(p.pi_lo + static_cast<size_t>(r) * D)[ch];
    }
    reinterpret_cast<uint4*>(smem + C::OFF_S + r * C::RB)[ch] =
        reinterpret_cast<const uint4*>(p.s_h + static_cast<size_t>(r) * D)[ch];
  }
  __syncthreads();

  uint8_t* stg = smem + C::OFF_STG;
  const int BH = p.B * p.Hkv;
  const int total = BH * p.tiles_per_bh;
  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    const int bh = tile / p.tiles_per_bh, ti = tile % p.tiles_per_bh;
    const int b = bh / p.Hkv;
    const int cl = p.cold_len[b];
    const int lpage = cl / ROWS + ti;
    const int s_lo = max(cl, lpage * ROWS) - lpage * ROWS;
    const int s_hi = min(cl + p.n_new, (lpage + 1) * ROWS) - lpage * ROWS;
    if (s_lo >= s_hi) continue;  // uniform across the CTA
    int page = -1;
    if (lpage < p.max_pages) page = p.page_table[static_cast<size_t>(bh) * p.max_pages + lpage];
    if (page < 0 || page >= p.pool_pages) {
      if (tid == 0) report(p.err, TQ_ERR_CAPACITY);
      continue;
    }
    const long long in_base = static_cast<long long>(bh) * p.n_new + (static_cast<long long>(lpage) * ROWS - cl);

    for (int pass = 0; pass < (p.v ? 2 : 1); ++pass) {
      const bool is_key = (pass == 0);
      const void* src = is_key ? p.k : p.v;
      float acc[C::NTL][4];
      float ss0 = 0.0f, ss1 = 0.0f;
      const int r0 = 16 * warp + g, r1 = r0 + 8;
      if constexpr (IN == IN_ROT_F32) {
        const float* x = static_cast<const float*>(src);
        const bool ok0 = r0 >= s_lo && r0 < s_hi, ok1 = r1 >= s_lo && r1 < s_hi;
#pragma unroll
        for (int t = 0; t < C::NTL; ++t) {
          float2 v0 = make_float2(0.f, 0.f), v1 = make_float2(0.f, 0.f);
          if (ok0) v0 = *reinterpret_cast<const float2*>(x + (in_base + r0) * D + 8 * t + 2 * c);
          if (ok1) v1 = *reinterpret_cast<const float2*>(x + (in_base + r1) * D + 8 * t + 2 * c);
          acc[t][0] = v0.x; acc[t][1] = v0.y; acc[t][2] = v1.x; acc[t][3] = v1.y;
          ss0 = fmaf(v0.x, v0.x, fmaf(v0.y, v0.y, ss0));
          ss1 = fmaf(v1.x, v1.x, fmaf(v1.y, v1.y, ss1));
        }
      } else {
        // stage the 16-bit input tile; slots outside [s_lo, s_hi) are zero
        const uint16_t* x = static_cast<const uint16_t*>(src);
        for (int i = tid; i < ROWS * (D / 8); i += blockDim.x) {
          const int r = i / (D / 8), ch = i % (D / 8);
          uint4 val = make_uint4(0u, 0u, 0u, 0u);
          if (r >= s_lo && r < s_hi)
            val = reinterpret_cast<const uint4*>(x + (in_base + r) * D)[ch];
          reinterpret_cast<uint4*>(smem + C::OFF_X + r * C::RB)[ch] = val;
        }
        __syncthreads();
        rotate_warp<D, IN>(smem, warp, lane, acc);
        // |x|^2 from the input row
#pragma unroll
        for (int t = 0; t < C::NTL; ++t) {
          const uint32_t w0 = *reinterpret_cast<const uint32_t*>(smem + C::OFF_X + r0 * C::RB + 2 * (8 * t + 2 * c));
          const uint32_t w1 = *reinterpret_cast<const uint32_t*>(smem + C::OFF_X + r1 * C::RB + 2 * (8 * t + 2 * c));
          const float a = in_to_float(w0 & 0xFFFFu, IN), bb = in_to_float(w0 >> 16, IN);
          const float e = in_to_float(w1 & 0xFFFFu, IN), f = in_to_float(w1 >> 16, IN);
          ss0 = fmaf(a, a, fmaf(bb, bb, ss0));
          ss1 = fmaf(e, e, fmaf(f, f, ss1));
        }
      }
      ss0 += __shfl_xor_sync(0xffffffffu, ss0, 1);
      ss0 += __shfl_xor_sync(0xffffffffu, ss0, 2);
      ss1 += __shfl_xor_sync(0xffffffffu, ss1, 1);
      ss1 += __shfl_xor_sync(0xffffffffu, ss1, 2);
      const __half nh0 = __float2half_rn(sqrtf(ss0)), nh1 = __float2half_rn(sqrtf(ss1));
      const float n0 = __half2float(nh0), n1 = __half2float(nh1);
      __syncwarp();  // every lane has read its input row: the rows may now hold r

      if (is_key) {
        const float T0 = __fmul_rn(n0, p.kt0), T1 = __fmul_rn(n1, p.kt0);
        const float inv0 = n0 > 0.0f ? 1.0f / n0 : 0.0f, inv1 = n1 > 0.0f ? 1.0f / n1 : 0.0f;
        // record words (keys-only pages) or plane masks H | L (pages with
        // values: word w < D/32 of H, word D/32 + w of L, bit j % 32)
        uint32_t kw0[D / 16], kw1[D / 16];
#pragma unroll
        for (int w = 0; w < D / 16; ++w) kw0[w] = kw1[w] = 0u;
        const bool planes = p.v != nullptr;
        float gg0 = 0.0f, gg1 = 0.0f;
#pragma unroll
        for (int t = 0; t < C::NTL; ++t) {
          float rr[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x = acc[t][e];
            const bool row1 = e >= 2;
            const float T = row1 ? T1 : T0, inv = row1 ? inv1 : inv0, nn = row1 ? n1 : n0;
            const uint32_t sg = (x < 0.0f) ? 1u : 0u;
            const uint32_t mg = (nn > 0.0f && fabsf(x) >= T) ? 1u : 0u;
            const float cpos = mg ? p.kc1 : p.kc0;
            const float r = (nn > 0.0f) ? fmaf(x, inv, sg ? cpos : -cpos) : 0.0f;
            rr[e] = r;
            const int ei = e & 1;
            const uint32_t sgn = nn > 0.0f ? sg : 0u;
            if (planes) {  // H = 1 - sign, L = sign XOR magnitude, bit j % 32
              const int j = 8 * t + 2 * c + ei;
              const uint32_t hb = (1u - sgn) << (j & 31), lb = (sgn ^ mg) << (j & 31);
              if (row1) { kw1[j >> 5] |= hb; kw1[D / 32 + (j >> 5)] |= lb; }
              else { kw0[j >> 5] |= hb; kw0[D / 32 + (j >> 5)] |= lb; }
            } else {
              const int sbit = 16 * (t & 1) + 15 - 4 * c - ei;
              const uint32_t bits = (sgn << sbit) | (mg << (sbit - 2));
              if (row1) kw1[t >> 1] |= bits; else kw0[t >> 1] |= bits;
            }
            if (row1) gg1 = fmaf(r, r, gg1); else gg0 = fmaf(r, r, gg0);
          }
          // r as fp16 into this warp's rows of the tile (A operand of the sketch)
          *reinterpret_cast<__half2*>(smem + C::OFF_X + r0 * C::RB + 2 * (8 * t + 2 * c)) =
              __floats2half2_rn(rr[0], rr[1]);
          *reinterpret_cast<__half2*>(smem + C::OFF_X + r1 * C::RB + 2 * (8 * t + 2 * c)) =
              __floats2half2_rn(rr[2], rr[3]);
        }
#pragma unroll
        for (int w = 0; w < D / 16; ++w) {
          kw0[w] |= __shfl_xor_sync(0xffffffffu, kw0[w], 1);
          kw0[w] |= __shfl_xor_sync(0xffffffffu, kw0[w], 2);
          kw1[w] |= __shfl_xor_sync(0xffffffffu, kw1[w], 1);
          kw1[w] |= __shfl_xor_sync(0xffffffffu, kw1[w], 2);
        }
#pragma unroll
        for (int w = 0; w < D / 16; ++w) {
          if (w / C::WPT == c) {
            if (planes) {  // [128][D/32] H masks, then [128][D/32] L masks
              const int pl = w / (D / 32), ww = w % (D / 32);
              uint32_t* mk = reinterpret_cast<uint32_t*>(stg + C::STG_KC + pl * (ROWS * D / 8));
              mk[r0 * (D / 32) + ww] = kw0[w];
              mk[r1 * (D / 32) + ww] = kw1[w];
            } else {
              reinterpret_cast<uint32_t*>(stg + C::STG_KC + r0 * (D / 4))[w] = kw0[w];
              reinterpret_cast<uint32_t*>(stg + C::STG_KC + r1 * (D / 4))[w] = kw1[w];
            }
          }
        }
        gg0 += __shfl_xor_sync(0xffffffffu, gg0, 1);
        gg0 += __shfl_xor_sync(0xffffffffu, gg0, 2);
        gg1 += __shfl_xor_sync(0xffffffffu, gg1, 1);
        gg1 += __shfl_xor_sync(0xffffffffu, gg1, 2);
        if (c == 0) {
          reinterpret_cast<__half*>(stg + C::STG_KN)[r0] = nh0;
          reinterpret_cast<__half*>(stg + C::STG_KN)[r1] = nh1;
          reinterpret_cast<__half*>(stg + C::STG_KG)[r0] = __float2half_rn(sqrtf(gg0));
          reinterpret_cast<__half*>(stg + C::STG_KG)[r1] = __float2half_rn(sqrtf(gg1));
        }
        __syncwarp();
        // sketch p = S r on the tensor cores (r fp16, S fp16)
        float pk[C::NTL][4];
#pragma unroll
        for (int t = 0; t < C::NTL; ++t) pk[t][0] = pk[t][1] = pk[t][2] = pk[t][3] = 0.0f;
        {
          const uint32_t ra = smem_u32(smem + C::OFF_X) + (16 * warp + (lane & 15)) * C::RB + (lane >> 4) * 16;
          const uint32_t sb = smem_u32(smem + C::OFF_S) +
                              ((lane & 7) + ((lane >> 4) & 1) * 8) * C::RB + ((lane >> 3) & 1) * 16;
#pragma unroll
          for (int s = 0; s < C::KS; ++s) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(ra + s * 32, a0, a1, a2, a3);
#pragma unroll
            for (int t = 0; t < C::NTL; t += 2) {
              uint32_t b0, b1, b2, b3;
              ldsm_x4(sb + t * 8 * C::RB + s * 32, b0, b1, b2, b3);
              mma_f16(pk[t], a0, a1, a2, a3, b0, b1);
              mma_f16(pk[t + 1], a0, a1, a2, a3, b2, b3);
            }
          }
        }
        uint32_t qw0[D / 32], qw1[D / 32];
#pragma unroll
        for (int w = 0; w < D / 32; ++w) qw0[w] = qw1[w] = 0u;
#pragma unroll
        for (int t = 0; t < C::NTL; ++t) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int ei = e & 1;
            const int within = 8 * (t & 3) + 2 * c + ei;  // index inside its 32-bit word
            // pages with values: plane mask bit i % 32; keys-only: record bit
            const int bit = planes ? within : 16 * (within >> 4) + 15 - (within & 15);
            const bool neg = (e < 2 ? n0 : n1) > 0.0f && pk[t][e] < 0.0f;
            if (neg) {
              if (e < 2) qw0[t >> 2] |= 1u << bit; else qw1[t >> 2] |= 1u << bit;
            }
          }
        }
#pragma unroll
        for (int w = 0; w < D / 32; ++w) {
          qw0[w] |= __shfl_xor_sync(0xffffffffu, qw0[w], 1);
          qw0[w] |= __shfl_xor_sync(0xffffffffu, qw0[w], 2);
          qw1[w] |= __shfl_xor_sync(0xffffffffu, qw1[w], 1);
          qw1[w] |= __shfl_xor_sync(0xffffffffu, qw1[w], 2);
          if (w == c) {
            reinterpret_cast<uint32_t*>(stg + C::STG_QS + r0 * (D / 8))[w] = qw0[w];
            reinterpret_cast<uint32_t*>(stg + C::STG_QS + r1 * (D / 8))[w] = qw1[w];
          }
        }
      } else {
        // values: 3-bit magnitude index against 7 thresholds, sign, nibble pairs
        float T0[7], T1[7];
#pragma unroll
        for (int k = 0; k < 7; ++k) {
          T0[k] = __fmul_rn(n0, p.vt[k]);
          T1[k] = __fmul_rn(n1, p.vt[k]);
        }
#pragma unroll
        for (int t = 0; t < C::NTL; ++t) {
          uint32_t packed = 0u;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x = acc[t][e];
            const bool row1 = e >= 2;
            const float nn = row1 ? n1 : n0;
            uint32_t mg = 0u;
#pragma unroll
            for (int k = 0; k < 7; ++k) mg += (fabsf(x) >= (row1 ? T1[k] : T0[k])) ? 1u : 0u;
            const uint32_t code = (nn > 0.0f) ? (((x < 0.0f) ? 8u : 0u) | mg) : 0u;
            packed |= code << (4 * e);  // (row g: e0, e1), (row g+8: e0, e1)
          }
          const uint32_t partner = __shfl_xor_sync(0xffffffffu, packed, 4);
          if ((g & 1) == 0) {
            const int j = 8 * t + 2 * c;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const int slot = (half ? r1 : r0);
              const int pair = slot >> 1;
              const uint32_t mine = (packed >> (8 * half)) & 0xFFu;   // codes (j, j+1), even slot
              const uint32_t other = (partner >> (8 * half)) & 0xFFu; // codes (j, j+1), odd slot
              stg[C::STG_VC + vc_pos<D>(j, pair)] = static_cast<uint8_t>((mine & 0xFu) | ((other & 0xFu) << 4));
              stg[C::STG_VC + vc_pos<D>(j + 1, pair)] = static_cast<uint8_t>((mine >> 4) | ((other >> 4) << 4));
            }
          }
        }
        if (c == 0) {
          reinterpret_cast<__half*>(stg + C::STG_VN)[r0] = nh0;
          reinterpret_cast<__half*>(stg + C::STG_VN)[r1] = nh1;
        }
      }
      __syncthreads();  // tile rows free for the next pass; staging complete after the last
    }

    // staging -> page, active slots [s_lo, s_hi) only
    uint8_t* pg = p.pool + static_cast<size_t>(page) * p.page_bytes;
    if (p.v) {  // block layout
      const uint32_t* mk = reinterpret_cast<const uint32_t*>(stg + C::STG_KC);
      key_planes_out<D>(mk, mk + ROWS * D / 32, reinterpret_cast<const uint32_t*>(stg + C::STG_QS), pg,
                        p.blk, p.off_kc, p.off_kl, p.off_qs, s_lo, s_hi, tid, blockDim.x);
      norms_out(reinterpret_cast<const uint16_t*>(stg + C::STG_KN),
                reinterpret_cast<const uint16_t*>(stg + C::STG_KG),
                reinterpret_cast<const uint16_t*>(stg + C::STG_VN), pg, p.blk, p.off_kn, p.off_vn,
                s_lo, s_hi, tid, blockDim.x);
      vc_copy_out<D>(stg + C::STG_VC, pg, p.blk, p.off_vc, s_lo, s_hi, tid, blockDim.x);
    } else {  // record layout
      constexpr int KC16 = D / 64;  // uint4 per key row
      for (int i = tid + s_lo * KC16; i < s_hi * KC16; i += blockDim.x)
        reinterpret_cast<uint4*>(pg + p.off_kc)[i] = reinterpret_cast<const uint4*>(stg + C::STG_KC)[i];
      if constexpr (D == 128) {
        for (int i = tid + s_lo; i < s_hi; i += blockDim.x)
          reinterpret_cast<uint4*>(pg + p.off_qs)[i] = reinterpret_cast<const uint4*>(stg + C::STG_QS)[i];
      } else {
        for (int i = tid + s_lo; i < s_hi; i += blockDim.x)
          reinterpret_cast<uint2*>(pg + p.off_qs)[i] = reinterpret_cast<const uint2*>(stg + C::STG_QS)[i];
      }
      for (int i = tid + s_lo; i < s_hi; i += blockDim.x) {
        reinterpret_cast<uint16_t*>(pg + p.off_kn)[i] = reinterpret_cast<const uint16_t*>(stg + C::STG_KN)[i];
        reinterpret_cast<uint16_t*>(pg + p.off_kg)[i] = reinterpret_cast<const uint16_t*>(stg + C::STG_KG)[i];
      }
    }
    __syncthreads();  // staging reused by the next tile
  }
}

__global__ void advance_kernel(int32_t* cold_len, int B, int n_new) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) cold_len[b] += n_new;
}

template <int D, int IN>
int run(const tq_ctx* ctx, Params& p, cudaStream_t st) {
  using C = Cfg<D>;
  static SmemAttr attr;
  if (!raise_smem_limit(compress_kernel<D, IN>, C::SMEM, attr)) return TQ_ERR_CUDA;
  const long long tiles = static_cast<long long>(p.B) * p.Hkv * p.tiles_per_bh;
  const int grid = static_cast<int>(tiles < ctx->num_sms ? tiles : ctx->num_sms);
  if (ctx->prof_start) cudaEventRecord(static_cast<cudaEvent_t>(ctx->prof_start), st);
  compress_kernel<D, IN><<<grid, NWARP * 32, C::SMEM, st>>>(p);
  if (ctx->prof_stop) cudaEventRecord(static_cast<cudaEvent_t>(ctx->prof_stop), st);
  advance_kernel<<<(p.B + 127) / 128, 128, 0, st>>>(const_cast<int32_t*>(p.cold_len), p.B, p.n_new);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace cmp

int launch_compress(const tq_ctx* ctx, const void* k, const void* v, tq_dtype dtype, int flags,
                    int B, int Hkv, int n_new, uint8_t* pool, int64_t pool_pages,
                    const int32_t* page_table, int max_pages, int32_t* cold_len, void* stream) {
  if (!(flags & TQ_INPUT_ROTATED))  // raw 16-bit input: rotation and sketch on tcgen05
    return launch_compress_tc(ctx, k, v, dtype == TQ_BF16, B, Hkv, n_new, pool, pool_pages,
                              page_table, max_pages, cold_len, stream);
  const int d = ctx->cfg.head_dim;
  const PageLayout L = page_layout(d, ctx->cfg.qjl_dim, v != nullptr);
  cmp::Params p{};
  p.k = k;
  p.v = v;
  p.B = B;
  p.Hkv = Hkv;
  p.n_new = n_new;
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
  const bool bf = (dtype == TQ_BF16);
  p.pi_hi = bf ? ctx->dev.rot_bf_hi : ctx->dev.rot_h_hi;
  p.pi_lo = bf ? ctx->dev.rot_bf_lo : ctx->dev.rot_h_lo;
  p.s_h = ctx->dev.qjl_h;
  p.kc0 = ctx->cb.key_c[0];
  p.kc1 = ctx->cb.key_c[1];
  p.kt0 = ctx->cb.key_t[0];
  for (int i = 0; i < 7; ++i) p.vt[i] = ctx->cb.val_t[i];
  p.err = ctx->dev.err;
  p.tiles_per_bh = (n_new + cmp::ROWS - 1) / cmp::ROWS + 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int in = (flags & TQ_INPUT_ROTATED) ? cmp::IN_ROT_F32 : (bf ? cmp::IN_BF16 : cmp::IN_F16);
  if (d == 128) {
    if (in == cmp::IN_F16) return cmp::run<128, cmp::IN_F16>(ctx, p, st);
    if (in == cmp::IN_BF16) return cmp::run<128, cmp::IN_BF16>(ctx, p, st);
    return cmp::run<128, cmp::IN_ROT_F32>(ctx, p, st);
  }
  if (d == 64) {
    if (in == cmp::IN_F16) return cmp::run<64, cmp::IN_F16>(ctx, p, st);
    if (in == cmp::IN_BF16) return cmp::run<64, cmp::IN_BF16>(ctx, p, st);
    return cmp::run<64, cmp::IN_ROT_F32>(ctx, p, st);
  }
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq
