// Device helpers for libtq kernels (sm_100a): mbarriers, 1-D bulk copies
// (TMA, no multicast), warp-level tensor-core MMA and byte permutes, and the
// device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "../../include/tq.h"

namespace tq {

// ---- error word: the first error recorded wins -------------------------
__device__ __forceinline__ void report(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// Range check of the debug build (compiled with TQ_DEBUG): true when
// 0 <= i < n; otherwise TQ_ERR_RANGE goes to the error word and the result
// is false, so that the caller skips the access (no trap, no assert).  In
// the release build it is the constant true.
#ifdef TQ_DEBUG
__device__ __forceinline__ bool in_range(int* err, long long i, long long n) {
  if (i >= 0 && i < n) return true;
  report(err, TQ_ERR_RANGE);
  return false;
}
#define TQ_IN_RANGE(err, i, n) \
  ::tq::in_range((err), static_cast<long long>(i), static_cast<long long>(n))
#else
#define TQ_IN_RANGE(err, i, n) true
#endif

// ---- shared-memory address ----------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// make mbarrier initialisation visible to the async (TMA) proxy
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// plain arrival (release semantics at CTA scope)
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of the barrier to complete, for at most
// `limit_ns` nanoseconds.  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint64_t limit_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0u && global_ns() - t0 > limit_ns) return false;
  }
}

// ---- 1-D bulk copy global -> shared, completing on an mbarrier ----------
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// order this thread's prior generic-proxy shared-memory accesses before
// subsequent async-proxy (bulk copy) accesses
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- byte permute -----------------------------------------------------------
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// ---- warp MMA m16n8k16, fp16 inputs, fp32 accumulate -----------------------
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

// fp16 hi/lo split of an fp32 value: hi = fp16(x), lo = fp16(x - hi)
// d = a * b + c on two fp16 lanes (round to nearest even)
__device__ __forceinline__ uint32_t hfma2_bits(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// key-plane value of two coordinates from a code word shifted so that their
// sign bits sit at 15 / 31 and magnitude bits at 13 / 29: the masked word is
// the fp16 pair +-m 2^-7, and one FMA gives +-(b + m (a - b)) exactly
// (d7 = fp16(2^7 (a - b)) chosen so; b2 = b in both halves)
__device__ __forceinline__ uint32_t key_plane_pair(uint32_t x, uint32_t d7, uint32_t b2) {
  return hfma2_bits(x & 0xA000A000u, d7, (x & 0x80008000u) | b2);
}

__device__ __forceinline__ void split_f16(float x, uint16_t& hi, uint16_t& lo) {
  __half h = __float2half_rn(x);
  hi = __half_as_ushort(h);
  lo = __half_as_ushort(__float2half_rn(x - __half2float(h)));
}

__device__ __forceinline__ float load_as_float(const void* p, size_t i, tq_dtype dt) {
  if (dt == TQ_F32) return static_cast<const float*>(p)[i];
  if (dt == TQ_F16) return __half2float(static_cast<const __half*>(p)[i]);
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

}  // namespace tq

namespace tq {

// ---------------------------------------------------------------------------
// Pages with values: 8 blocks of 16 token slots.  A block holds the key
// planes H and L (the key code is the index u = 2H + L of its level in
// ascending order), the QJL sign plane, the value codes, the (n, gamma) fp16
// pairs and the value norms; PageLayout gives the offsets inside a block.
// ---------------------------------------------------------------------------

// Byte, inside a block's plane, of plane index j (coordinate or sketch index)
// for token t (0..15); the bit is t % 8.  A 32-bit word holds 4 consecutive
// indices x 8 tokens; word w = 16 (j / 32) + 4 ((j / 4) % 4) + 2 ((j / 16) % 2)
// + t / 8, so that the four words a lane reads for indices 32k + 4c .. + 3 and
// 32k + 16 + 4c .. + 3 are adjacent.
__host__ __device__ __forceinline__ int plane_byte(int j, int t) {
  return 16 * (4 * (j >> 5) + ((j >> 2) & 3)) + 4 * (2 * ((j >> 4) & 1) + (t >> 3)) + (j & 3);
}

// Value-code section of a block: token pair p (tokens 2p, 2p+1 of the block)
// of coordinate j is one byte (even token in the low nibble).  Tiles of 16
// coordinates (i): the 32-bit word of lane 4g + c at (i/4)*512 + (4g + c)*16 +
// (i%4)*4 holds coordinates (g, g+8) x token pairs (c, c+4) -- one m16n8k16 A
// fragment (rows = coordinates, k = tokens) after dequantisation.  A staged
// page image holds the 8 blocks' sections back to back (vc_pos with the pair
// index of the page).
template <int D>
__host__ __device__ __forceinline__ int vc_pos(int j, int p) {
  const int kb = p >> 3, q = p & 7, c = q & 3, th = q >> 2;
  const int i = j >> 4, g = j & 7, jh = (j >> 3) & 1;
  return kb * (8 * D) + (i >> 2) * 512 + (4 * g + c) * 16 + (i & 3) * 4 + jh + 2 * th;
}

// Write the key planes H, L and the QJL plane (m = D) of the active slots
// [s_lo, s_hi) of a page with values, from per-slot masks staged in shared
// memory: mask[s * (D/32) + j/32] bit j % 32 is the plane bit of index j for
// slot s.  One 32-bit word (4 indices x 8 tokens) per thread and step; in a
// word with inactive tokens those tokens' bits keep their stored values.
template <int D>
__device__ __forceinline__ void key_planes_out(const uint32_t* mh, const uint32_t* ml,
                                               const uint32_t* mq, uint8_t* pg, int blk,
                                               int off_h, int off_l, int off_q, int s_lo,
                                               int s_hi, int tid, int nthr) {
  constexpr int WPB = D / 2;  // words per plane and block: D indices x 16 tokens / 32
  const int b_lo = s_lo >> 4, b_hi = (s_hi + 15) >> 4;
  const int n = (b_hi - b_lo) * 3 * WPB;
  for (int i = tid; i < n; i += nthr) {
    const int w = i % WPB, pl = (i / WPB) % 3, kb = b_lo + i / (3 * WPB);
    const int kap = w >> 4, c = (w >> 2) & 3, r = w & 3;
    const int s0 = 16 * kb + 8 * (r & 1);      // first slot of the word's 8 tokens
    const int shift = 16 * (r >> 1) + 4 * c;   // bit of its first index in the mask word
    const uint32_t* src = pl == 0 ? mh : pl == 1 ? ml : mq;
    uint32_t out = 0u, act = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int s = s0 + k;
      const uint32_t nib = (src[s * (D / 32) + kap] >> shift) & 0xFu;
      out |= ((nib * 0x00204081u) & 0x01010101u) << k;  // bit jj of nib -> bit 8 jj
      if (s >= s_lo && s < s_hi) act |= 1u << k;
    }
    if (act == 0u) continue;
    uint32_t* dst = reinterpret_cast<uint32_t*>(pg + kb * blk + (pl == 0 ? off_h : pl == 1 ? off_l : off_q) + 4 * w);
    if (act != 0xFFu) {
      const uint32_t m = act * 0x01010101u;
      out = (*dst & ~m) | (out & m);
    }
    *dst = out;
  }
}

// Norm fields of the active slots of a page with values: (n, gamma) pairs
// and (if vn) the value norms, from per-slot fp16 bits staged in shared memory.
__device__ __forceinline__ void norms_out(const uint16_t* kn, const uint16_t* kg,
                                          const uint16_t* vn, uint8_t* pg, int blk, int off_kn,
                                          int off_vn, int s_lo, int s_hi, int tid, int nthr) {
  for (int s = s_lo + tid; s < s_hi; s += nthr) {
    uint8_t* bk = pg + (s >> 4) * blk;
    const int t = s & 15;
    *reinterpret_cast<uint32_t*>(bk + off_kn + 4 * t) =
        static_cast<uint32_t>(kn[s]) | (static_cast<uint32_t>(kg[s]) << 16);
    if (vn) *reinterpret_cast<uint16_t*>(bk + off_vn + 2 * t) = vn[s];
  }
}

// Copy a staged value-code image (8 blocks of 8 D bytes, vc_pos layout) to the
// blocks of a page, for the active slots [s_lo, s_hi): 16-byte copies of the
// blocks wholly inside the range, byte copies (keeping the nibble of a pair's
// token outside the range) elsewhere.
template <int D>
__device__ __forceinline__ void vc_copy_out(const uint8_t* stg, uint8_t* pg, int blk, int off_vc,
                                            int s_lo, int s_hi, int tid, int nthr) {
  constexpr int BV = 8 * D;  // value bytes per block
  const int f_lo = (s_lo + 15) >> 4, f_hi = s_hi >> 4;  // whole blocks [f_lo, f_hi)
  for (int i = tid; i < (f_hi - f_lo) * (BV / 16); i += nthr) {
    const int kb = f_lo + i / (BV / 16), k = i % (BV / 16);
    reinterpret_cast<uint4*>(pg + kb * blk + off_vc)[k] = reinterpret_cast<const uint4*>(stg + kb * BV)[k];
  }
  // the partial blocks at either end
  for (int e = 0; e < 2; ++e) {
    const int kb = e == 0 ? (s_lo >> 4) : ((s_hi - 1) >> 4);
    if (kb >= f_lo && kb < f_hi) continue;
    if (e == 1 && kb == (s_lo >> 4)) continue;  // one partial block only
    const int a = max(s_lo, 16 * kb), z = min(s_hi, 16 * kb + 16);
    const int p_lo = a >> 1, p_hi = (z + 1) >> 1, np = p_hi - p_lo;
    for (int i = tid; i < D * np; i += nthr) {
      const int j = i / np, p = p_lo + i % np;
      const int off = vc_pos<D>(j, p);
      uint8_t* dst = pg + kb * blk + off_vc + (off - kb * BV);
      uint8_t b = stg[off];
      const bool ev = 2 * p >= s_lo && 2 * p < s_hi;
      const bool od = 2 * p + 1 >= s_lo && 2 * p + 1 < s_hi;
      if (!(ev && od)) {
        const uint8_t keep = ev ? 0xF0 : 0x0F;
        b = static_cast<uint8_t>((*dst & keep) | (b & ~keep));
      }
      *dst = b;
    }
  }
}

}  // namespace tq
