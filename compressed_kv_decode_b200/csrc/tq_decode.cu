// Decode attention over a hot fp16 window and cold compressed pages, one
// softmax over both ("Monarch v3: NES-inspiriertes KV-Paging", sections "Wie es
// funktioniert" and "Vereinfachte Decode-Schleife"); cold scores use the
// TurboQuant key estimator with the 1-bit QJL correction ("TurboQuant"
// summary, sections "Funktionsweise von TurboQuant" and "QJL: Eine 1-Bit-
// Methode ohne Overhead").
//
// Three launches:
//  1. prep      one CTA per (batch, kv head): q_rot = Pi q, q_s = S q_rot, the
//               constants of the estimator folded in, split into fixed-point
//               (cold) and fp16 hi/lo (hot) parts and laid out as the
//               tensor-core B fragments each lane needs (the cold ones only
//               when the call has cold pages); one extra CTA builds the work
//               schedule (units per segment, prefix sums, partial-record
//               slots).
//  2. attention persistent warps, each owning a contiguous range of work
//               units (64 cold tokens = 4 page blocks, or 13 hot tokens).  A
//               warp streams its units through a private ring of shared-memory
//               slots, one 1-D bulk copy (TMA) per cold unit and one per hot
//               row, completing on mbarriers.  Cold keys are scored with 8-bit integer MMAs
//               (m16n8k32; tokens on M, q heads x {hi, lo} of 16-bit
//               fixed-point query weights on N): the key planes H, L and the
//               QJL plane hold 8 tokens per byte, so a lane's operand is its
//               token's bit of every byte, one AND.  Values are dequantised
//               through a lane-replicated byte -> fp16 pair table in shared
//               memory (each address one byte dot product) straight into
//               m16n8k16 A fragments.  The warp keeps an online softmax,
//               accumulates P.V (cold values in the rotated domain) and
//               writes one partial (m, l, o) per segment it touched.
//  3. combine   per (batch, kv head): log-sum-exp merge of the cold partials,
//               o_cold = Pi^T o_rot, merge with the hot partials, divide.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace dec {

constexpr int NW = 12;        // warps per attention CTA
constexpr int COLD_TOK = 64;  // tokens per cold unit (4 blocks, half a page)
constexpr int HOT_TOK = 13;   // tokens per hot unit (K, V and a zero row fill a cold unit's slot)
constexpr float NEG_INF = -__builtin_huge_valf();

template <int D, int G>
struct Cfg {
  static constexpr int KS = D / 16;              // k-steps of a hot key row, coordinate tiles of a value
  static constexpr int NT = (2 * G + 7) / 8;     // score n-tiles: G heads x {hi, lo}
  static constexpr int KK = D / 32;              // int8 k-steps per cold plane (m = D)
  static constexpr int RC = 3 * KK * NT * 2;     // cold B-fragment registers per lane (planes H, L, QJL)
  static constexpr int RH = KS * NT * 2;         // hot B-fragment registers per lane
  // one 16-token block of a page with values (offsets as the page layout)
  static constexpr int OFF_H = 0, OFF_L = 2 * D, OFF_Q = 4 * D, OFF_V = 6 * D;
  static constexpr int OFF_NK = 14 * D, OFF_VN = 14 * D + 64;
  static constexpr int BLK = 14 * D + 96;
  static constexpr int COLD_B = 4 * BLK;          // one cold unit: 4 blocks, one copy
  static constexpr int HROW = 2 * D + 16;         // padded hot row: conflict-free ldmatrix
  static constexpr int HOT_B = 2 * HOT_TOK * HROW;
  static constexpr int SLOT = ((COLD_B > HOT_B ? COLD_B : HOT_B) + 127) / 128 * 128;
  static constexpr int NSLOT = (D == 128) ? 2 : 3;
  static constexpr int PBUF = COLD_TOK * 16;  // fp16 P' tile [64 tokens][8 heads]
  // one zero row (read for token rows past a hot unit), never written by copies
  static constexpr int OFF_ZERO = (NW * (NSLOT * SLOT + PBUF) + NW * NSLOT * 8 + NW * NSLOT * 4 + 15) / 16 * 16;
  static constexpr int SMEM = OFF_ZERO + HROW;
  static_assert(HOT_TOK <= 16 && HOT_B <= COLD_B, "a hot unit fills at most a cold unit's slot");
};

constexpr int DESC_N = 6;
enum { DS_UK = 0, DS_HOT = 1, DS_CK = 2, DS_UQ = 3, DS_CQ = 4 };
constexpr float FIX_MAX = 32511.0f;  // 16-bit fixed point whose hi byte stays within int8

struct Work {
  int* sched;         // [4 + 2 (S+1) + S]: U, unit_off, slot_off, seg_len
  uint32_t* frag_c;   // [BH][RC][32]
  uint32_t* frag_h;   // [BH][RH][32]
  float* desc;        // [BH][DESC_N][8] per head: key unit, hot descale, key constant,
                      // QJL unit, QJL constant (softmax scale folded in)
  float* part;        // [(Wtot + S)][G][D + 2]
  float* gmax;        // [BH][gate_nsplit][G] raw hot-score maxima per slot range (gated form)
  int* gmask;         // [BH] bit g set: q head g of the group reads its cold tokens
};

struct Params {
  const void* q;
  int q_dtype;
  int B, Hq, Hkv, max_pages, W_max;
  float sl;  // softmax scale * log2(e)
  const __half* k_hot;
  const __half* v_hot;
  const int32_t* hot_len;
  const int32_t* hot_start;  // [B] ring slot of the oldest hot token, or null (= 0)
  const uint8_t* pool;
  long long pool_pages;
  long long page_bytes;
  int blk;  // block bytes of a page with values (block layout)
  const int32_t* page_table;
  const int32_t* cold_len;
  float* out;
  const float* rot;
  const float* qjl;
  const float* sp;  // S Pi
  float kc0, kc1, alpha;       // key centroids, QJL constant sqrt(pi/2)/m
  float vc[8];
  int* err;
  Work w;
  int S;     // segments = 2 * B * Hkv
  int Wtot;  // attention warps
  // threshold gate: a q head reads its cold tokens only when its largest raw
  // hot score <q, k_t> is below gate_thr
  int gated;
  float gate_thr;
  int gate_nsplit;     // hot slot ranges of GATE_TOK slots
  int32_t* cold_used;  // [B, Hq] out (gated form), or null
  DecodeFuse fuse;     // combine epilogue (fuse.r null: none)
  // testing aid for the bounded waits: the cold unit whose copy is armed but
  // not issued (-1: none), and the bound of every wait of the attention
  int skip_unit;
  unsigned long long wait_ns;
  DecodePromo promo;  // Monarch's promotion (promo.logits null: none)
};

__device__ __forceinline__ int* unit_off(const Params& p) { return p.w.sched + 4; }
__device__ __forceinline__ int* slot_off(const Params& p) { return p.w.sched + 4 + p.S + 1; }
__device__ __forceinline__ int* seg_len(const Params& p) { return p.w.sched + 4 + 2 * (p.S + 1); }

// largest warp index whose range starts at or before unit u
__device__ __forceinline__ int warp_of(long long u, long long U, long long W) {
  return static_cast<int>(((u + 1) * W - 1) / U);
}

// Programmatic dependent launch: a kernel lets the next one in the stream be
// scheduled early (launch_dependents), and the next one waits for this one's
// completion and memory before touching its results (wait).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// slot of the ring holding the oldest hot token of sequence b (0 without a ring)
__device__ __forceinline__ int hot_start_of(const Params& p, int b) {
  if (!p.hot_start) return 0;
  const int s = p.hot_start[b];
  return (s >= 0 && s < p.W_max) ? s : 0;
}

// ---------------------------------------------------------------------------
// 0. threshold gate (gated form only)
// ---------------------------------------------------------------------------
constexpr int GATE_TOK = 256;   // hot slots per gate CTA
constexpr int GATE_TILES = 2;   // 16-slot tiles per warp (8 warps)

// bit g set: q head g of group bh reads its cold tokens (after the gate launch)
__device__ int gate_mask_of(const Params& p, int bh) {
  const int G = p.Hq / p.Hkv;
  int mask = 0;
  for (int g = 0; g < G; ++g) {
    float m = NEG_INF;
    for (int s = 0; s < p.gate_nsplit; ++s)
      m = fmaxf(m, p.w.gmax[(static_cast<size_t>(bh) * p.gate_nsplit + s) * G + g]);
    if (m < p.gate_thr) mask |= 1 << g;
  }
  return mask;
}

// ---------------------------------------------------------------------------
// 1. prep
// ---------------------------------------------------------------------------
__device__ int block_exclusive_scan(int v, int* scratch /* >= 32 ints */, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = (lane < nw) ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < nw) scratch[lane] = s;
  }
  __syncthreads();
  int before = (warp > 0) ? scratch[warp - 1] : 0;
  total = scratch[nw - 1];
  __syncthreads();
  return before + x - v;
}

__device__ void build_schedule(const Params& p) {
  __shared__ int scratch[32];
  __shared__ int carry_s;
  const int S = p.S;
  int* uoff = unit_off(p);
  int* soff = slot_off(p);
  int* slen = seg_len(p);
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int base = 0; base < S; base += blockDim.x) {
    const int sg = base + threadIdx.x;
    int units = 0;
    if (sg < S) {
      const int bh = sg >> 1, b = bh / p.Hkv;
      int len;
      if ((sg & 1) == 0) {
        len = p.cold_len ? p.cold_len[b] : 0;
        const int cap = p.max_pages * TQ_PAGE_TOKENS;
        if (len < 0 || len > cap) {
          report(p.err, TQ_ERR_CAPACITY);
          len = len < 0 ? 0 : cap;
        }
        if (p.gated) {
          const int mask = gate_mask_of(p, bh);
          p.w.gmask[bh] = mask;
          if (mask == 0) len = 0;  // no head of the group reads its cold tokens
        }
        units = (len + COLD_TOK - 1) / COLD_TOK;
      } else {
        len = p.hot_len ? p.hot_len[b] : 0;
        if (len < 0 || len > p.W_max) {
          report(p.err, TQ_ERR_CAPACITY);
          len = len < 0 ? 0 : p.W_max;
        }
        if (p.hot_start && p.W_max > 0 && (p.hot_start[b] < 0 || p.hot_start[b] >= p.W_max))
          report(p.err, TQ_ERR_CAPACITY);
        units = (len + HOT_TOK - 1) / HOT_TOK;
      }
      slen[sg] = len;
    }
    int total;
    const int ex = block_exclusive_scan(units, scratch, total);
    if (sg < S) uoff[sg] = carry_s + ex;
    __syncthreads();
    if (threadIdx.x == 0) carry_s += total;
    __syncthreads();
  }
  const int U = carry_s;
  // spread the units over min(Wtot, U) warps so that every one of them owns
  // at least one unit: the warps touching a segment are then consecutive and
  // each writes a partial record
  const int Weff = U < p.Wtot ? U : p.Wtot;
  if (threadIdx.x == 0) {
    uoff[S] = U;
    p.w.sched[0] = U;
    p.w.sched[1] = Weff;
  }
  __syncthreads();
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int base = 0; base < S; base += blockDim.x) {
    const int sg = base + threadIdx.x;
    int nwarps = 0;
    if (sg < S) {
      const int a = uoff[sg], e = uoff[sg + 1];
      if (e > a) nwarps = warp_of(e - 1, U, Weff) - warp_of(a, U, Weff) + 1;
    }
    int total;
    const int ex = block_exclusive_scan(nwarps, scratch, total);
    if (sg < S) soff[sg] = carry_s + ex;
    __syncthreads();
    if (threadIdx.x == 0) carry_s += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) soff[S] = carry_s;
}

__device__ __forceinline__ uint32_t pack_split(float xlo, float xhi, int part) {
  uint16_t h0, l0, h1, l1;
  split_f16(xlo, h0, l0);
  split_f16(xhi, h1, l1);
  return part == 0 ? (static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16))
                   : (static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16));
}

// scale factor 2^E putting max|w| in [128, 256): keeps the fp16 lo parts normal
__device__ __forceinline__ float prescale_for(float mx) {
  if (!(mx > 0.0f) || !isfinite(mx)) return 1.0f;
  int e;
  frexpf(mx, &e);  // mx = f * 2^e, f in [0.5, 1)
  return ldexpf(1.0f, 8 - e);
}

// y1[g][r] = sum_k M1[r][k] x[g][k] and y2 = M2 x, for all rows r of two
// D x D matrices.  Four lanes share a row: lane qq of the four takes the
// float4 chunks qq, qq + 4, ... of the row (coalesced row reads, conflict-free
// reads of x), so a row costs its FMAs plus a two-step shuffle reduction.
// Every row load of both matrices is issued at the start of the kernel,
// before the query is loaded (the rows do not depend on it).
constexpr int PREP_WARPS = 8;

template <int D>
struct MatRows {
  static constexpr int CH = D / 16;                     // float4 chunks per lane and row
  static constexpr int ROWS_PER_PASS = PREP_WARPS * 8;  // 8 rows per warp
  static constexpr int PASSES = D / ROWS_PER_PASS;
  float4 m[2][PASSES][CH];
};

// the lane's row chunks of both matrices, loaded before the query is ready
template <int D>
__device__ __forceinline__ void matvec_prefetch(const float* __restrict__ M1,
                                                const float* __restrict__ M2, MatRows<D>& mr) {
  using R = MatRows<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qq = lane & 3, rsub = lane >> 2;
#pragma unroll
  for (int w = 0; w < 2; ++w)
#pragma unroll
    for (int ps = 0; ps < R::PASSES; ++ps) {
      const int r = ps * R::ROWS_PER_PASS + warp * 8 + rsub;
      const float* M = w == 0 ? M1 : M2;
#pragma unroll
      for (int i = 0; i < R::CH; ++i)
        mr.m[w][ps][i] = __ldg(reinterpret_cast<const float4*>(M + static_cast<size_t>(r) * D) + qq + 4 * i);
    }
}

template <int D, int G>
__device__ __forceinline__ void matvec_rows2(const MatRows<D>& mr, const float (*x)[D],
                                             float (*y1)[D], float (*y2)[D]) {
  using R = MatRows<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qq = lane & 3, rsub = lane >> 2;
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    float (*y)[D] = w == 0 ? y1 : y2;
#pragma unroll
    for (int ps = 0; ps < R::PASSES; ++ps) {
      const int r = ps * R::ROWS_PER_PASS + warp * 8 + rsub;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float acc = 0.0f;
#pragma unroll
        for (int i = 0; i < R::CH; ++i) {
          const float4 xv = reinterpret_cast<const float4*>(x[g])[qq + 4 * i];
          const float4 mv = mr.m[w][ps][i];
          acc = fmaf(mv.x, xv.x, fmaf(mv.y, xv.y, fmaf(mv.z, xv.z, fmaf(mv.w, xv.w, acc))));
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (qq == 0) y[g][r] = acc;
      }
    }
  }
}

template <int D, int G>
__global__ void __launch_bounds__(256) prep_kernel(Params p) {
  using C = Cfg<D, G>;
  pdl_launch_dependents();
  const int BH = p.B * p.Hkv;
  if (blockIdx.x == BH) {
    if (p.gated) pdl_wait();  // the gate launch's maxima
    build_schedule(p);
    return;
  }
  const int bh = blockIdx.x, b = bh / p.Hkv, kvh = bh % p.Hkv;
  if (p.fuse.k_new) {  // the step's token into its ring slot (the attention waits for this launch)
    const int len = p.hot_len[b];
    if (len > 0 && len <= p.W_max) {
      int slot = hot_start_of(p, b) + len - 1;
      if (slot >= p.W_max) slot -= p.W_max;
      const size_t row = (static_cast<size_t>(bh) * p.W_max + slot) * D;
      const __half* kn = static_cast<const __half*>(p.fuse.k_new) + static_cast<size_t>(bh) * D;
      const __half* vn = static_cast<const __half*>(p.fuse.v_new) + static_cast<size_t>(bh) * D;
      for (int i = threadIdx.x; i < 2 * D; i += blockDim.x) {
        if (i < D) static_cast<__half*>(p.fuse.k_ring)[row + i] = kn[i];
        else static_cast<__half*>(p.fuse.v_ring)[row + i - D] = vn[i - D];
      }
    }
  }
  __shared__ __align__(16) float sq[G][D], sqr[G][D], sqs[G][D];
  __shared__ unsigned smax[2][G];
  __shared__ float sfac[2][G];
  const int tid = threadIdx.x;
  // without cold pages (a call over the hot window alone) only the hot
  // operands are needed: no rotation of the query
  const bool cold = p.max_pages > 0;
  MatRows<D> mr;
  if (cold) matvec_prefetch<D>(p.rot, p.sp, mr);  // Pi and S Pi rows do not wait for the query
  if (tid < 2 * G) smax[tid / G][tid % G] = 0u;
  for (int i = tid; i < G * D; i += blockDim.x) {
    const int g = i / D, j = i % D;
    sq[g][j] = load_as_float(p.q, (static_cast<size_t>(b) * p.Hq + kvh * G + g) * D + j,
                             static_cast<tq_dtype>(p.q_dtype));
  }
  __syncthreads();
  if (cold) matvec_rows2<D, G>(mr, sq, sqr, sqs);  // q_rot = Pi q, q_s = (S Pi) q
  __syncthreads();
  // Cold keys: three 0/1 operand planes against 16-bit fixed-point query
  // weights (int8 hi, lo).  The key code is the index u = 2H + L of its level
  // in ascending order (-c1, -c0, +c0, +c1), so the level is affine in the two
  // bits and the QJL term is affine in the sign bits b:
  //   <q_rot, c_hat> = -c1 sum(q_rot) + (c1 + c0) <q_rot, H> + (c1 - c0) <q_rot, L>
  //   <q_s, 1 - 2 b> = sum(q_s) - 2 <q_s, b>
  // One fixed-point unit per head for the two key planes, one for the QJL plane.
  const float wh = p.kc1 + p.kc0, wl = p.kc1 - p.kc0;
  __shared__ unsigned smr[G], sms[G];
  __shared__ float s_uk[G], s_uq[G];  // reciprocals of the fixed-point units
  if (tid < G) smr[tid] = sms[tid] = 0u;
  __syncthreads();
  // per-head maxima: the 32 lanes of a warp share one head (D >= 32), so a
  // warp reduction leaves one shared-memory atomic per warp and quantity
  for (int i = tid; i < G * D; i += blockDim.x) {
    const int g = i / D, j = i % D;
    float a = cold ? fabsf(sqr[g][j]) : 0.0f, c = cold ? fabsf(sqs[g][j]) : 0.0f;
    float e = fabsf(p.sl * sq[g][j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      c = fmaxf(c, __shfl_xor_sync(0xffffffffu, c, o));
      e = fmaxf(e, __shfl_xor_sync(0xffffffffu, e, o));
    }
    if ((tid & 31) == 0) {
      atomicMax(&smr[g], __float_as_uint(a));
      atomicMax(&sms[g], __float_as_uint(c));
      atomicMax(&smax[1][g], __float_as_uint(e));
    }
  }
  __syncthreads();
  {
    // per-head sums (one warp per head, fixed order)
    const int wp = tid >> 5, ln = tid & 31;
    if (wp < G) {
      float a = 0.0f, b2 = 0.0f;
      for (int j = ln; j < D && cold; j += 32) {
        a += sqr[wp][j];
        b2 += sqs[wp][j];
      }
      for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b2 += __shfl_xor_sync(0xffffffffu, b2, o);
      }
      if (ln == 0) {
        const float mr = __uint_as_float(smr[wp]), ms = __uint_as_float(sms[wp]);
        const float uk = mr > 0.0f ? wh * mr / FIX_MAX : 1.0f;
        const float uq = ms > 0.0f ? 2.0f * p.alpha * ms / FIX_MAX : 1.0f;
        s_uk[wp] = 1.0f / uk;
        s_uq[wp] = 1.0f / uq;
        float* ds = p.w.desc + static_cast<size_t>(bh) * DESC_N * 8;
        ds[DS_UK * 8 + wp] = p.sl * uk;
        ds[DS_CK * 8 + wp] = -p.sl * p.kc1 * a;
        ds[DS_UQ * 8 + wp] = p.sl * uq;
        ds[DS_CQ * 8 + wp] = p.sl * p.alpha * b2;
        const float f = prescale_for(__uint_as_float(smax[1][wp]));
        sfac[1][wp] = f;
        ds[DS_HOT * 8 + wp] = 1.0f / f;
      }
    }
  }
  __syncthreads();
  // cold fragments (m16n8k32, B = [k][n], 4 int8 of k per register):
  // r = ((plane * KK + kappa) * NT + nt) * 2 + reg, lane = 4 g' + c'; register
  // reg holds k = 4 c' + j + 16 reg (j = byte), index 32 kappa + k of the plane
  // (coordinate, or sketch index for the QJL plane), column n = g' = head
  // 4 nt + g' / 2, part g' % 2 (hi, lo).
  for (int idx = tid; idx < C::RC * 32 && cold; idx += blockDim.x) {
    const int r = idx >> 5, lane = idx & 31;
    const int reg = r & 1, nt = (r >> 1) % C::NT, pk = (r >> 1) / C::NT;
    const int plane = pk / C::KK, kap = pk % C::KK;
    const int gc = lane >> 2, cc = lane & 3;
    const int h = nt * 4 + (gc >> 1), part = gc & 1;
    uint32_t val = 0u;
    if (h < G) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = 32 * kap + 4 * cc + j + 16 * reg;
        const float qv = plane == 0 ? wh * sqr[h][k] * s_uk[h]
                       : plane == 1 ? wl * sqr[h][k] * s_uk[h]
                                    : -2.0f * p.alpha * sqs[h][k] * s_uq[h];
        const int q16 = max(-32511, min(32511, __float2int_rn(qv)));
        const int lo = ((q16 + 128) & 255) - 128, hi = (q16 - lo) >> 8;
        val |= static_cast<uint32_t>((part == 0 ? hi : lo) & 0xFF) << (8 * j);
      }
    }
    p.w.frag_c[(static_cast<size_t>(bh) * C::RC + r) * 32 + lane] = val;
  }
  // hot fragments: natural coordinate order, k = 16 s + 2 c' (+1), + 8 for reg 1
  for (int idx = tid; idx < C::RH * 32; idx += blockDim.x) {
    const int r = idx >> 5, lane = idx & 31;
    const int reg = r & 1, nt = (r >> 1) % C::NT, s = (r >> 1) / C::NT;
    const int gc = lane >> 2, cc = lane & 3;
    const int h = nt * 4 + (gc >> 1), part = gc & 1;
    uint32_t val = 0u;
    if (h < G) {
      const float wc = sfac[1][h] * p.sl;
      const int k0 = 16 * s + 2 * cc + 8 * reg;
      val = pack_split(wc * sq[h][k0], wc * sq[h][k0 + 1], part);
    }
    p.w.frag_h[(static_cast<size_t>(bh) * C::RH + r) * 32 + lane] = val;
  }
}

// ---------------------------------------------------------------------------
// 0. threshold gate (gated form only), launched before prep
// ---------------------------------------------------------------------------
// Largest raw hot score max_t <q_g, k_t> of each q head g of a (batch, kv
// head) group over one range of GATE_TOK ring slots (-inf where no slot of the
// range holds a token).  Each warp scores GATE_TILES tiles of 16 slots with m16n8k16
// MMAs: tokens on M, the group's heads x {hi, lo} fp16 parts of the
// prescaled query on N, fp32 accumulation.  The contraction order inside a
// k-step is free, so a lane's A fragment is two whole 16-byte chunks of its
// two rows (k-steps 2i and 2i+1 take the halves of chunk c + 4i) and the B
// fragment takes the query coordinates of the same chunks.
template <int D, int G>
__global__ void __launch_bounds__(256) gate_kernel(Params p) {
  pdl_launch_dependents();
  constexpr int NT = (2 * G + 7) / 8;  // n-tiles: G heads x {hi, lo}
  constexpr int NCH = D / 32;          // 16-byte chunks per lane and row
  const int split = blockIdx.x, bh = blockIdx.y, b = bh / p.Hkv, kvh = bh % p.Hkv;
  __shared__ __align__(16) float sq[G][D];
  __shared__ unsigned smx[G];
  __shared__ float sf[G];
  __shared__ float wmax[8][G];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, c = lane & 3;
  // the warp's tiles (tile tt covers 16 slots from (tt * 8 + warp) * 16); per
  // tile two rows per lane: row g and row g + 8 of the tile.  Every slot below
  // W_max is loaded before the lengths are known (slots without a token only
  // feed their own rows of the MMA and are masked).
  uint4 kr[GATE_TILES][2][NCH];
#pragma unroll
  for (int tt = 0; tt < GATE_TILES; ++tt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int slot = split * GATE_TOK + (tt * 8 + warp) * 16 + g + 8 * h;
      const uint4* row =
          reinterpret_cast<const uint4*>(p.k_hot + (static_cast<size_t>(bh) * p.W_max + slot) * D);
#pragma unroll
      for (int i = 0; i < NCH; ++i)
        kr[tt][h][i] = slot < p.W_max ? __ldg(row + c + 4 * i) : make_uint4(0u, 0u, 0u, 0u);
    }
  constexpr int QPT = (G * D + 255) / 256;  // query elements per thread
  float qv[QPT];
#pragma unroll
  for (int k = 0; k < QPT; ++k) {
    const int i = tid + 256 * k;
    qv[k] = i < G * D ? load_as_float(p.q, (static_cast<size_t>(b) * p.Hq + kvh * G) * D + i,
                                      static_cast<tq_dtype>(p.q_dtype))
                      : 0.0f;
  }
  int len = p.hot_len[b];
  len = len < 0 ? 0 : (len > p.W_max ? p.W_max : len);  // the schedule reports the error
  const int start = hot_start_of(p, b);
  bool valid[GATE_TILES][2];
#pragma unroll
  for (int tt = 0; tt < GATE_TILES; ++tt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int slot = split * GATE_TOK + (tt * 8 + warp) * 16 + g + 8 * h;
      int rel = slot - start;
      if (rel < 0) rel += p.W_max;
      valid[tt][h] = slot < p.W_max && rel < len;
    }
  if (tid < G) smx[tid] = 0u;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < QPT; ++k) {
    const int i = tid + 256 * k;
    if (i < G * D) {
      sq[i / D][i % D] = qv[k];
      atomicMax(&smx[i / D], __float_as_uint(fabsf(qv[k])));
    }
  }
  __syncthreads();
  if (tid < G) sf[tid] = prescale_for(__uint_as_float(smx[tid]));
  __syncthreads();
  // B fragments: column n = lane >> 2 of n-tile nt is head (8 nt + n) / 2, part n % 2
  uint32_t bfr[NCH][2][NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int n = 8 * nt + g, hh = n >> 1, part = n & 1;
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        const int d0 = 8 * (c + 4 * i) + 4 * hs;
        if (hh < G) {
          const float f = sf[hh];
          bfr[i][hs][nt][0] = pack_split(f * sq[hh][d0], f * sq[hh][d0 + 1], part);
          bfr[i][hs][nt][1] = pack_split(f * sq[hh][d0 + 2], f * sq[hh][d0 + 3], part);
        } else {
          bfr[i][hs][nt][0] = bfr[i][hs][nt][1] = 0u;
        }
      }
  }
  float mx[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) mx[nt] = NEG_INF;
#pragma unroll
  for (int tt = 0; tt < GATE_TILES; ++tt) {
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_f16(acc[nt], kr[tt][0][i].x, kr[tt][1][i].x, kr[tt][0][i].y, kr[tt][1][i].y,
                bfr[i][0][nt][0], bfr[i][0][nt][1]);
        mma_f16(acc[nt], kr[tt][0][i].z, kr[tt][1][i].z, kr[tt][0][i].w, kr[tt][1][i].w,
                bfr[i][1][nt][0], bfr[i][1][nt][1]);
      }
    // lane (g, c) holds, for head c + 4 nt, the hi and lo parts of rows g and g + 8
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (valid[tt][0]) mx[nt] = fmaxf(mx[nt], acc[nt][0] + acc[nt][1]);
      if (valid[tt][1]) mx[nt] = fmaxf(mx[nt], acc[nt][2] + acc[nt][3]);
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float m = mx[nt];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int hh = c + 4 * nt;
    if (g == 0 && hh < G) wmax[warp][hh] = m;
  }
  __syncthreads();
  if (tid < G) {
    float m = NEG_INF;
    for (int w = 0; w < 8; ++w) m = fmaxf(m, wmax[w][tid]);
    // undo the power-of-two prescale (exact)
    p.w.gmax[(static_cast<size_t>(bh) * p.gate_nsplit + split) * G + tid] = m / sf[tid];
  }
}

// ---------------------------------------------------------------------------
// 2. attention
// ---------------------------------------------------------------------------
template <int D, int G>
__device__ __forceinline__ void issue_unit(const Params& p, int u, int sg, int lu, int len, int page,
                                           uint8_t* dst, uint32_t bar, int lane) {
  using C = Cfg<D, G>;
  const int bh = sg >> 1;
  const uint32_t d0 = smem_u32(dst);
  if ((sg & 1) == 0) {
    // cold: blocks 4 (lu % 2) .. + 3 of the page, contiguous, one copy
    const bool ok = page >= 0 && page < p.pool_pages;
    if (lane == 0) {
      if (!ok) {
        report(p.err, TQ_ERR_CAPACITY);
        mbar_arrive_expect_tx(bar, 0);
      } else {
        mbar_arrive_expect_tx(bar, C::COLD_B);
        if (u != p.skip_unit)  // (testing aid: the skipped unit's wait runs out)
          bulk_g2s(d0, p.pool + static_cast<size_t>(page) * p.page_bytes + (lu & 1) * C::COLD_B,
                   C::COLD_B, bar);
      }
    }
    __syncwarp();
  } else {
    // hot: K rows then V rows of HOT_TOK ring slots, one row per lane
    const int t0 = lu * HOT_TOK;
    const int rows = min(HOT_TOK, len - t0);
    if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows) * 2u * (2u * D));
    __syncwarp();
    const int r = lane % HOT_TOK, isv = lane / HOT_TOK;
    if (lane < 2 * HOT_TOK && r < rows) {
      int slot = t0 + r + hot_start_of(p, bh / p.Hkv);
      if (slot >= p.W_max) slot -= p.W_max;
      const __half* src = (isv ? p.v_hot : p.k_hot) +
                          (static_cast<size_t>(bh) * p.W_max + slot) * D;
      bulk_g2s(d0 + isv * HOT_TOK * C::HROW + r * C::HROW, src, 2 * D, bar);
    }
  }
}

// d += a * b, m16n8k32, a unsigned 8-bit, b signed 8-bit, s32 accumulate
__device__ __forceinline__ void imma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Value dequantisation table: entry e (a code byte: two 4-bit codes, the even
// token's in the low nibble) = fp16 pair (v(e & 15), v(e >> 4)), v(code) =
// (-1)^(code >> 3) fp16(c[code & 7]).  32 copies, copy L in bank L: lane L
// reads entry e at byte 128 e + 4 L, so a warp's lookups never conflict.
__shared__ uint32_t g_vlut[256 * 32];

// 2^x by the hardware approximation; results below 2^-126 flush to zero,
// which a softmax weight next to its running maximum (weight 1) can take
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t vlut(const char* lut, uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(lut + off);
}

// PR: the promotion form (moved-back tokens masked, cold logits written).
template <int D, int G, bool PR>
__global__ void __launch_bounds__(NW * 32, 1) attn_kernel(Params p) {
  using C = Cfg<D, G>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  // value table (before waiting on the prep launch: it needs only the codebook)
  for (int i = threadIdx.x; i < 256 * 32; i += NW * 32) {
    const int e = i >> 5;
    const float v0 = ((e & 8) ? -1.0f : 1.0f) * p.vc[e & 7];
    const float v1 = ((e & 128) ? -1.0f : 1.0f) * p.vc[(e >> 4) & 7];
    const __half2 h2 = __floats2half2_rn(v0, v1);
    g_vlut[i] = *reinterpret_cast<const uint32_t*>(&h2);
  }
  for (int i = threadIdx.x; i < C::HROW / 4; i += NW * 32)
    reinterpret_cast<uint32_t*>(smem + C::OFF_ZERO)[i] = 0u;
  __syncthreads();
  pdl_wait();  // schedule and query operands come from the prep launch
  pdl_launch_dependents();
  uint8_t* slots = smem + warp * (C::NSLOT * C::SLOT);
  uint8_t* pbuf = smem + NW * C::NSLOT * C::SLOT + warp * C::PBUF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NW * (C::NSLOT * C::SLOT + C::PBUF)) +
                   warp * C::NSLOT;
  // page index of the unit staged in each slot (validity of cold pages)
  int* slot_page = reinterpret_cast<int*>(smem + NW * (C::NSLOT * C::SLOT + C::PBUF) + NW * C::NSLOT * 8) +
                   warp * C::NSLOT;

  const int* sched = p.w.sched;
  const int U = sched[0];
  const int* uoff = sched + 4;
  const int* soff = uoff + p.S + 1;
  const int* slen = soff + p.S + 1;
  const int Weff = sched[1];
  const int gw = blockIdx.x * NW + warp;
  if (U <= 0 || gw >= Weff) return;
  const int u0 = static_cast<int>(static_cast<long long>(gw) * U / Weff);
  const int u1 = static_cast<int>(static_cast<long long>(gw + 1) * U / Weff);
  if (u0 >= u1) return;

  if (lane < C::NSLOT) mbar_init(smem_u32(&bars[lane]), 1);
  mbar_init_fence();
  // P' tile: columns of absent heads stay zero
  for (int i = lane; i < C::PBUF / 4; i += 32) reinterpret_cast<uint32_t*>(pbuf)[i] = 0u;
  __syncwarp();

  // segment containing u0 (largest sg with uoff[sg] <= u0)
  int lo = 0, hi = p.S - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (uoff[mid] <= u0) lo = mid; else hi = mid - 1;
  }
  // issue cursor
  int isg = lo, ilu = u0 - uoff[lo], iend = uoff[lo + 1], ilen = slen[lo];
  int iu = u0;
  // the next unit to stage: located (and its page looked up) one unit ahead
  // of its copy, so the page-table load overlaps a unit of compute
  int nx_sg = 0, nx_lu = 0, nx_len = 0, nx_page = -1;
  auto prep_next = [&]() {
    while (iend <= iu) {  // segment ends and lengths are read once per segment
      ++isg;
      ilu = 0;
      iend = uoff[isg + 1];
      ilen = slen[isg];
    }
    nx_sg = isg;
    nx_lu = ilu;
    nx_len = ilen;
    nx_page = ((isg & 1) == 0) ? p.page_table[static_cast<size_t>(isg >> 1) * p.max_pages + (ilu >> 1)] : 0;
  };
  auto fire_next = [&](int slot) {
    if (lane == 0) slot_page[slot] = nx_page;
    issue_unit<D, G>(p, iu, nx_sg, nx_lu, nx_len, nx_page, slots + slot * C::SLOT,
                     smem_u32(&bars[slot]), lane);
    ++iu;
    ++ilu;
  };
  for (int s = 0; s < C::NSLOT && iu < u1; ++s) {
    prep_next();
    fire_next(s);
  }

  // consume cursor
  int sg = lo, lu = u0 - uoff[lo], send = uoff[lo + 1], len = slen[lo];
  uint32_t bfr[C::RC > C::RH ? C::RC : C::RH];
  float dsc[C::NT];                                   // hot: descale
  float uk[C::NT], ck[C::NT], uq[C::NT], cq[C::NT];  // cold: fixed-point units (row scale 2^-g folded in) and constants
  float mrun[C::NT], lrun[C::NT];
  float oacc[C::KS][4];
  const float rowscale = 1.0f / static_cast<float>(1 << g);  // operand bytes are bit << g
  auto load_segment = [&]() {
    const int bh = sg >> 1, dom = sg & 1;
    if (dom == 0) {
#pragma unroll
      for (int r = 0; r < C::RC; ++r)
        bfr[r] = p.w.frag_c[(static_cast<size_t>(bh) * C::RC + r) * 32 + lane];
    } else {
#pragma unroll
      for (int r = 0; r < C::RH; ++r)
        bfr[r] = p.w.frag_h[(static_cast<size_t>(bh) * C::RH + r) * 32 + lane];
    }
    const float* ds = p.w.desc + static_cast<size_t>(bh) * DESC_N * 8;
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) {
      const int h = c + 4 * nt;
      const bool in = h < G;
      dsc[nt] = in ? ds[DS_HOT * 8 + h] : 0.0f;
      uk[nt] = in ? ds[DS_UK * 8 + h] * rowscale : 0.0f;
      ck[nt] = in ? ds[DS_CK * 8 + h] : 0.0f;
      uq[nt] = in ? ds[DS_UQ * 8 + h] * rowscale : 0.0f;
      cq[nt] = in ? ds[DS_CQ * 8 + h] : 0.0f;
      mrun[nt] = NEG_INF;
      lrun[nt] = 0.0f;
    }
#pragma unroll
    for (int i = 0; i < C::KS; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.0f;
  };
  load_segment();

  // online-softmax update for scores sv (log2 domain); rescales oacc
  auto softmax_update = [&](float* sv, int count_per_nt) {
    float alpha[C::NT];
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) {
      float mx = NEG_INF;
      for (int i = 0; i < count_per_nt; ++i) mx = fmaxf(mx, sv[nt * count_per_nt + i]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float mnew = fmaxf(mrun[nt], mx);
      float ps = 0.0f;
      if (mnew == NEG_INF) {
        alpha[nt] = 1.0f;
        for (int i = 0; i < count_per_nt; ++i) sv[nt * count_per_nt + i] = 0.0f;
      } else {
        alpha[nt] = ex2_ftz(mrun[nt] - mnew);
        for (int i = 0; i < count_per_nt; ++i) {
          const float e = ex2_ftz(sv[nt * count_per_nt + i] - mnew);
          sv[nt * count_per_nt + i] = e;
          ps += e;
        }
      }
      mrun[nt] = mnew;
      lrun[nt] = lrun[nt] * alpha[nt] + ps;
    }
    // accumulator columns 2c, 2c+1 hold heads 2c and 2c+1
    const int hA = 2 * c, hB = 2 * c + 1;
    const int srcA = (lane & ~3) | (hA & 3), srcB = (lane & ~3) | (hB & 3);
    float aA = __shfl_sync(0xffffffffu, alpha[0], srcA);
    float aB = __shfl_sync(0xffffffffu, alpha[0], srcB);
    if (C::NT > 1) {
      const float a1A = __shfl_sync(0xffffffffu, alpha[C::NT > 1 ? 1 : 0], srcA);
      const float a1B = __shfl_sync(0xffffffffu, alpha[C::NT > 1 ? 1 : 0], srcB);
      if (hA >= 4) aA = a1A;
      if (hB >= 4) aB = a1B;
    }
    // the output only needs rescaling when some head's running max moved
    if (__any_sync(0xffffffffu, aA != 1.0f || aB != 1.0f)) {
#pragma unroll
      for (int i = 0; i < C::KS; ++i) {
        oacc[i][0] *= aA;
        oacc[i][1] *= aB;
        oacc[i][2] *= aA;
        oacc[i][3] *= aB;
      }
    }
  };

  auto flush_segment = [&]() {
    float lt[C::NT];
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) {
      float l = lrun[nt];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      lt[nt] = l;
    }
    const int first = warp_of(uoff[sg], U, Weff);
    if (!TQ_IN_RANGE(p.err, soff[sg] + (gw - first), p.Wtot + p.S)) return;  // partial record
    float* rec = p.w.part + static_cast<size_t>(soff[sg] + (gw - first)) * G * (D + 2);
    if (g == 0) {
#pragma unroll
      for (int nt = 0; nt < C::NT; ++nt) {
        const int h = c + 4 * nt;
        if (h < G) {
          rec[h] = mrun[nt];
          rec[G + h] = lt[nt];
        }
      }
    }
    float* o = rec + 2 * G;
#pragma unroll
    for (int i = 0; i < C::KS; ++i) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = 2 * c + (e & 1);
        const int coord = 16 * i + g + 8 * (e >> 1);
        if (h < G) o[h * D + coord] = oacc[i][e];
      }
    }
  };

  const uint32_t pb_addr = smem_u32(pbuf);
  const uint32_t zr_addr = smem_u32(smem + C::OFF_ZERO);
  const unsigned long long wait_ns = p.wait_ns ? p.wait_ns : 2000000000ull;
  const uint32_t msk = 0x01010101u << g;  // this lane's token in every plane byte
  const uint32_t l4 = static_cast<uint32_t>(lane) * 4u;
  const char* lut = reinterpret_cast<const char*>(g_vlut);
  for (int u = u0, k = 0; u < u1; ++u, ++k) {
    if (iu < u1) prep_next();
    const int slot = k % C::NSLOT;
    const uint32_t parity = static_cast<uint32_t>(k / C::NSLOT) & 1u;
    uint8_t* sb = slots + slot * C::SLOT;
    if (!mbar_wait_bounded(smem_u32(&bars[slot]), parity, wait_ns)) {
      if (lane == 0) report(p.err, TQ_ERR_TIMEOUT);
      // let copies already in flight land before the CTA can exit
      for (int s = 0; s < C::NSLOT; ++s)
        mbar_wait_bounded(smem_u32(&bars[s]), static_cast<uint32_t>((k + s) / C::NSLOT) & 1u, wait_ns);
      return;
    }
    if ((sg & 1) == 0) {
      // ---------------- cold unit: 64 tokens, 4 blocks ----------------
      const int page = slot_page[slot];
      const int nv = (page >= 0 && page < p.pool_pages) ? min(COLD_TOK, len - lu * COLD_TOK) : 0;
      // tokens of the unit that take part: inside the sequence and not moved
      // back to the hot window (Monarch's promotion)
      uint64_t valid = nv >= COLD_TOK ? ~0ull : (nv <= 0 ? 0ull : ((1ull << nv) - 1ull));
      int b_seq = 0;
      if constexpr (PR) {
        b_seq = (sg >> 1) / p.Hkv;
        const uint32_t* mw = p.promo.cold_mask + static_cast<size_t>(b_seq) * p.max_pages * 4 + 2 * lu;
        valid &= ~(static_cast<uint64_t>(mw[0]) | (static_cast<uint64_t>(mw[1]) << 32));
      }
      float sv[C::NT * 8];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const uint8_t* bp = sb + mt * C::BLK;
        // integer accumulators: key planes H and L (two chains, added
        // exactly at the end), and the QJL plane
        int ak[C::NT][4], al[C::NT][4], aq[C::NT][4];
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) ak[nt][e] = al[nt][e] = aq[nt][e] = 0;
#pragma unroll
        for (int kap = 0; kap < C::KK; ++kap) {
          // words for indices 32 kap + 4c .. (tokens 0-7, 8-15) and 32 kap + 16 + 4c ..
          const uint4 wh = *reinterpret_cast<const uint4*>(bp + C::OFF_H + (kap * 4 + c) * 16);
          const uint4 wl = *reinterpret_cast<const uint4*>(bp + C::OFF_L + (kap * 4 + c) * 16);
          const uint4 wq = *reinterpret_cast<const uint4*>(bp + C::OFF_Q + (kap * 4 + c) * 16);
#pragma unroll
          for (int nt = 0; nt < C::NT; ++nt) {
            const uint32_t* bH = bfr + ((0 * C::KK + kap) * C::NT + nt) * 2;
            const uint32_t* bL = bfr + ((1 * C::KK + kap) * C::NT + nt) * 2;
            const uint32_t* bQ = bfr + ((2 * C::KK + kap) * C::NT + nt) * 2;
            imma_u8s8(ak[nt], wh.x & msk, wh.y & msk, wh.z & msk, wh.w & msk, bH[0], bH[1]);
            imma_u8s8(al[nt], wl.x & msk, wl.y & msk, wl.z & msk, wl.w & msk, bL[0], bL[1]);
            imma_u8s8(aq[nt], wq.x & msk, wq.y & msk, wq.z & msk, wq.w & msk, bQ[0], bQ[1]);
          }
        }
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) ak[nt][e] += al[nt][e];
        // (n, gamma) of tokens g and g + 8 of the block
        const uint32_t nk0 = *reinterpret_cast<const uint32_t*>(bp + C::OFF_NK + 4 * g);
        const uint32_t nk1 = *reinterpret_cast<const uint32_t*>(bp + C::OFF_NK + 4 * (g + 8));
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&nk0));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&nk1));
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
          // columns 2c, 2c+1: the hi and lo bytes of head c's weights
          const float vk0 = static_cast<float>(ak[nt][0] * 256 + ak[nt][1]);
          const float vk1 = static_cast<float>(ak[nt][2] * 256 + ak[nt][3]);
          const float vq0 = static_cast<float>(aq[nt][0] * 256 + aq[nt][1]);
          const float vq1 = static_cast<float>(aq[nt][2] * 256 + aq[nt][3]);
          sv[nt * 8 + 2 * mt] = fmaf(f0.y, fmaf(uq[nt], vq0, cq[nt]), fmaf(uk[nt], vk0, ck[nt])) * f0.x;
          sv[nt * 8 + 2 * mt + 1] = fmaf(f1.y, fmaf(uq[nt], vq1, cq[nt]), fmaf(uk[nt], vk1, ck[nt])) * f1.x;
        }
        if (valid != ~0ull) {  // tokens past the sequence or moved back
          const int t0 = 16 * mt + g;
#pragma unroll
          for (int nt = 0; nt < C::NT; ++nt) {
            if (!((valid >> t0) & 1ull)) sv[nt * 8 + 2 * mt] = NEG_INF;
            if (!((valid >> (t0 + 8)) & 1ull)) sv[nt * 8 + 2 * mt + 1] = NEG_INF;
          }
        }
        if constexpr (PR) {  // every cold logit, for the promotion
          const int kvh = (sg >> 1) % p.Hkv, cap = p.max_pages * TQ_PAGE_TOKENS;
          const int pos = lu * COLD_TOK + 16 * mt + g;
#pragma unroll
          for (int nt = 0; nt < C::NT; ++nt) {
            const int h = c + 4 * nt;
            if (h < G) {
              float* lg = p.promo.logits + (static_cast<size_t>(b_seq) * p.Hq + kvh * G + h) * cap;
              if (TQ_IN_RANGE(p.err, pos + 8, cap)) {
                lg[pos] = sv[nt * 8 + 2 * mt];
                lg[pos + 8] = sv[nt * 8 + 2 * mt + 1];
              }
            }
          }
        }
      }
      softmax_update(sv, 8);
      // P' = p * n_v as fp16 into the [64 tokens][8 heads] tile
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const int t0 = 16 * mt + g, t1 = t0 + 8;
        const __half* vn = reinterpret_cast<const __half*>(sb + mt * C::BLK + C::OFF_VN);
        const float nv0 = __half2float(vn[g]), nv1 = __half2float(vn[g + 8]);
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
          const int h = c + 4 * nt;
          if (h < G) {
            float p0 = sv[nt * 8 + 2 * mt] * nv0, p1 = sv[nt * 8 + 2 * mt + 1] * nv1;
            if (valid != ~0ull) {
              if (!((valid >> t0) & 1ull)) p0 = 0.0f;
              if (!((valid >> t1) & 1ull)) p1 = 0.0f;
            }
            reinterpret_cast<__half*>(pbuf)[t0 * 8 + h] = __float2half_rn(p0);
            reinterpret_cast<__half*>(pbuf)[t1 * 8 + h] = __float2half_rn(p1);
          }
        }
      }
      __syncwarp();
      // value codes: the lane's word for coordinate tile i of a block
      // dequantises, byte by byte through the table, to its A fragment
      // (coordinates x tokens)
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        uint32_t bp0, bp1;
        ldsm_x2_t(pb_addr + (16 * mt + (lane & 15)) * 16, bp0, bp1);
        const uint8_t* vb = sb + mt * C::BLK + C::OFF_V + lane * 16;
        uint32_t xw[C::KS];
#pragma unroll
        for (int q4 = 0; q4 < C::KS / 4; ++q4) {
          const uint4 v = *reinterpret_cast<const uint4*>(vb + 512 * q4);
          xw[4 * q4] = v.x; xw[4 * q4 + 1] = v.y; xw[4 * q4 + 2] = v.z; xw[4 * q4 + 3] = v.w;
        }
        // table address of code byte j: 128 * byte + 4 lane, one 4-way byte
        // dot product with a weight of 128 on byte j (sum < 2^15, exact)
#pragma unroll
        for (int i = 0; i < C::KS; ++i) {
          const uint32_t x = xw[i];
          const uint32_t a0 = vlut(lut, __dp4a(x, 0x00000080u, l4));
          const uint32_t a1 = vlut(lut, __dp4a(x, 0x00008000u, l4));
          const uint32_t a2 = vlut(lut, __dp4a(x, 0x00800000u, l4));
          const uint32_t a3 = vlut(lut, __dp4a(x, 0x80000000u, l4));
          mma_f16(oacc[i], a0, a1, a2, a3, bp0, bp1);
        }
      }
    } else {
      // ---------------- hot unit: HOT_TOK tokens ----------------
      // K rows then V rows; the MMAs read 16 token rows, and rows at or past
      // nv (not copied, or past the unit) read the CTA's zero row
      const int nv = min(HOT_TOK, len - lu * HOT_TOK);
      const uint32_t kt_addr = smem_u32(sb), vt_addr = kt_addr + HOT_TOK * C::HROW;
      // scores: tokens on M; rows at or past nv are masked
      // (two accumulator chains, even and odd k-steps, summed at the end)
      float acc[C::NT][4], acc2[C::NT][4];
#pragma unroll
      for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = acc2[nt][e] = 0.0f;
      const int krow = (lane & 7) + ((lane >> 3) & 1) * 8;
      const uint32_t krow_addr = krow < nv ? kt_addr + krow * C::HROW : zr_addr;
#pragma unroll
      for (int s = 0; s < C::KS; ++s) {
        const int col = 16 * s + (lane >> 4) * 8;
        uint32_t a0, a1, a2, a3;
        ldsm_x4(krow_addr + col * 2, a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
          const uint32_t b0 = bfr[(s * C::NT + nt) * 2], b1 = bfr[(s * C::NT + nt) * 2 + 1];
          if (s & 1) mma_f16(acc2[nt], a0, a1, a2, a3, b0, b1);
          else mma_f16(acc[nt], a0, a1, a2, a3, b0, b1);
        }
      }
#pragma unroll
      for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] += acc2[nt][e];
      // accumulator columns 2c, 2c + 1: the hi and lo parts of head c
      float sv[C::NT * 2];
#pragma unroll
      for (int nt = 0; nt < C::NT; ++nt) {
        sv[nt * 2] = (g < nv) ? (acc[nt][0] + acc[nt][1]) * dsc[nt] : NEG_INF;
        sv[nt * 2 + 1] = (g + 8 < nv) ? (acc[nt][2] + acc[nt][3]) * dsc[nt] : NEG_INF;
      }
      softmax_update(sv, 2);
#pragma unroll
      for (int nt = 0; nt < C::NT; ++nt) {
        const int h = c + 4 * nt;
        if (h < G) {
          reinterpret_cast<__half*>(pbuf)[g * 8 + h] = __float2half_rn(sv[nt * 2]);
          reinterpret_cast<__half*>(pbuf)[(g + 8) * 8 + h] = __float2half_rn(sv[nt * 2 + 1]);
        }
      }
      __syncwarp();
      // P V over 16 token rows: A = V^T (coordinates x tokens) by transposed
      // loads of the V rows, B = the P' tile
      uint32_t bp0, bp1;
      ldsm_x2_t(pb_addr + (lane & 15) * 16, bp0, bp1);
      const int vrow = (lane & 7) + ((lane >> 4) & 1) * 8;
      const uint32_t vrow_addr = vrow < nv ? vt_addr + vrow * C::HROW : zr_addr;
#pragma unroll
      for (int i = 0; i < C::KS; ++i) {
        const int col = 16 * i + ((lane >> 3) & 1) * 8;
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(vrow_addr + col * 2, a0, a1, a2, a3);
        mma_f16(oacc[i], a0, a1, a2, a3, bp0, bp1);
      }
    }
    // all lanes are done with this slot (every value read from it has been
    // consumed): refill it
    __syncwarp();
    if (iu < u1) fire_next(slot);
    ++lu;
    if (u + 1 == u1 || u + 1 >= send) {
      flush_segment();
      if (u + 1 < u1) {
        ++sg;
        while (uoff[sg + 1] <= u + 1) ++sg;
        send = uoff[sg + 1];
        len = slen[sg];
        lu = 0;
        load_segment();
      }
    }
  }
}

// ---------------------------------------------------------------------------
// 3. combine
// ---------------------------------------------------------------------------
constexpr int COMB_THREADS = 256;
constexpr int COMB_CHUNK = 256;  // records whose weights are staged in shared memory at once

// Shared memory of the combine kernel: Pi, the staged record weights, and the
// per-slice output sums.
template <int D, int G>
struct CombCfg {
  static constexpr int NSL = COMB_THREADS / D;  // record slices
  static constexpr int OFF_W = D * D * 4;
  static constexpr int OFF_S = OFF_W + COMB_CHUNK * G * 4;
  static constexpr int SMEM = OFF_S + NSL * 2 * G * D * 4;
};

// max (op 0) or sum (op 1) of v over the threads that share thread index mod G
template <int G>
__device__ __forceinline__ float group_reduce(float v, float (*red)[G], int op) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int o = G; o < 32; o <<= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = op == 0 ? fmaxf(v, w) : v + w;
  }
  __syncthreads();
  if (lane < G) red[warp][lane] = v;
  __syncthreads();
  float r = red[0][tid % G];
  for (int w = 1; w < COMB_THREADS / 32; ++w) r = op == 0 ? fmaxf(r, red[w][tid % G]) : r + red[w][tid % G];
  return r;
}

// Per (batch, kv head): log-sum-exp merge of the group's partial records
// (cold records hold rotated-domain outputs), o_cold = Pi^T o_rot, merge of
// cold and hot, division by the softmax denominator.  Three passes over the
// records: per-head maxima; softmax weights (staged in shared memory, one
// chunk at a time); weighted outputs, NSL slices of records accumulated in
// parallel with many loads in flight.
template <int D, int G>
__global__ void __launch_bounds__(COMB_THREADS) combine_kernel(Params p) {
  using CC = CombCfg<D, G>;
  constexpr int NSL = CC::NSL;
  constexpr int RB = G * (D + 2);  // floats per record
  constexpr float NINF = -__builtin_huge_valf();
  const int bh = blockIdx.x, b = bh / p.Hkv, kvh = bh % p.Hkv;
  const int tid = threadIdx.x, sl = tid / D, j = tid % D;
  extern __shared__ __align__(16) uint8_t csm[];
  float* spi = reinterpret_cast<float*>(csm);               // [D][D]
  float* wts = reinterpret_cast<float*>(csm + CC::OFF_W);   // [COMB_CHUNK][G]
  float* ssum = reinterpret_cast<float*>(csm + CC::OFF_S);  // [NSL][2][G][D]
  __shared__ float red[COMB_THREADS / 32][G];
  __shared__ float sM[2][G], sL[2][G];
  // Pi does not depend on the attention launch: stage it first, overlapping
  // the tail of that launch (a call without cold pages has no rotated sums)
  const bool cold = p.max_pages > 0;
  if (cold) {
    constexpr int PER = D * D / 4 / COMB_THREADS;
#pragma unroll
    for (int i = 0; i < PER; ++i)
      reinterpret_cast<float4*>(spi)[i * COMB_THREADS + tid] =
          __ldg(reinterpret_cast<const float4*>(p.rot) + i * COMB_THREADS + tid);
  }
  pdl_wait();  // partial records come from the attention launch
  const int* soff = p.w.sched + 4 + p.S + 1;
  const int a0 = soff[2 * bh], a1 = soff[2 * bh + 1], e1 = soff[2 * bh + 2];
  const int R = e1 - a0;
  const float* part = p.w.part;
  // pass 1: per (domain, head) maxima over records that hold tokens; the
  // thread's head is tid % G throughout (COMB_THREADS is a multiple of G)
  const int hg = tid % G;
  float mx0 = NINF, mx1 = NINF;
  for (int i = tid; i < R * G; i += COMB_THREADS) {
    const int r = a0 + i / G;
    const float* rec = part + static_cast<size_t>(r) * RB;
    const float m = rec[hg], l = rec[G + hg];
    if (l > 0.0f) {
      if (r < a1) mx0 = fmaxf(mx0, m);
      else mx1 = fmaxf(mx1, m);
    }
  }
  mx0 = group_reduce<G>(mx0, red, 0);
  mx1 = group_reduce<G>(mx1, red, 0);
  if (tid < G) {
    sM[0][tid] = mx0;
    sM[1][tid] = mx1;
  }
  float O[2][G];
#pragma unroll
  for (int d2 = 0; d2 < 2; ++d2)
#pragma unroll
    for (int g = 0; g < G; ++g) O[d2][g] = 0.0f;
  float l0 = 0.0f, l1 = 0.0f;
  for (int base = 0; base < R; base += COMB_CHUNK) {
    const int n = min(COMB_CHUNK, R - base);
    __syncthreads();
    // pass 2: weights exp2(m - M) of this chunk, and the denominators
    for (int i = tid; i < n * G; i += COMB_THREADS) {
      const int r = a0 + base + i / G;
      const float* rec = part + static_cast<size_t>(r) * RB;
      const float m = rec[hg], l = rec[G + hg];
      const float M = r < a1 ? mx0 : mx1;
      const float w = (l > 0.0f) ? exp2f(m - M) : 0.0f;
      wts[i] = w;
      if (r < a1) l0 += l * w;
      else l1 += l * w;
    }
    __syncthreads();
    // pass 3: weighted outputs; slice sl takes records sl, sl + NSL, ...
    int r = sl;
    for (; r + 3 * NSL < n; r += 4 * NSL) {
      float ov[4][G];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int g = 0; g < G; ++g)
          ov[u][g] = part[static_cast<size_t>(a0 + base + r + u * NSL) * RB + 2 * G + g * D + j];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int rr = r + u * NSL;
        const int dom = (a0 + base + rr) < a1 ? 0 : 1;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float w = wts[rr * G + g] * ov[u][g];
          if (dom == 0) O[0][g] += w;
          else O[1][g] += w;
        }
      }
    }
    for (; r < n; r += NSL) {
      const int dom = (a0 + base + r) < a1 ? 0 : 1;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float w = wts[r * G + g] * part[static_cast<size_t>(a0 + base + r) * RB + 2 * G + g * D + j];
        if (dom == 0) O[0][g] += w;
        else O[1][g] += w;
      }
    }
  }
  l0 = group_reduce<G>(l0, red, 1);
  l1 = group_reduce<G>(l1, red, 1);
  if (tid < G) {
    sL[0][tid] = l0;
    sL[1][tid] = l1;
  }
#pragma unroll
  for (int d2 = 0; d2 < 2; ++d2)
#pragma unroll
    for (int g = 0; g < G; ++g) ssum[((sl * 2 + d2) * G + g) * D + j] = O[d2][g];
  __syncthreads();
  // slice sums; the cold one back into slice 0's rows for the rotation
  if (sl == 0) {
#pragma unroll
    for (int d2 = 0; d2 < 2; ++d2)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float s = O[d2][g];
#pragma unroll
        for (int k = 1; k < NSL; ++k) s += ssum[((k * 2 + d2) * G + g) * D + j];
        ssum[(d2 * G + g) * D + j] = s;
      }
  }
  __syncthreads();
  int mask = (1 << G) - 1;
  if (p.gated) mask = p.w.gmask[bh];
  // o_cold = Pi^T o_rot; thread (sl, j) takes heads g = sl, sl + NSL, ...
  for (int g = sl; g < G; g += NSL) {
    const float* so = ssum + g * D;  // cold sums (domain 0)
    float oc = 0.0f;
    if (cold) {  // four partial sums: a quarter of the dependent chain each
      float o4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 16
      for (int i = 0; i < D; i += 4)
#pragma unroll
        for (int k = 0; k < 4; ++k) o4[k] = fmaf(spi[(i + k) * D + j], so[i + k], o4[k]);
      oc = (o4[0] + o4[1]) + (o4[2] + o4[3]);
    }
    const float oh = ssum[(G + g) * D + j];
    const bool open = (mask >> g) & 1;
    const float Mc = sM[0][g], Mh = sM[1][g];
    const float Lc = open ? sL[0][g] : 0.0f, Lh = sL[1][g];
    const float Mx = fmaxf(Lc > 0.0f ? Mc : NINF, Lh > 0.0f ? Mh : NINF);
    float res = 0.0f;
    if (Mx != NINF) {
      const float fc = (Lc > 0.0f) ? exp2f(Mc - Mx) : 0.0f;
      const float fh = (Lh > 0.0f) ? exp2f(Mh - Mx) : 0.0f;
      const float den = Lc * fc + Lh * fh;
      res = (den > 0.0f) ? ((fc > 0.0f ? oc * fc : 0.0f) + (fh > 0.0f ? oh * fh : 0.0f)) / den : 0.0f;
    }
    const size_t oi = (static_cast<size_t>(b) * p.Hq + kvh * G + g) * D + j;
    if (p.promo.lse && j == 0) {  // log-sum-exp of the head's attended tokens (promotion)
      const float den = (Mx != NINF) ? Lc * ((Lc > 0.0f) ? exp2f(Mc - Mx) : 0.0f) +
                                           Lh * ((Lh > 0.0f) ? exp2f(Mh - Mx) : 0.0f)
                                     : 0.0f;
      p.promo.lse[static_cast<size_t>(b) * p.Hq + kvh * G + g] =
          (open && den > 0.0f) ? Mx + log2f(den) : __builtin_huge_valf();
    }
    if (p.fuse.r) {  // out += sigmoid(gate) r
      const float sg = 1.0f / (1.0f + expf(-p.fuse.gate[kvh * G + g]));
      res = fmaf(sg, p.fuse.r[oi], res);
    }
    if (TQ_IN_RANGE(p.err, oi, static_cast<long long>(p.B) * p.Hq * D)) p.out[oi] = res;
    if (j == 0 && p.gated && p.cold_used)
      p.cold_used[static_cast<size_t>(b) * p.Hq + kvh * G + g] = open;
  }
  if (p.fuse.r && kvh == 0 && tid == 0) {
    p.fuse.dst_start[b] = p.fuse.src_start[b];
    p.fuse.dst_len[b] = p.fuse.src_len[b];
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct WsLayout {
  size_t sched, frag_c, frag_h, desc, part, gmax, gmask, total;
};

inline int gate_splits(int W_max) { return (W_max + GATE_TOK - 1) / GATE_TOK; }

template <int D, int G>
WsLayout ws_layout(int B, int Hkv, int Wtot, int W_max) {
  using C = Cfg<D, G>;
  const size_t BH = static_cast<size_t>(B) * Hkv, S = 2 * BH;
  WsLayout L;
  size_t off = 0;
  L.sched = off;
  off = align256(off + sizeof(int) * (4 + 2 * (S + 1) + S));
  L.frag_c = off;
  off = align256(off + sizeof(uint32_t) * BH * C::RC * 32);
  L.frag_h = off;
  off = align256(off + sizeof(uint32_t) * BH * C::RH * 32);
  L.desc = off;
  off = align256(off + sizeof(float) * BH * DESC_N * 8);
  L.part = off;
  off = align256(off + sizeof(float) * (static_cast<size_t>(Wtot) + S) * G * (D + 2));
  L.gmax = off;
  off = align256(off + sizeof(float) * BH * gate_splits(W_max) * G);
  L.gmask = off;
  off = align256(off + sizeof(int) * BH);
  L.total = off;
  return L;
}

template <int D, int G>
int run(const tq_ctx* ctx, Params& p, void* ws, size_t ws_bytes, cudaStream_t st) {
  using C = Cfg<D, G>;
  if (p.blk != C::BLK || p.page_bytes != 8LL * C::BLK) return TQ_ERR_UNSUPPORTED;  // block layout
  const int grid = ctx->num_sms;
  p.Wtot = grid * NW;
  p.S = 2 * p.B * p.Hkv;
  const WsLayout L = ws_layout<D, G>(p.B, p.Hkv, p.Wtot, p.W_max);
  if (ws_bytes < L.total) return TQ_ERR_INVALID_ARG;
  uint8_t* base = static_cast<uint8_t*>(ws);
  p.w.sched = reinterpret_cast<int*>(base + L.sched);
  p.w.frag_c = reinterpret_cast<uint32_t*>(base + L.frag_c);
  p.w.frag_h = reinterpret_cast<uint32_t*>(base + L.frag_h);
  p.w.desc = reinterpret_cast<float*>(base + L.desc);
  p.w.part = reinterpret_cast<float*>(base + L.part);
  p.w.gmax = reinterpret_cast<float*>(base + L.gmax);
  p.w.gmask = reinterpret_cast<int*>(base + L.gmask);
  p.gate_nsplit = gate_splits(p.W_max);
  static SmemAttr attn_attr, attn_attr_pr;
  auto attn = p.promo.logits ? attn_kernel<D, G, true> : attn_kernel<D, G, false>;
  if (!raise_smem_limit(attn, C::SMEM, p.promo.logits ? attn_attr_pr : attn_attr))
    return TQ_ERR_CUDA;
  if (p.gated && p.gate_nsplit > 0) {
    // gate, then prep overlapping it: only prep's schedule CTA waits for the maxima
    gate_kernel<D, G><<<dim3(p.gate_nsplit, p.B * p.Hkv), 256, 0, st>>>(p);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.B * p.Hkv + 1);
    cfg.blockDim = dim3(PREP_WARPS * 32);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, prep_kernel<D, G>, p) != cudaSuccess) return TQ_ERR_CUDA;
  } else {
    prep_kernel<D, G><<<p.B * p.Hkv + 1, PREP_WARPS * 32, 0, st>>>(p);
  }
  if (ctx->prof_start) cudaEventRecord(static_cast<cudaEvent_t>(ctx->prof_start), st);
  {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NW * 32);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, attn, p) != cudaSuccess) return TQ_ERR_CUDA;
  }
  if (ctx->prof_stop) cudaEventRecord(static_cast<cudaEvent_t>(ctx->prof_stop), st);
  static SmemAttr comb_attr;
  if (!raise_smem_limit(combine_kernel<D, G>, CombCfg<D, G>::SMEM, comb_attr)) return TQ_ERR_CUDA;
  {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.B * p.Hkv);
    cfg.blockDim = dim3(COMB_THREADS);
    cfg.dynamicSmemBytes = CombCfg<D, G>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, combine_kernel<D, G>, p) != cudaSuccess) return TQ_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace dec

size_t decode_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_pages, int W_max) {
  (void)max_pages;
  if (B <= 0 || Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0) return 0;
  const int G = Hq / Hkv;
  const int Wtot = ctx->num_sms * dec::NW;
  // the largest layout over the supported group sizes of this head dim
  size_t best = 0;
  auto take = [&](size_t v) { best = v > best ? v : best; };
  if (ctx->cfg.head_dim == 128) {
    if (G == 1) take(dec::ws_layout<128, 1>(B, Hkv, Wtot, W_max).total);
    if (G == 2) take(dec::ws_layout<128, 2>(B, Hkv, Wtot, W_max).total);
    if (G == 4) take(dec::ws_layout<128, 4>(B, Hkv, Wtot, W_max).total);
    if (G == 8) take(dec::ws_layout<128, 8>(B, Hkv, Wtot, W_max).total);
  } else {
    if (G == 1) take(dec::ws_layout<64, 1>(B, Hkv, Wtot, W_max).total);
    if (G == 2) take(dec::ws_layout<64, 2>(B, Hkv, Wtot, W_max).total);
    if (G == 4) take(dec::ws_layout<64, 4>(B, Hkv, Wtot, W_max).total);
    if (G == 8) take(dec::ws_layout<64, 8>(B, Hkv, Wtot, W_max).total);
  }
  return best;
}

int launch_decode(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq, int Hkv,
                  float scale, const void* k_hot, const void* v_hot, int W_max,
                  const int32_t* hot_start, const int32_t* hot_len, const uint8_t* pool,
                  int64_t pool_pages, const int32_t* page_table, int max_pages,
                  const int32_t* cold_len, const DecodeGate* gate, float* out, void* ws,
                  size_t ws_bytes, void* stream, const DecodeFuse* fuse,
                  const DecodePromo* promo) {
  const int d = ctx->cfg.head_dim;
  const int G = Hq / Hkv;
  const PageLayout L = page_layout(d, ctx->cfg.qjl_dim, true);
  dec::Params p{};
  p.q = q;
  p.q_dtype = static_cast<int>(q_dtype);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.max_pages = max_pages;
  p.W_max = W_max;
  const float sc = (scale == 0.0f) ? 1.0f / std::sqrt(static_cast<float>(d)) : scale;
  p.sl = sc * 1.4426950408889634f;
  p.k_hot = static_cast<const __half*>(k_hot);
  p.v_hot = static_cast<const __half*>(v_hot);
  p.hot_len = hot_len;
  p.hot_start = hot_start;
  if (fuse) p.fuse = *fuse;
  if (promo) p.promo = *promo;
  if (gate) {
    p.gated = 1;
    p.gate_thr = gate->threshold;
    p.cold_used = gate->cold_used;
  }
  p.pool = pool;
  p.pool_pages = pool_pages;
  p.page_bytes = static_cast<long long>(L.bytes);
  p.blk = static_cast<int>(L.block);
  p.page_table = page_table;
  p.cold_len = cold_len;
  p.out = out;
  p.rot = ctx->dev.rot;
  p.qjl = ctx->dev.qjl;
  p.sp = ctx->dev.sp;
  p.kc0 = ctx->cb.key_c[0];
  p.kc1 = ctx->cb.key_c[1];
  p.alpha = std::sqrt(3.14159265358979323846f / 2.0f) / static_cast<float>(ctx->cfg.qjl_dim);
  for (int k = 0; k < 8; ++k) p.vc[k] = ctx->cb.val_c[k];
  p.err = ctx->dev.err;
  p.skip_unit = ctx->wait_skip_unit;
  p.wait_ns = ctx->wait_ns;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128) {
    switch (G) {
      case 1: return dec::run<128, 1>(ctx, p, ws, ws_bytes, st);
      case 2: return dec::run<128, 2>(ctx, p, ws, ws_bytes, st);
      case 4: return dec::run<128, 4>(ctx, p, ws, ws_bytes, st);
      case 8: return dec::run<128, 8>(ctx, p, ws, ws_bytes, st);
    }
  } else if (d == 64) {
    switch (G) {
      case 1: return dec::run<64, 1>(ctx, p, ws, ws_bytes, st);
      case 2: return dec::run<64, 2>(ctx, p, ws, ws_bytes, st);
      case 4: return dec::run<64, 4>(ctx, p, ws, ws_bytes, st);
      case 8: return dec::run<64, 8>(ctx, p, ws, ws_bytes, st);
    }
  }
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq
