// Stage-1 quantiser variants on rotated vectors ("TurboQuant" summary,
// de.news.hada.io topic 27867, section "Funktionsweise von TurboQuant": a
// standard per-coordinate quantiser after the rotation; section "PolarQuant:
// Ein neuer Winkel auf Kompression": pairs of coordinates to polar form, the
// radii paired again recursively until one radius and a set of angles
// remain, the angles quantised on fixed grids).
//
//  MSE    b bits per coordinate: sign + (b-1)-bit Lloyd-Max magnitude index of
//         x_rot / n, n = fp16(|x|); no QJL sketch.  Code of coordinate j in
//         bits [b j, b j + b) of a little-endian bit stream.
//  POLAR  level-1 angles of the coordinate pairs on 2^b1 equal bins of
//         [0, 2 pi), level-l angles (l >= 2) of the block radii with a
//         2^b2-level Lloyd-Max codebook of their density sin^(k-1)(2 phi),
//         k = 2^(l-1); the final radius as fp16.  Codes: level 1 first (b1
//         bits per pair), then level 2, 3, ... (b2 bits per node).
//
// One warp per vector, D/32 coordinates per lane (coalesced 8- or 16-byte
// loads); a record's codes are a whole number of 32-bit words, assembled
// across lanes with shuffles (level-1 and MSE codes) or shared-memory ORs
// (the polar levels >= 2) and moved as words.  Every decision is an fp32 comparison whose operands are formed the
// same way in the CPU oracle: radii sqrtf(fmaf(u, u, v * v)), level-1 bins by
// exact turns into the first quadrant and v >= u * tan(boundary), higher
// levels by r_o >= r_e * tan(boundary), MSE codes by |x_j| >= fp32(n t_k).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {
namespace s1 {

constexpr int MAX_LEVELS = 6;  // levels >= 2 at d = 128
constexpr int MAX_B2 = 8;      // 2^3 levels per higher-level angle

struct PolarTables {
  float tq1[7];              // tan(2 pi j / M), j = 1 .. M/4 - 1 (first-quadrant boundaries)
  float cos1[32], sin1[32];  // level-1 bin centres
  float T[MAX_LEVELS][MAX_B2 - 1];  // tan of the level boundaries
  float cosl[MAX_LEVELS][MAX_B2], sinl[MAX_LEVELS][MAX_B2];
};

struct MseTables {
  float c[8];  // positive levels
  float t[7];  // positive boundaries
};

__host__ __device__ constexpr int log2i(int v) { return v <= 1 ? 0 : 1 + log2i(v / 2); }

__device__ __forceinline__ void or_bits(uint32_t* words, int pos, int nbits, uint32_t v) {
  const int w = pos >> 5, o = pos & 31;
  atomicOr(&words[w], v << o);
  if (o + nbits > 32) atomicOr(&words[w + 1], v >> (32 - o));
}

__device__ __forceinline__ uint32_t read_bits(const uint32_t* words, int pos, int nbits) {
  const int w = pos >> 5, o = pos & 31;
  uint64_t x = words[w];
  if (o + nbits > 32) x |= static_cast<uint64_t>(words[w + 1]) << 32;
  return static_cast<uint32_t>(x >> o) & ((1u << nbits) - 1u);
}

// Lane l holds v (bpl bits) destined for bits [bpl l, bpl l + bpl) of a
// stream of bpl words; returns word `lane` of it (lanes >= bpl get 0).  Each
// word gathers the few lanes that overlap it with shuffles.
__device__ __forceinline__ uint32_t assemble_words(uint32_t v, int bpl, int lane) {
  const int lo_bit = 32 * lane;
  const int l0 = lo_bit / bpl;
  const int K = (32 + bpl - 1) / bpl + 1;  // warp-uniform
  uint32_t word = 0u;
  for (int k = 0; k < K; ++k) {
    const int src = l0 + k;
    const uint32_t vs = __shfl_sync(0xffffffffu, v, src < 32 ? src : 31);
    const int sh = bpl * src - lo_bit;
    if (lane < bpl && src < 32 && sh < 32) word |= sh >= 0 ? (vs << sh) : (vs >> (-sh));
  }
  return word;
}

__device__ __forceinline__ float tree_radius(float u, float v) {
  return __fsqrt_rn(__fmaf_rn(u, u, __fmul_rn(v, v)));
}

__device__ __forceinline__ int level1_bin(float a, float b, int M, const PolarTables& tb) {
  int q;
  float u, v;
  if (a > 0.0f && b >= 0.0f) { q = 0; u = a; v = b; }
  else if (a <= 0.0f && b > 0.0f) { q = 1; u = b; v = -a; }
  else if (a < 0.0f && b <= 0.0f) { q = 2; u = -a; v = -b; }
  else if (a >= 0.0f && b < 0.0f) { q = 3; u = -b; v = a; }
  else return 0;  // zero pair
  int j = 0;
  for (int i = 0; i < M / 4 - 1; ++i)
    if (v >= __fmul_rn(u, tb.tq1[i])) j = i + 1;
  return q * (M / 4) + j;
}

constexpr int WARPS = 8;
constexpr int VPW = 4;              // vectors per warp and iteration, all loads issued first
constexpr int MAX_CODE_WORDS = 16;  // 64 bytes of codes per vector

template <int PER>
__device__ __forceinline__ void load_row(const float* x, long long n, long long N, int lane,
                                         float (&v)[PER]) {
  if (n >= N) {
#pragma unroll
    for (int e = 0; e < PER; ++e) v[e] = 0.0f;
    return;
  }
  if constexpr (PER == 4) {
    const float4 t = reinterpret_cast<const float4*>(x + n * (32 * PER))[lane];
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else {
    const float2 t = reinterpret_cast<const float2*>(x + n * (32 * PER))[lane];
    v[0] = t.x; v[1] = t.y;
  }
}

template <int D, int B1, int B2>
__global__ void __launch_bounds__(WARPS * 32) polar_encode_kernel(const float* __restrict__ x,
                                                                  long long N,
                                                                  int code_bytes,
                                                                  uint8_t* __restrict__ codes,
                                                                  uint16_t* __restrict__ radius,
                                                                  PolarTables tb) {
  constexpr int PER = D / 32;     // coordinates per lane
  constexpr int PAIRS = PER / 2;  // level-1 pairs per lane
  constexpr int NL = log2i(D) - 1;
  __shared__ uint32_t words[WARPS][MAX_CODE_WORDS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int b1 = B1, b2 = B2, M = 1 << B1, L = 1 << B2;
  for (long long n = static_cast<long long>(blockIdx.x) * WARPS + warp; n < N;
       n += static_cast<long long>(gridDim.x) * WARPS) {
    if (lane < MAX_CODE_WORDS) words[warp][lane] = 0u;
    __syncwarp();
    float v[PER];
    if constexpr (PER == 4) {
      const float4 t = reinterpret_cast<const float4*>(x + n * D)[lane];
      v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
      const float2 t = reinterpret_cast<const float2*>(x + n * D)[lane];
      v[0] = t.x; v[1] = t.y;
    }
    // level 1: the lane's pairs, contiguous bits, assembled across lanes
    float r[PAIRS];
    uint32_t mine = 0u;
#pragma unroll
    for (int p = 0; p < PAIRS; ++p) {
      mine |= static_cast<uint32_t>(level1_bin(v[2 * p], v[2 * p + 1], M, tb)) << (b1 * p);
      r[p] = tree_radius(v[2 * p], v[2 * p + 1]);
    }
    const uint32_t w1 = assemble_words(mine, PAIRS * b1, lane);  // words 0 .. PAIRS b1 - 1
    uint32_t w2 = 0u;  // (d = 128) the level-2 words, held by lanes 0 .. b2 - 1
    // levels >= 2: node i of a level pairs the radii of nodes 2i, 2i + 1 below
    int base = b1 * (D / 2);
    int nodes = D / 2;
    float rr = r[0];  // the radius of the node this lane holds after in-lane levels
    int held = lane * PAIRS;  // index (at the current level) of the node held in rr
    int lvl = 0;
    if constexpr (PAIRS == 2) {
      // level 2 pairs the lane's own two radii
      nodes /= 2;
      const float re = r[0], ro = r[1];
      int j = 0;
      if (ro > 0.0f)
#pragma unroll
        for (int s = 0; s < L - 1; ++s)
          if (ro >= __fmul_rn(re, tb.T[0][s])) j = s + 1;
      w2 = assemble_words(static_cast<uint32_t>(j), b2, lane);  // one code per lane
      rr = tree_radius(re, ro);
      held = lane;
      base += b2 * nodes;
      lvl = 1;
    }
    // remaining levels across lanes: at stride st the node held by lane l
    // (l a multiple of 2 st) pairs with the one held by lane l + st
    for (int st = 1; lvl < NL; st *= 2, ++lvl) {
      nodes /= 2;
      const float ro = __shfl_down_sync(0xffffffffu, rr, st);
      const bool owner = (lane % (2 * st)) == 0;
      if (owner) {
        const float re = rr;
        int j = 0;
        if (ro > 0.0f)
#pragma unroll
          for (int s = 0; s < L - 1; ++s)
            if (ro >= __fmul_rn(re, tb.T[lvl][s])) j = s + 1;
        const int node = held / 2;
        or_bits(words[warp], base + b2 * node, b2, static_cast<uint32_t>(j));
        rr = tree_radius(re, ro);
        held = node;
      }
      base += b2 * nodes;
    }
    __syncwarp();
    // words: level 1 from w1, (d = 128) level 2 from w2, the rest from shared memory
    constexpr int n1 = PAIRS * b1, n2 = (PAIRS == 2) ? b2 : 0;
    const uint32_t w2l = __shfl_sync(0xffffffffu, w2, (lane - n1) & 31);
    if (lane < code_bytes / 4)
      reinterpret_cast<uint32_t*>(codes + n * code_bytes)[lane] =
          lane < n1 ? w1 : (lane < n1 + n2 ? w2l : words[warp][lane]);
    if (lane == 0) radius[n] = __half_as_ushort(__float2half_rn(rr));
    __syncwarp();
  }
}

template <int D, int B1, int B2>
__global__ void __launch_bounds__(WARPS * 32) polar_decode_kernel(const uint8_t* __restrict__ codes,
                                                                  const uint16_t* __restrict__ radius,
                                                                  long long N,
                                                                  int code_bytes,
                                                                  float* __restrict__ xhat,
                                                                  PolarTables tb) {
  constexpr int PER = D / 32;
  constexpr int PAIRS = PER / 2;
  constexpr int NL = log2i(D) - 1;
  constexpr int b1 = B1, b2 = B2;
  __shared__ uint32_t words[WARPS][MAX_CODE_WORDS];
  // the tables are read with per-lane indices: from shared memory, not the
  // kernel parameters (whose reads serialise over distinct addresses)
  __shared__ PolarTables st;
  for (int i = threadIdx.x; i < static_cast<int>(sizeof(PolarTables) / 4); i += blockDim.x)
    reinterpret_cast<float*>(&st)[i] = reinterpret_cast<const float*>(&tb)[i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = code_bytes / 4;
  for (long long n0 = (static_cast<long long>(blockIdx.x) * WARPS + warp) * VPW; n0 < N;
       n0 += static_cast<long long>(gridDim.x) * WARPS * VPW) {
  uint32_t cw[VPW];
  float rad[VPW];
#pragma unroll
  for (int u = 0; u < VPW; ++u) {
    const bool ok = n0 + u < N;
    cw[u] = (ok && lane < nw) ? reinterpret_cast<const uint32_t*>(codes + (n0 + u) * code_bytes)[lane] : 0u;
    rad[u] = ok ? __half2float(__ushort_as_half(radius[n0 + u])) : 0.0f;
  }
#pragma unroll
  for (int u = 0; u < VPW; ++u) {
    if (n0 + u >= N) break;
    const long long n = n0 + u;
    if (lane < MAX_CODE_WORDS) words[warp][lane] = lane < nw ? cw[u] : 0u;
    __syncwarp();
    // section offsets of the levels >= 2
    int off[NL];
    {
      int base = b1 * (D / 2), cnt = D / 2;
#pragma unroll
      for (int l = 0; l < NL; ++l) {
        cnt /= 2;
        off[l] = base;
        base += b2 * cnt;
      }
    }
    const float R = rad[u];
    float out[PER];
#pragma unroll
    for (int p = 0; p < PAIRS; ++p) {
      const int i = lane * PAIRS + p;  // level-1 pair index
      float r = R;
      // walk from the top level down to the pair: at level l (0 = level 2)
      // the pair lies under node i >> (l + 1), in child (i >> l) & 1
#pragma unroll
      for (int l = NL - 1; l >= 0; --l) {
        const int node = i >> (l + 1), child = (i >> l) & 1;
        const int j = static_cast<int>(read_bits(words[warp], off[l] + b2 * node, b2));
        r = __fmul_rn(r, child ? st.sinl[l][j] : st.cosl[l][j]);
      }
      const int k = static_cast<int>(read_bits(words[warp], b1 * i, b1));
      out[2 * p] = __fmul_rn(r, st.cos1[k]);
      out[2 * p + 1] = __fmul_rn(r, st.sin1[k]);
    }
    if constexpr (PER == 4)
      reinterpret_cast<float4*>(xhat + n * D)[lane] = make_float4(out[0], out[1], out[2], out[3]);
    else
      reinterpret_cast<float2*>(xhat + n * D)[lane] = make_float2(out[0], out[1]);
    __syncwarp();
  }
  }
}

template <int D, int BITS>
__global__ void __launch_bounds__(WARPS * 32) mse_encode_kernel(const float* __restrict__ x,
                                                                long long N, int code_bytes,
                                                                uint8_t* __restrict__ codes,
                                                                uint16_t* __restrict__ norms,
                                                                MseTables tb) {
  constexpr int PER = D / 32;
  constexpr int bits = BITS, L = 1 << (BITS - 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (long long n0 = (static_cast<long long>(blockIdx.x) * WARPS + warp) * VPW; n0 < N;
       n0 += static_cast<long long>(gridDim.x) * WARPS * VPW) {
  float vin[VPW][PER];
#pragma unroll
  for (int u = 0; u < VPW; ++u) load_row<PER>(x, n0 + u, N, lane, vin[u]);
#pragma unroll
  for (int u = 0; u < VPW; ++u) {
    const long long n = n0 + u;
    if (n >= N) break;
    float v[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) v[e] = vin[u][e];
    float ss = 0.0f;
#pragma unroll
    for (int e = 0; e < PER; ++e) ss = fmaf(v[e], v[e], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const __half nh = __float2half_rn(sqrtf(ss));
    const float nf = __half2float(nh);
    const bool degenerate = !(nf > 0.0f) || isinf(nf);  // zero or overflowing norm: all codes 0
    uint32_t mine = 0u;  // the lane's PER codes, contiguous
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const float a = fabsf(v[e]);
      int k = 0;
#pragma unroll
      for (int s = 0; s < L - 1; ++s)
        if (a >= __fmul_rn(nf, tb.t[s])) k = s + 1;
      const uint32_t sgn = (v[e] < 0.0f) ? 1u : 0u;
      const uint32_t code = degenerate ? 0u : ((sgn << (bits - 1)) | static_cast<uint32_t>(k));
      mine |= code << (bits * e);
    }
    const uint32_t w = assemble_words(mine, PER * bits, lane);  // PER bits words = the record
    if (lane < PER * bits) reinterpret_cast<uint32_t*>(codes + n * code_bytes)[lane] = w;
    if (lane == 0) norms[n] = __half_as_ushort(nh);
  }
  }
}

template <int D, int BITS>
__global__ void __launch_bounds__(WARPS * 32) mse_decode_kernel(const uint8_t* __restrict__ codes,
                                                                const uint16_t* __restrict__ norms,
                                                                long long N, int code_bytes,
                                                                float* __restrict__ xhat,
                                                                MseTables tb) {
  constexpr int PER = D / 32;
  constexpr int BPL = PER * BITS;  // code bits per lane; the record is BPL words
  constexpr uint32_t MMASK = (1u << (BITS - 1)) - 1u;
  __shared__ float sc[8];  // levels, read with per-lane indices
  if (threadIdx.x < 8) sc[threadIdx.x] = tb.c[threadIdx.x];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = code_bytes / 4;
  const int lo_bit = BPL * lane, w0 = lo_bit >> 5, w1 = (lo_bit + BPL - 1) >> 5, sh = lo_bit & 31;
  for (long long n0 = (static_cast<long long>(blockIdx.x) * WARPS + warp) * VPW; n0 < N;
       n0 += static_cast<long long>(gridDim.x) * WARPS * VPW) {
  uint32_t cw[VPW];
  float nrm[VPW];
#pragma unroll
  for (int u = 0; u < VPW; ++u) {
    const bool ok = n0 + u < N;
    cw[u] = (ok && lane < nw) ? reinterpret_cast<const uint32_t*>(codes + (n0 + u) * code_bytes)[lane] : 0u;
    nrm[u] = ok ? __half2float(__ushort_as_half(norms[n0 + u])) : 0.0f;
  }
#pragma unroll
  for (int u = 0; u < VPW; ++u) {
    if (n0 + u >= N) break;
    const long long n = n0 + u;
    // the lane's BPL code bits from the (at most two) words holding them
    const uint32_t lo = __shfl_sync(0xffffffffu, cw[u], w0);
    const uint32_t hi = __shfl_sync(0xffffffffu, cw[u], w1);
    const uint32_t mine =
        static_cast<uint32_t>(((static_cast<uint64_t>(hi) << 32) | lo) >> sh);
    const float nf = nrm[u];
    float out[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const uint32_t code = (mine >> (BITS * e)) & ((1u << BITS) - 1u);
      const float c = sc[code & MMASK];
      out[e] = __fmul_rn(nf, (code >> (BITS - 1)) ? -c : c);
    }
    if constexpr (PER == 4)
      reinterpret_cast<float4*>(xhat + n * D)[lane] = make_float4(out[0], out[1], out[2], out[3]);
    else
      reinterpret_cast<float2*>(xhat + n * D)[lane] = make_float2(out[0], out[1]);
  }
  }
}

// host tables, computed once per (kind, d, b1, b2) and kept for the process
std::mutex g_mu;
std::map<std::tuple<int, int, int>, PolarTables> g_polar;
std::map<std::pair<int, int>, MseTables> g_mse;

PolarTables polar_tables(int d, int b1, int b2) {
  std::lock_guard<std::mutex> lock(g_mu);
  const auto key = std::make_tuple(d, b1, b2);
  auto it = g_polar.find(key);
  if (it != g_polar.end()) return it->second;
  PolarTables tb{};
  const int M = 1 << b1, L = 1 << b2;
  const double two_pi = 6.283185307179586476925286766559;
  for (int i = 0; i < M / 4 - 1; ++i) tb.tq1[i] = static_cast<float>(std::tan(two_pi * (i + 1) / M));
  for (int j = 0; j < M; ++j) {
    tb.cos1[j] = static_cast<float>(std::cos(two_pi * (j + 0.5) / M));
    tb.sin1[j] = static_cast<float>(std::sin(two_pi * (j + 0.5) / M));
  }
  const int nl = log2i(d) - 1;
  for (int l = 0; l < nl; ++l) {
    std::vector<double> c, t;
    angle_lloyd_max(1 << (l + 1), b2, c, t);
    for (int s = 0; s < L - 1; ++s) tb.T[l][s] = static_cast<float>(std::tan(t[s]));
    for (int j = 0; j < L; ++j) {
      tb.cosl[l][j] = static_cast<float>(std::cos(c[j]));
      tb.sinl[l][j] = static_cast<float>(std::sin(c[j]));
    }
  }
  g_polar[key] = tb;
  return tb;
}

MseTables mse_tables(int d, int bits) {
  std::lock_guard<std::mutex> lock(g_mu);
  const auto key = std::make_pair(d, bits);
  auto it = g_mse.find(key);
  if (it != g_mse.end()) return it->second;
  MseTables tb{};
  std::vector<double> c, t;
  sphere_lloyd_max(d, bits, c, t);
  for (size_t i = 0; i < c.size(); ++i) tb.c[i] = static_cast<float>(c[i]);
  for (size_t i = 0; i < t.size(); ++i) tb.t[i] = static_cast<float>(t[i]);
  g_mse[key] = tb;
  return tb;
}

}  // namespace s1

size_t stage1_code_bytes(int d, int kind, int b1, int b2) {
  if (d != 64 && d != 128) return 0;
  if (kind == TQ_STAGE1_MSE) {
    if (b1 < 2 || b1 > 4) return 0;
    return (static_cast<size_t>(b1) * d + 7) / 8;
  }
  if (kind == TQ_STAGE1_POLAR) {
    if (b1 < 2 || b1 > 5 || b2 < 1 || b2 > 3) return 0;
    return (static_cast<size_t>(b1) * (d / 2) + static_cast<size_t>(b2) * (d / 2 - 1) + 7) / 8;
  }
  return 0;
}

int launch_stage1(const tq_ctx* ctx, int kind, int b1, int b2, bool encode, const float* x,
                  const uint8_t* codes_in, uint8_t* codes_out, const uint16_t* norms_in,
                  uint16_t* norms_out, float* xhat, long long N, void* stream) {
  const int d = ctx->cfg.head_dim;
  const int cb = static_cast<int>(stage1_code_bytes(d, kind, b1, b2));
  if (cb == 0) return TQ_ERR_UNSUPPORTED;
  if (N == 0) return TQ_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long blocks_needed = (N + s1::WARPS * s1::VPW - 1) / (s1::WARPS * s1::VPW);
  const int grid = static_cast<int>(blocks_needed < 16LL * ctx->num_sms ? blocks_needed : 16LL * ctx->num_sms);
  const int threads = s1::WARPS * 32;
  if (kind == TQ_STAGE1_POLAR) {
    const s1::PolarTables tb = s1::polar_tables(d, b1, b2);
#define TQ_S1_POLAR(DD, BB1, BB2)                                                                  \
  do {                                                                                             \
    if (encode)                                                                                    \
      s1::polar_encode_kernel<DD, BB1, BB2><<<grid, threads, 0, st>>>(x, N, cb, codes_out,          \
                                                                      norms_out, tb);               \
    else                                                                                           \
      s1::polar_decode_kernel<DD, BB1, BB2><<<grid, threads, 0, st>>>(codes_in, norms_in, N, cb,    \
                                                                      xhat, tb);                    \
  } while (0)
#define TQ_S1_POLAR_B2(DD, BB1)                 \
  do {                                          \
    if (b2 == 1) TQ_S1_POLAR(DD, BB1, 1);       \
    else if (b2 == 2) TQ_S1_POLAR(DD, BB1, 2);  \
    else TQ_S1_POLAR(DD, BB1, 3);               \
  } while (0)
#define TQ_S1_POLAR_D(DD)                       \
  do {                                          \
    if (b1 == 2) TQ_S1_POLAR_B2(DD, 2);         \
    else if (b1 == 3) TQ_S1_POLAR_B2(DD, 3);    \
    else if (b1 == 4) TQ_S1_POLAR_B2(DD, 4);    \
    else TQ_S1_POLAR_B2(DD, 5);                 \
  } while (0)
    if (d == 128) TQ_S1_POLAR_D(128);
    else TQ_S1_POLAR_D(64);
#undef TQ_S1_POLAR_D
#undef TQ_S1_POLAR_B2
#undef TQ_S1_POLAR
  } else {
    const s1::MseTables tb = s1::mse_tables(d, b1);
#define TQ_S1_MSE(DD, BB)                                                                          \
  do {                                                                                             \
    if (encode)                                                                                    \
      s1::mse_encode_kernel<DD, BB><<<grid, threads, 0, st>>>(x, N, cb, codes_out, norms_out, tb); \
    else                                                                                           \
      s1::mse_decode_kernel<DD, BB><<<grid, threads, 0, st>>>(codes_in, norms_in, N, cb, xhat, tb); \
  } while (0)
    if (d == 128) {
      if (b1 == 2) TQ_S1_MSE(128, 2);
      else if (b1 == 3) TQ_S1_MSE(128, 3);
      else TQ_S1_MSE(128, 4);
    } else {
      if (b1 == 2) TQ_S1_MSE(64, 2);
      else if (b1 == 3) TQ_S1_MSE(64, 3);
      else TQ_S1_MSE(64, 4);
    }
#undef TQ_S1_MSE
  }
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace tq
