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
// Encoders and the polar decoder give each vector a quad of lanes (D/4
// coordinates per lane, 8 vectors per warp), staged through shared memory so
// that global loads and stores stay coalesced; the MSE decoder gives each
// vector a warp.  A record's codes are a whole number of 32-bit words,
// assembled with shared-memory ORs and moved as words.  Every decision is an
// fp32 comparison whose operands are formed the same way in the CPU oracle:
// radii sqrtf(fmaf(u, u, v * v)), level-1 bins by exact turns into the first
// quadrant and v >= u * tan(boundary), higher levels by r_o >= r_e *
// tan(boundary), MSE codes by |x_j| >= fp32(n t_k).
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

__device__ __forceinline__ float tree_radius(float u, float v) {
  return __fsqrt_rn(__fmaf_rn(u, u, __fmul_rn(v, v)));
}

constexpr int WARPS = 8;
constexpr int VPW = 4;  // MSE decoder: vectors per warp and iteration, all loads issued first

// The encoder gives each vector a quad of lanes (8 vectors per warp and
// iteration): lane i of a quad holds coordinates [D/4 i, D/4 (i + 1)), so
// level 1 and the next log2(D/8) levels run inside the lane and only the last
// two levels cross lanes.  A warp's 8 vectors are loaded coalesced (512
// contiguous bytes per instruction) into a staging tile whose lane chunks are
// padded so that the quads' 16-byte reads hit distinct banks.
constexpr int QVEC = 8;

template <int D>
struct QuadTile {
  static constexpr int PER = D / 4;           // coordinates per lane
  static constexpr int F4 = PER / 4;          // float4 per lane
  static constexpr int CHUNK = PER * 4 + 16;  // bytes of a lane's chunk, padded
  static constexpr int VSTRIDE = 4 * CHUNK;   // bytes per staged vector (an odd multiple of 64)
  static constexpr int BYTES = QVEC * VSTRIDE;
};

// 16-byte asynchronous copy into shared memory; src_bytes 0 zero-fills (a
// vector past the end, whose address is not read)
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Copies the warp's 8 vectors n0 .. n0 + 7 (512 contiguous bytes per
// instruction at d = 128) into the padded staging tile, asynchronously.
template <int D>
__device__ __forceinline__ void stage_vectors(const float* x, long long n0, long long N,
                                              uint8_t* tile, int lane) {
  using QT = QuadTile<D>;
#pragma unroll
  for (int s = 0; s < D / 16; ++s) {
    const int f = s * 32 + lane, v = f / (D / 4), u = f % (D / 4);
    const bool ok = n0 + v < N;
    cp_async16(tile + v * QT::VSTRIDE + (u / QT::F4) * QT::CHUNK + (u % QT::F4) * 16,
               ok ? static_cast<const void*>(x + (n0 + v) * D + 4 * u) : static_cast<const void*>(x),
               ok);
  }
  cp_async_commit();
}

// first bit of level l >= 2 (l = 0 is level 2) in a vector's code stream
template <int D, int B1, int B2>
__host__ __device__ constexpr int polar_level_base(int l) {
  return l == 0 ? B1 * (D / 2) : polar_level_base<D, B1, B2>(l - 1) + B2 * (D >> (l + 1));
}

// level-1 code of the pair (a, b): quadrant q and the count of first-quadrant
// boundaries at or below the turned pair (u, v); the boundaries increase, so
// the count is the bin.  A zero (or NaN) pair has code 0.
template <int B1>
__device__ __forceinline__ uint32_t level1_code(float a, float b, const PolarTables& tb) {
  constexpr int Q = (1 << B1) / 4;
  // quadrants 2 and 3 are quadrants 0 and 1 of (-a, -b); in the upper half
  // quadrant 0 is a > 0 and quadrant 1 turns (a, b) into (b, -a)
  const bool lower = b < 0.0f || (b == 0.0f && a < 0.0f);
  const float a2 = lower ? -a : a, b2 = lower ? -b : b;
  const bool first = a2 > 0.0f;
  const float u = first ? a2 : b2;
  const float v = first ? b2 : -a2;
  int j = 0;
#pragma unroll
  for (int i = 0; i < Q - 1; ++i) j += (v >= __fmul_rn(u, tb.tq1[i])) ? 1 : 0;
  const int q = (lower ? 2 : 0) + (first ? 0 : 1);
  const bool pair = (a != 0.0f || b != 0.0f) && a == a && b == b;  // not zero, not NaN
  return pair ? static_cast<uint32_t>(q * Q + j) : 0u;
}

// level-l code of the node (r_e, r_o): the count of boundaries with
// r_o >= r_e tan(t_s) (increasing), 0 when r_o is not positive
template <int B2>
__device__ __forceinline__ uint32_t level_code(float re, float ro, const float* T) {
  int j = 0;
#pragma unroll
  for (int s = 0; s < (1 << B2) - 1; ++s) j += (ro >= __fmul_rn(re, T[s])) ? 1 : 0;
  return ro > 0.0f ? static_cast<uint32_t>(j) : 0u;
}

template <int D, int B1, int B2>
__global__ void __launch_bounds__(WARPS * 32, 4) polar_encode_kernel(const float* __restrict__ x,
                                                                  long long N,
                                                                  int code_bytes,
                                                                  uint8_t* __restrict__ codes,
                                                                  uint16_t* __restrict__ radius,
                                                                  PolarTables tb) {
  using QT = QuadTile<D>;
  constexpr int PER = QT::PER, PAIRS = PER / 2;
  constexpr int LIN = log2i(PAIRS);  // levels >= 2 inside a lane
  constexpr int CB = (B1 * (D / 2) + B2 * (D / 2 - 1) + 7) / 8;
  constexpr int CBW = CB / 4;        // code words per vector (CB is a multiple of 4)
  constexpr int C1 = 32 / B1;        // level-1 codes per packed chunk
  static_assert(CB % 4 == 0 && QVEC * CBW <= 128, "code words");
  static_assert(log2i(D) - 1 == LIN + 2, "two levels cross lanes");
  __shared__ __align__(16) uint8_t stage[WARPS][QT::BYTES];
  __shared__ uint32_t cw[WARPS][QVEC * CBW];
  (void)code_bytes;  // equal to CB (checked by the launcher)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qv = lane >> 2, qi = lane & 3;  // vector of the warp's 8, lane of its quad
  uint8_t* tile = stage[warp];
  uint32_t* words = cw[warp] + qv * CBW;
  const long long step = static_cast<long long>(gridDim.x) * WARPS * QVEC;
  long long n0 = (static_cast<long long>(blockIdx.x) * WARPS + warp) * QVEC;
  if (n0 < N) stage_vectors<D>(x, n0, N, tile, lane);
  for (; n0 < N; n0 += step) {
    // this iteration's vectors have landed; once every lane holds its
    // coordinates the tile takes the next iteration's copies
    cp_async_wait_all();
    __syncwarp();
    float xv[PER];
#pragma unroll
    for (int k = 0; k < QT::F4; ++k) {
      const float4 c4 =
          *reinterpret_cast<const float4*>(tile + qv * QT::VSTRIDE + qi * QT::CHUNK + k * 16);
      xv[4 * k] = c4.x; xv[4 * k + 1] = c4.y; xv[4 * k + 2] = c4.z; xv[4 * k + 3] = c4.w;
    }
    for (int w = lane; w < QVEC * CBW; w += 32) cw[warp][w] = 0u;
    __syncwarp();
    if (n0 + step < N) stage_vectors<D>(x, n0 + step, N, tile, lane);
    // level 1: the lane's pairs PAIRS qi .. PAIRS qi + PAIRS - 1, packed in chunks
    float r[PAIRS];
#pragma unroll
    for (int c0 = 0; c0 < PAIRS; c0 += C1) {
      const int cnt = (PAIRS - c0) < C1 ? (PAIRS - c0) : C1;
      uint32_t val = 0u;
#pragma unroll
      for (int p = c0; p < c0 + C1 && p < PAIRS; ++p) {
        val |= level1_code<B1>(xv[2 * p], xv[2 * p + 1], tb) << (B1 * (p - c0));
        r[p] = tree_radius(xv[2 * p], xv[2 * p + 1]);
      }
      or_bits(words, B1 * (PAIRS * qi + c0), B1 * cnt, val);
    }
    // levels 2 .. LIN + 1 inside the lane: node n of the lane pairs r[2n], r[2n+1]
#pragma unroll
    for (int l = 0; l < LIN; ++l) {
      const int npl = PAIRS >> (l + 1);
      uint32_t val = 0u;
#pragma unroll
      for (int n = 0; n < npl; ++n) {
        val |= level_code<B2>(r[2 * n], r[2 * n + 1], tb.T[l]) << (B2 * n);
        r[n] = tree_radius(r[2 * n], r[2 * n + 1]);
      }
      or_bits(words, polar_level_base<D, B1, B2>(l) + B2 * npl * qi, B2 * npl, val);
    }
    // the last two levels across the quad: lanes 0 and 2 pair with 1 and 3, then lane 0 with 2
    float rr = r[0];
    {
      const float ro = __shfl_down_sync(0xffffffffu, rr, 1);
      if ((qi & 1) == 0) {
        or_bits(words, polar_level_base<D, B1, B2>(LIN) + B2 * (qi >> 1), B2,
                level_code<B2>(rr, ro, tb.T[LIN]));
        rr = tree_radius(rr, ro);
      }
    }
    {
      const float ro = __shfl_down_sync(0xffffffffu, rr, 2);
      if (qi == 0) {
        or_bits(words, polar_level_base<D, B1, B2>(LIN + 1), B2,
                level_code<B2>(rr, ro, tb.T[LIN + 1]));
        rr = tree_radius(rr, ro);
        if (n0 + qv < N) radius[n0 + qv] = __half_as_ushort(__float2half_rn(rr));
      }
    }
    __syncwarp();
    // the 8 vectors' codes are contiguous in memory: copy the words out
    const long long left = N - n0;
    const int nv = left < QVEC ? static_cast<int>(left) : QVEC;
    uint32_t* dst = reinterpret_cast<uint32_t*>(codes + n0 * CB);
    for (int w = lane; w < nv * CBW; w += 32) dst[w] = cw[warp][w];
    __syncwarp();
  }
}

// The decoder uses the same quads: a lane finds the radius of its subtree
// root from the two cross-lane levels, expands it down to its pairs (each
// child radius is its parent's times the cosine or sine of the parent's
// level angle, multiplied in the same order from the top as a per-pair walk),
// and the 8 vectors are written back through the staging tile with coalesced
// stores.
template <int D, int B1, int B2>
__global__ void __launch_bounds__(WARPS * 32) polar_decode_kernel(const uint8_t* __restrict__ codes,
                                                                  const uint16_t* __restrict__ radius,
                                                                  long long N,
                                                                  int code_bytes,
                                                                  float* __restrict__ xhat,
                                                                  PolarTables tb) {
  using QT = QuadTile<D>;
  constexpr int PER = QT::PER, PAIRS = PER / 2;
  constexpr int LIN = log2i(PAIRS);
  constexpr int CB = (B1 * (D / 2) + B2 * (D / 2 - 1) + 7) / 8;
  constexpr int CBW = CB / 4;
  constexpr int LOADS = D / 16;
  static_assert(CB % 4 == 0 && QVEC * CBW <= 128, "code words");
  __shared__ __align__(16) uint8_t stage[WARPS][QT::BYTES];
  __shared__ uint32_t cw[WARPS][QVEC * CBW];
  // the tables are read with per-lane indices: from shared memory, not the
  // kernel parameters (whose reads serialise over distinct addresses)
  __shared__ PolarTables st;
  for (int i = threadIdx.x; i < static_cast<int>(sizeof(PolarTables) / 4); i += blockDim.x)
    reinterpret_cast<float*>(&st)[i] = reinterpret_cast<const float*>(&tb)[i];
  __syncthreads();
  (void)code_bytes;  // equal to CB (checked by the launcher)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qv = lane >> 2, qi = lane & 3;
  uint8_t* tile = stage[warp];
  const uint32_t* words = cw[warp] + qv * CBW;
  for (long long n0 = (static_cast<long long>(blockIdx.x) * WARPS + warp) * QVEC; n0 < N;
       n0 += static_cast<long long>(gridDim.x) * WARPS * QVEC) {
    const long long left = N - n0;
    const int nv = left < QVEC ? static_cast<int>(left) : QVEC;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(codes + n0 * CB);
    for (int w = lane; w < QVEC * CBW; w += 32) cw[warp][w] = w < nv * CBW ? src[w] : 0u;
    const float R = (qi == 0 && qv < nv) ? __half2float(__ushort_as_half(radius[n0 + qv])) : 0.0f;
    __syncwarp();
    // the two cross-lane levels: the root's code splits R between the halves,
    // the half's code between its two quarters (lane qi holds quarter qi)
    const float Rq = __shfl_sync(0xffffffffu, R, lane & ~3);
    const int jt = static_cast<int>(read_bits(words, polar_level_base<D, B1, B2>(LIN + 1), B2));
    const float rh = __fmul_rn(Rq, (qi >> 1) ? st.sinl[LIN + 1][jt] : st.cosl[LIN + 1][jt]);
    const int jh = static_cast<int>(
        read_bits(words, polar_level_base<D, B1, B2>(LIN) + B2 * (qi >> 1), B2));
    float rad[PAIRS];
    rad[0] = __fmul_rn(rh, (qi & 1) ? st.sinl[LIN][jh] : st.cosl[LIN][jh]);
    // in-lane levels, top down; node n of the lane at level l has children 2n, 2n + 1
#pragma unroll
    for (int l = LIN - 1; l >= 0; --l) {
      const int npl = PAIRS >> (l + 1);
      const uint32_t lc = read_bits(words, polar_level_base<D, B1, B2>(l) + B2 * npl * qi, B2 * npl);
#pragma unroll
      for (int n = npl - 1; n >= 0; --n) {
        const int j = static_cast<int>((lc >> (B2 * n)) & ((1u << B2) - 1u));
        const float rp = rad[n];
        rad[2 * n] = __fmul_rn(rp, st.cosl[l][j]);
        rad[2 * n + 1] = __fmul_rn(rp, st.sinl[l][j]);
      }
    }
    // level 1: the pair's angle bin centre
    float out[PER];
#pragma unroll
    for (int p = 0; p < PAIRS; ++p) {
      const int k = static_cast<int>(read_bits(words, B1 * (PAIRS * qi + p), B1));
      out[2 * p] = __fmul_rn(rad[p], st.cos1[k]);
      out[2 * p + 1] = __fmul_rn(rad[p], st.sin1[k]);
    }
#pragma unroll
    for (int k = 0; k < QT::F4; ++k)
      *reinterpret_cast<float4*>(tile + qv * QT::VSTRIDE + qi * QT::CHUNK + k * 16) =
          make_float4(out[4 * k], out[4 * k + 1], out[4 * k + 2], out[4 * k + 3]);
    __syncwarp();
#pragma unroll
    for (int s = 0; s < LOADS; ++s) {
      const int f = s * 32 + lane, v = f / (D / 4), u = f % (D / 4);
      if (v < nv)
        reinterpret_cast<float4*>(xhat + (n0 + v) * D)[u] = *reinterpret_cast<const float4*>(
            tile + v * QT::VSTRIDE + (u / QT::F4) * QT::CHUNK + (u % QT::F4) * 16);
    }
    __syncwarp();
  }
}

// The MSE encoder uses the polar encoder's quads and staging tile: the norm
// is the lane's sum of squares reduced over its quad, and each lane's codes
// are a contiguous field of the record.
template <int D, int BITS>
__global__ void __launch_bounds__(WARPS * 32) mse_encode_kernel(const float* __restrict__ x,
                                                                long long N, int code_bytes,
                                                                uint8_t* __restrict__ codes,
                                                                uint16_t* __restrict__ norms,
                                                                MseTables tb) {
  using QT = QuadTile<D>;
  constexpr int PER = QT::PER;
  constexpr int bits = BITS, L = 1 << (BITS - 1);
  constexpr int CB = (BITS * D) / 8;
  constexpr int CBW = CB / 4;
  constexpr int C1 = 32 / BITS;  // codes per packed chunk
  static_assert(CB % 4 == 0 && QVEC * CBW <= 128, "code words");
  __shared__ __align__(16) uint8_t stage[WARPS][QT::BYTES];
  __shared__ uint32_t cw[WARPS][QVEC * CBW];
  (void)code_bytes;  // equal to CB (checked by the launcher)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qv = lane >> 2, qi = lane & 3;
  uint8_t* tile = stage[warp];
  uint32_t* words = cw[warp] + qv * CBW;
  const long long step = static_cast<long long>(gridDim.x) * WARPS * QVEC;
  long long n0 = (static_cast<long long>(blockIdx.x) * WARPS + warp) * QVEC;
  if (n0 < N) stage_vectors<D>(x, n0, N, tile, lane);
  for (; n0 < N; n0 += step) {
    cp_async_wait_all();
    __syncwarp();
    float v[PER];
#pragma unroll
    for (int k = 0; k < QT::F4; ++k) {
      const float4 c4 =
          *reinterpret_cast<const float4*>(tile + qv * QT::VSTRIDE + qi * QT::CHUNK + k * 16);
      v[4 * k] = c4.x; v[4 * k + 1] = c4.y; v[4 * k + 2] = c4.z; v[4 * k + 3] = c4.w;
    }
    for (int w = lane; w < QVEC * CBW; w += 32) cw[warp][w] = 0u;
    __syncwarp();
    if (n0 + step < N) stage_vectors<D>(x, n0 + step, N, tile, lane);
    float ss = 0.0f;
#pragma unroll
    for (int e = 0; e < PER; ++e) ss = fmaf(v[e], v[e], ss);
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    const __half nh = __float2half_rn(sqrtf(ss));
    const float nf = __half2float(nh);
    const bool degenerate = !(nf > 0.0f) || isinf(nf);  // zero or overflowing norm: all codes 0
    float thr[L - 1];
#pragma unroll
    for (int s = 0; s < L - 1; ++s) thr[s] = __fmul_rn(nf, tb.t[s]);
#pragma unroll
    for (int c0 = 0; c0 < PER; c0 += C1) {
      const int cnt = (PER - c0) < C1 ? (PER - c0) : C1;
      uint32_t val = 0u;
#pragma unroll
      for (int e = c0; e < c0 + C1 && e < PER; ++e) {
        const float a = fabsf(v[e]);
        int k = 0;
#pragma unroll
        for (int s = 0; s < L - 1; ++s) k += (a >= thr[s]) ? 1 : 0;  // increasing boundaries
        const uint32_t sgn = (v[e] < 0.0f) ? 1u : 0u;
        val |= ((sgn << (bits - 1)) | static_cast<uint32_t>(k)) << (bits * (e - c0));
      }
      if (!degenerate) or_bits(words, bits * (PER * qi + c0), bits * cnt, val);
    }
    if (qi == 0 && n0 + qv < N) norms[n0 + qv] = __half_as_ushort(nh);
    __syncwarp();
    const long long left = N - n0;
    const int nv = left < QVEC ? static_cast<int>(left) : QVEC;
    uint32_t* dst = reinterpret_cast<uint32_t*>(codes + n0 * CB);
    for (int w = lane; w < nv * CBW; w += 32) dst[w] = cw[warp][w];
    __syncwarp();
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
  // vectors per CTA and iteration: a quad of lanes per vector, except for the
  // MSE decoder (a warp per vector)
  const int per_cta = (kind == TQ_STAGE1_POLAR || encode) ? s1::WARPS * s1::QVEC : s1::WARPS * s1::VPW;
  const long long blocks_needed = (N + per_cta - 1) / per_cta;
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
