// The tensor-core form of a key's 2-bit code (sign, magnitude index): one
// fp16 operand plane holding +-b (index 0) or +-a (index 1), with a / b the
// nearest ratio of two fp16 values to kc1 / kc0; the query side carries
// kc0 / b.  A record's score then needs one contraction over the key
// coordinates instead of one for the signs and one for the magnitudes.
#pragma once

#include <cmath>
#include <cstdint>

namespace tq {

struct KeyPlane {
  double a, b;        // fp16-exact magnitudes, b in [1, 2)
  double rel_err;     // |a/b - kc1/kc0| / (kc1/kc0)
  uint32_t b2;        // fp16 bits of b in both halves of a word
  uint32_t diff;      // fp16 bits(a) - bits(b)
  uint32_t d7;        // fp16 bits of d = fp16(2^7 (a - b)) in both halves;
                      // fp16(2^-7 d + b) == a
};

// whether v > 0 is an fp16 value in the normal range
inline bool f16_exact(double v) {
  if (!(v >= 0x1p-14) || v > 65504.0) return false;
  const int e = static_cast<int>(std::floor(std::log2(v)));
  const double m = std::ldexp(v, 10 - e);  // significand scaled to [1024, 2048)
  return m == std::floor(m);
}

// v > 0 rounded to fp16 (nearest, ties to even; normal range)
inline double round_f16(double v) {
  const int e = static_cast<int>(std::floor(std::log2(v)));
  const double ulp = std::ldexp(1.0, e - 10);
  return std::nearbyint(v / ulp) * ulp;  // the default rounding mode: ties to even
}

// fp16 bits of a positive value with at most 11 significant bits in the
// normal range
inline uint32_t f16_bits_exact(double v) {
  const int e = static_cast<int>(std::floor(std::log2(v)));
  const double mant = v / std::ldexp(1.0, e) - 1.0;
  return (static_cast<uint32_t>(e + 15) << 10) | static_cast<uint32_t>(std::lround(mant * 1024.0));
}

// a / b: among ratios p/q (p, q < 2048, times a power of two) for which one
// fp16 FMA, 2^-7 d + b with d = fp16(2^7 (a - b)), returns a exactly, the
// nearest to kc1 / kc0.  Returns false unless kc1 > kc0 > 0 and the ratio
// is carried to within 2^-19.
inline bool key_plane(double kc0, double kc1, KeyPlane& kp) {
  if (!(kc0 > 0.0) || !(kc1 > kc0)) return false;
  const double r = kc1 / kc0;
  double best = -1.0;
  kp.a = r;
  kp.b = 1.0;
  for (int sh = -3; sh <= 3; ++sh) {
    const double t = std::ldexp(r, -sh);
    for (int qd = 1; qd < 2048; ++qd) {
      const double pn = std::nearbyint(qd * t);
      if (pn < 1.0 || pn > 2047.0) continue;
      const double err = std::fabs(std::ldexp(pn / qd, sh) - r);
      if (best < 0.0 || err < best) {
        const double sc = std::ldexp(1.0, -static_cast<int>(std::floor(std::log2(static_cast<double>(qd)))));
        const double bb = qd * sc, aa = std::ldexp(pn, sh) * sc;
        if (!f16_exact(aa) || !(round_f16(round_f16(128.0 * (aa - bb)) / 128.0 + bb) == aa)) continue;
        best = err;
        kp.b = bb;
        kp.a = aa;
      }
    }
  }
  kp.rel_err = best / r;
  const uint32_t ba = f16_bits_exact(kp.a), bb = f16_bits_exact(kp.b);
  if (!(kp.a > kp.b) || ba >= 0x7C00u || !(kp.rel_err <= 0x1p-19)) return false;
  kp.b2 = bb * 0x10001u;
  kp.diff = ba - bb;
  kp.d7 = f16_bits_exact(round_f16(128.0 * (kp.a - kp.b))) * 0x10001u;
  return true;
}

}  // namespace tq
