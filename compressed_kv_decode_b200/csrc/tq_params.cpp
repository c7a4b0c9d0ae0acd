// Host-side generation of the codec tables: Haar rotation, QJL matrix and
// Lloyd-Max codebooks ("TurboQuant" summary, de.news.hada.io topic 27867,
// section "Funktionsweise von TurboQuant" and the discussion's remark on
// Lloyd-Max boundaries and reconstruction values after the rotation; section
// "QJL: Eine 1-Bit-Methode ohne Overhead" for the JL matrix).
//
// Random numbers: SplitMix64 (Steele, Lea, Flood 2014) -> 53-bit uniforms ->
// Box-Muller (both outputs, cosine first).  The rotation is the Q factor of a
// Gaussian matrix, orthonormalised here by classical Gram-Schmidt with one
// re-orthogonalisation pass (CGS2); the positive-diagonal convention makes it
// the same matrix as any other QR of that matrix.  Codebook cell masses use
// the regularised incomplete beta function (a coordinate X of a uniform unit
// vector has X^2 ~ Beta(1/2, (d-1)/2)), evaluated by its continued fraction.
#include "tq_internal.h"

#include <cmath>
#include <cstring>
#include <vector>

namespace tq {
namespace {

struct SplitMix64 {
  uint64_t s;
  explicit SplitMix64(uint64_t seed) : s(seed) {}
  uint64_t next() {
    s += 0x9E3779B97F4A7C15ULL;
    uint64_t z = s;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
  }
  double uniform() { return static_cast<double>(next() >> 11) * (1.0 / 9007199254740992.0); }
};

// Fill `out` with standard normals: pairs (r cos t, r sin t), r = sqrt(-2 ln(1-u1)).
void normal_stream(uint64_t seed, std::vector<double>& out) {
  SplitMix64 g(seed);
  const double two_pi = 6.283185307179586476925286766559;
  size_t i = 0;
  while (i < out.size()) {
    double u1 = 1.0 - g.uniform();
    double u2 = g.uniform();
    double rad = std::sqrt(-2.0 * std::log(u1));
    double ang = two_pi * u2;
    out[i++] = rad * std::cos(ang);
    if (i < out.size()) out[i++] = rad * std::sin(ang);
  }
}

// Columns of g (d x d row-major) orthonormalised in order: q_j = g_j minus its
// projections on q_0..q_{j-1}, twice, then normalised.  R_jj > 0 by construction.
bool haar_rotation(int d, uint64_t seed, std::vector<double>& pi) {
  std::vector<double> g(static_cast<size_t>(d) * d);
  normal_stream(2ULL * seed, g);
  std::vector<std::vector<double>> cols(d, std::vector<double>(d));
  for (int j = 0; j < d; ++j)
    for (int i = 0; i < d; ++i) cols[j][i] = g[static_cast<size_t>(i) * d + j];
  for (int j = 0; j < d; ++j) {
    std::vector<double>& v = cols[j];
    for (int pass = 0; pass < 2; ++pass) {
      std::vector<double> proj(j, 0.0);
      for (int p = 0; p < j; ++p) {
        double s = 0.0;
        for (int i = 0; i < d; ++i) s += cols[p][i] * v[i];
        proj[p] = s;
      }
      for (int p = 0; p < j; ++p)
        for (int i = 0; i < d; ++i) v[i] -= proj[p] * cols[p][i];
    }
    double nrm = 0.0;
    for (int i = 0; i < d; ++i) nrm += v[i] * v[i];
    nrm = std::sqrt(nrm);
    if (!(nrm > 0.0)) return false;
    for (int i = 0; i < d; ++i) v[i] /= nrm;
  }
  pi.assign(static_cast<size_t>(d) * d, 0.0);
  for (int j = 0; j < d; ++j)
    for (int i = 0; i < d; ++i) pi[static_cast<size_t>(i) * d + j] = cols[j][i];
  return true;
}

// Regularised incomplete beta I_x(a, b) by the continued fraction (modified
// Lentz), using the symmetry I_x(a,b) = 1 - I_{1-x}(b,a) where it converges
// faster.
long double betacf(long double a, long double b, long double x) {
  const long double tiny = 1e-4000L;
  long double c = 1.0L, dd = 1.0L - (a + b) * x / (a + 1.0L);
  if (fabsl(dd) < tiny) dd = tiny;
  dd = 1.0L / dd;
  long double h = dd;
  for (int m = 1; m < 100000; ++m) {
    long double m2 = 2.0L * m;
    long double aa = m * (b - m) * x / ((a + m2 - 1.0L) * (a + m2));
    dd = 1.0L + aa * dd;
    if (fabsl(dd) < tiny) dd = tiny;
    c = 1.0L + aa / c;
    if (fabsl(c) < tiny) c = tiny;
    dd = 1.0L / dd;
    h *= dd * c;
    aa = -(a + m) * (a + b + m) * x / ((a + m2) * (a + m2 + 1.0L));
    dd = 1.0L + aa * dd;
    if (fabsl(dd) < tiny) dd = tiny;
    c = 1.0L + aa / c;
    if (fabsl(c) < tiny) c = tiny;
    dd = 1.0L / dd;
    long double del = dd * c;
    h *= del;
    if (fabsl(del - 1.0L) < 1e-19L) break;
  }
  return h;
}

long double ibeta(long double a, long double b, long double x) {
  if (x <= 0.0L) return 0.0L;
  if (x >= 1.0L) return 1.0L;
  long double lbt = lgammal(a + b) - lgammal(a) - lgammal(b) + a * logl(x) + b * log1pl(-x);
  long double front = expl(lbt);
  if (x < (a + 1.0L) / (a + b + 2.0L)) return front * betacf(a, b, x) / a;
  return 1.0L - front * betacf(b, a, 1.0L - x) / b;
}

// P(0 <= X <= t) for one coordinate X of a uniform unit vector in R^d.
long double half_mass(int d, long double t) {
  return 0.5L * ibeta(0.5L, 0.5L * (d - 1), t * t);
}

// int_a^b x f(x) dx = C_d ((1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)) / (d-1).
long double first_moment(int d, long double a, long double b) {
  long double cd = expl(lgammal(0.5L * d) - lgammal(0.5L * (d - 1))) / sqrtl(3.14159265358979323846264338327950288L);
  long double e = 0.5L * (d - 1);
  return cd * (powl(1.0L - a * a, e) - powl(1.0L - b * b, e)) / (d - 1);
}

// Lloyd-Max on the positive half-line (levels +-c_k), L = 2^(bits-1) levels:
// boundaries are midpoints, levels are cell means; iterate to a fixed point.
void lloyd_max(int d, int bits, std::vector<double>& c_out, std::vector<double>& t_out) {
  const int L = 1 << (bits - 1);
  std::vector<long double> c(L), t(L > 1 ? L - 1 : 0);
  const long double sd = 1.0L / sqrtl(static_cast<long double>(d));
  for (int k = 0; k < L; ++k) c[k] = sd * 3.0L * (k + 0.5L) / L;  // any positive increasing start
  for (int it = 0; it < 200000; ++it) {
    for (int k = 0; k + 1 < L; ++k) t[k] = 0.5L * (c[k] + c[k + 1]);
    long double delta = 0.0L;
    for (int k = 0; k < L; ++k) {
      long double a = (k == 0) ? 0.0L : t[k - 1];
      long double b = (k == L - 1) ? 1.0L : t[k];
      long double mass = half_mass(d, b) - half_mass(d, a);
      long double nc = first_moment(d, a, b) / mass;
      delta = fmaxl(delta, fabsl(nc - c[k]));
      c[k] = nc;
    }
    if (delta < 1e-16L) break;
  }
  for (int k = 0; k + 1 < L; ++k) t[k] = 0.5L * (c[k] + c[k + 1]);
  c_out.assign(c.begin(), c.end());
  t_out.assign(t.begin(), t.end());
}

// Lloyd-Max levels and boundaries of the angle phi = atan(r_o / r_e) between
// the radii of two blocks of k coordinates of a uniform direction, density
// proportional to sin^(k-1)(2 phi) on [0, pi/2]: cell masses and first
// moments by composite Simpson (double): iterated to a 1e-13 fixed point on a
// coarse rule, then polished on a rule 16 times finer (Simpson's error falls
// as the fourth power of the step) to a 1e-14 fixed point.
double angle_integral(int k, double a, double b, int order, int n /* even */) {
  const double h = (b - a) / n;
  double s = 0.0;
  for (int i = 0; i <= n; ++i) {
    const double x = a + h * i;
    const double f = std::pow(std::sin(2.0 * x), k - 1) * (order ? x : 1.0);
    s += f * ((i == 0 || i == n) ? 1.0 : ((i & 1) ? 4.0 : 2.0));
  }
  return s * h / 3.0;
}

}  // namespace

void angle_lloyd_max(int k, int bits, std::vector<double>& c_out, std::vector<double>& t_out) {
  const int L = 1 << bits;
  const double half_pi = 1.5707963267948966192;
  std::vector<double> c(L), t(L - 1);
  for (int j = 0; j < L; ++j) c[j] = half_pi * (j + 0.5) / L;
  for (int phase = 0; phase < 2; ++phase) {
    const int n = phase == 0 ? 1000 : 16000;
    const double tol = phase == 0 ? 1e-13 : 1e-14;
    for (int it = 0; it < 20000; ++it) {
      for (int j = 0; j + 1 < L; ++j) t[j] = 0.5 * (c[j] + c[j + 1]);
      double delta = 0.0;
      for (int j = 0; j < L; ++j) {
        const double a = (j == 0) ? 0.0 : t[j - 1];
        const double b = (j == L - 1) ? half_pi : t[j];
        const double nc = angle_integral(k, a, b, 1, n) / angle_integral(k, a, b, 0, n);
        delta = std::fmax(delta, std::fabs(nc - c[j]));
        c[j] = nc;
      }
      if (delta < tol) break;
    }
  }
  for (int j = 0; j + 1 < L; ++j) t[j] = 0.5 * (c[j] + c[j + 1]);
  c_out = c;
  t_out = t;
}

void sphere_lloyd_max(int d, int bits, std::vector<double>& c_out, std::vector<double>& t_out) {
  lloyd_max(d, bits, c_out, t_out);
}

namespace {

float round_to_half(double x) {
  // nearest fp16 value (ties to even), returned as float
  if (x == 0.0 || !std::isfinite(x)) return static_cast<float>(x);
  double a = std::fabs(x);
  int e = 0;
  std::frexp(a, &e);
  int lead = e - 1;
  if (lead < -14) lead = -14;
  double ulp = std::ldexp(1.0, lead - 10);
  double q = std::nearbyint(a / ulp);
  double r = q * ulp;
  if (r > 65504.0) r = INFINITY;
  return static_cast<float>(std::copysign(r, x));
}

}  // namespace

bool config_supported(const tq_config& c) {
  return (c.head_dim == 64 || c.head_dim == 128) && c.key_bits == 2 && c.qjl_dim == c.head_dim &&
         c.value_bits == 4 && c.page_tokens == TQ_PAGE_TOKENS;
}

bool config_valid(const tq_config& c) {
  return c.head_dim >= 16 && c.head_dim % 16 == 0 && c.head_dim <= 1024 && c.key_bits >= 1 &&
         c.key_bits <= 8 && c.value_bits >= 1 && c.value_bits <= 8 && c.qjl_dim >= 32 &&
         c.qjl_dim % 32 == 0 && c.page_tokens > 0;
}

bool generate_tables(const tq_config& cfg, HostTables& out) {
  const int d = cfg.head_dim, m = cfg.qjl_dim;
  std::vector<double> pi;
  if (!haar_rotation(d, cfg.seed, pi)) return false;
  out.rot.resize(static_cast<size_t>(d) * d);
  for (size_t i = 0; i < pi.size(); ++i) out.rot[i] = static_cast<float>(pi[i]);
  std::vector<double> s(static_cast<size_t>(m) * d);
  normal_stream(2ULL * cfg.seed + 1ULL, s);
  out.qjl.resize(s.size());
  for (size_t i = 0; i < s.size(); ++i) out.qjl[i] = round_to_half(s[i]);
  std::vector<double> c, t;
  lloyd_max(d, cfg.key_bits, c, t);
  out.key_c.assign(c.begin(), c.end());
  out.key_t.assign(t.begin(), t.end());
  lloyd_max(d, cfg.value_bits, c, t);
  out.val_c.assign(c.begin(), c.end());
  out.val_t.assign(t.begin(), t.end());
  return true;
}

}  // namespace tq
