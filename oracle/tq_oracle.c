/*
 * tq_oracle.c -- plain, slow CPU reference for TurboQuant-style KV-cache
 * compression, compressed-cache decode attention and compressed top-k search.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, imports or
 * runs this file; only the tests, the package's smoke check and the CPU
 * baseline of the benchmark do.  It shares no code with the CUDA library.
 *
 * Everything is computed in double precision.  Where a floating-point value
 * decides an integer (a quantiser code, a sign bit) the decision is taken in
 * the precision stated beside it, which is also the precision the GPU path
 * uses for that decision.
 *
 * Sources (web pages on the subject; sections as titled on each page):
 *  [TQ]   "TurboQuant" summary and discussion, de.news.hada.io topic 27867:
 *         "Funktionsweise von TurboQuant" (random rotation, then a standard
 *         per-coordinate quantiser; then 1-bit QJL on the residual),
 *         "QJL: Eine 1-Bit-Methode ohne Overhead" (JL transform, sign bits,
 *         estimator pairing a full-precision query with 1-bit data),
 *         the discussion's note that Lloyd-Max boundaries/reconstruction
 *         values are used after the rotation, and "Leistung bei der
 *         Vektorsuche" (inner-product search, top-k).
 *  [EXP]  "Die KV-Cache-Optimierung von Google erklaert", chatgpz.de:
 *         "Stufe 1: Die zufaellige Rotation", "Stufe 2: ... (quantisierte JL)"
 *         (unbiased estimator).
 *  [MON]  "Monarch v3: NES-inspiriertes KV-Paging", openclawradar.com:
 *         "Wie es funktioniert" (hot full-precision window, cold compressed
 *         region) and "Vereinfachte Decode-Schleife" (hot and cold scores,
 *         softmax, aggregation).
 *
 * Readings taken where the pages are silent:
 *  - rotation: dense Haar-orthogonal matrix = Q of a QR factorisation of a
 *    Gaussian matrix with diag(R) made positive;
 *  - quantiser: Lloyd-Max for the exact marginal of one coordinate of a
 *    uniform point on the unit sphere of R^d; a vector is normalised by its
 *    stored fp16 norm; sign-magnitude codes;
 *  - QJL: S has iid standard-normal entries rounded to fp16; estimator
 *    <q,r> ~ sqrt(pi/2)/m * |r| * <S q, sign(S r)>;
 *  - attention: one softmax over hot and cold tokens on every step.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* Random numbers: SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) giving     */
/* 53-bit uniforms, and the Box-Muller transform (1958) using both outputs. */
/* ------------------------------------------------------------------------ */
typedef struct {
  uint64_t state;
  int have_spare;
  double spare;
} or_rng;

static void rng_seed(or_rng* g, uint64_t seed) {
  g->state = seed;
  g->have_spare = 0;
  g->spare = 0.0;
}

static uint64_t rng_u64(or_rng* g) {
  g->state += 0x9E3779B97F4A7C15ULL;
  uint64_t z = g->state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static double rng_uniform(or_rng* g) { /* in [0, 1) */
  return (double)(rng_u64(g) >> 11) * 0x1.0p-53;
}

static double rng_normal(or_rng* g) {
  if (g->have_spare) {
    g->have_spare = 0;
    return g->spare;
  }
  double u1 = 1.0 - rng_uniform(g); /* (0, 1]: log is finite */
  double u2 = rng_uniform(g);
  double rad = sqrt(-2.0 * log(u1));
  double ang = 2.0 * M_PI * u2;
  g->spare = rad * sin(ang);
  g->have_spare = 1;
  return rad * cos(ang);
}

OR_API void or_normals(uint64_t seed, int64_t count, double* out) {
  or_rng g;
  rng_seed(&g, seed);
  for (int64_t i = 0; i < count; ++i) out[i] = rng_normal(&g);
}

OR_API void or_uniforms(uint64_t seed, int64_t count, double* out) {
  or_rng g;
  rng_seed(&g, seed);
  for (int64_t i = 0; i < count; ++i) out[i] = rng_uniform(&g);
}

/* ------------------------------------------------------------------------ */
/* Rounding to fp32 and fp16 (round to nearest, ties to even).              */
/* ------------------------------------------------------------------------ */
static double round_f32(double x) { return (double)(float)x; }

OR_API double or_round_f16(double x) {
  if (x == 0.0 || !isfinite(x)) return x;
  double a = fabs(x);
  if (a >= 65520.0) return copysign(INFINITY, x); /* beyond max + half ulp */
  int e;
  frexp(a, &e); /* a = f * 2^e, f in [0.5, 1) */
  int lead = e - 1; /* a in [2^lead, 2^(lead+1)) */
  if (lead < -14) lead = -14; /* subnormal range: fixed spacing 2^-24 */
  double ulp = ldexp(1.0, lead - 10);
  double q = nearbyint(a / ulp); /* exact quotient; default mode = ties-even */
  return copysign(q * ulp, x);
}

/* bit pattern of a value that is already exactly representable in fp16 */
static uint16_t f16_bits(double v) {
  uint16_t sign = signbit(v) ? 0x8000u : 0u;
  double a = fabs(v);
  if (a == 0.0) return sign;
  if (isinf(a)) return (uint16_t)(sign | 0x7C00u);
  if (isnan(a)) return 0x7E00u;
  if (a < 0x1.0p-14) { /* subnormal: a = mant * 2^-24 */
    return (uint16_t)(sign | (uint16_t)(a * 0x1.0p24));
  }
  int e;
  double f = frexp(a, &e); /* a = f*2^e, f in [0.5,1) -> 1.m * 2^(e-1) */
  int biased = (e - 1) + 15;
  uint16_t mant = (uint16_t)((f * 2.0 - 1.0) * 1024.0);
  return (uint16_t)(sign | (uint16_t)(biased << 10) | mant);
}

static double f16_value(uint16_t h) {
  int sign = (h >> 15) & 1;
  int ex = (h >> 10) & 0x1F;
  int mant = h & 0x3FF;
  double v;
  if (ex == 0)
    v = ldexp((double)mant, -24);
  else if (ex == 31)
    v = mant ? NAN : INFINITY;
  else
    v = ldexp(1.0 + mant / 1024.0, ex - 15);
  return sign ? -v : v;
}

OR_API uint16_t or_f16_bits(double v) { return f16_bits(or_round_f16(v)); }
OR_API double or_f16_value(uint16_t h) { return f16_value(h); }

/* ------------------------------------------------------------------------ */
/* Random rotation [TQ "Funktionsweise", EXP "Stufe 1"]:                    */
/* G (d x d, filled row by row from the normal stream 2*seed) = Q R by      */
/* Householder reflections; Pi = Q diag(sign(R_ii)).  x_rot = Pi x.         */
/* ------------------------------------------------------------------------ */
OR_API int or_rotation(int d, uint64_t seed, double* pi /* d*d row-major */) {
  double* a = (double*)malloc(sizeof(double) * d * d); /* becomes R */
  double* q = (double*)malloc(sizeof(double) * d * d); /* accumulates Q */
  double* v = (double*)malloc(sizeof(double) * d);
  if (!a || !q || !v) {
    free(a); free(q); free(v);
    return -1;
  }
  or_rng g;
  rng_seed(&g, 2ULL * seed);
  for (int i = 0; i < d * d; ++i) a[i] = rng_normal(&g);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) q[i * d + j] = (i == j) ? 1.0 : 0.0;

  for (int k = 0; k < d - 1; ++k) {
    /* Householder vector for column k, rows k..d-1 */
    double norm = 0.0;
    for (int i = k; i < d; ++i) norm += a[i * d + k] * a[i * d + k];
    norm = sqrt(norm);
    if (norm == 0.0) continue;
    double alpha = (a[k * d + k] > 0.0) ? -norm : norm;
    for (int i = 0; i < d; ++i) v[i] = 0.0;
    for (int i = k; i < d; ++i) v[i] = a[i * d + k];
    v[k] -= alpha;
    double vv = 0.0;
    for (int i = k; i < d; ++i) vv += v[i] * v[i];
    if (vv == 0.0) continue;
    /* A <- H A, H = I - 2 v v^T / (v^T v) */
    for (int j = 0; j < d; ++j) {
      double dot = 0.0;
      for (int i = k; i < d; ++i) dot += v[i] * a[i * d + j];
      double f = 2.0 * dot / vv;
      for (int i = k; i < d; ++i) a[i * d + j] -= f * v[i];
    }
    /* Q <- Q H */
    for (int i = 0; i < d; ++i) {
      double dot = 0.0;
      for (int j = k; j < d; ++j) dot += q[i * d + j] * v[j];
      double f = 2.0 * dot / vv;
      for (int j = k; j < d; ++j) q[i * d + j] -= f * v[j];
    }
  }
  /* Pi = Q diag(sign(R_jj)) */
  for (int j = 0; j < d; ++j) {
    double s = (a[j * d + j] < 0.0) ? -1.0 : 1.0;
    for (int i = 0; i < d; ++i) pi[i * d + j] = q[i * d + j] * s;
  }
  free(a); free(q); free(v);
  return 0;
}

/* QJL matrix S (m x d): normal stream 2*seed+1, row-major, each entry
 * rounded to the nearest fp16 value [TQ "QJL"; rounding is a reading]. */
OR_API void or_qjl_matrix(int m, int d, uint64_t seed, double* s) {
  or_rng g;
  rng_seed(&g, 2ULL * seed + 1ULL);
  for (int i = 0; i < m * d; ++i) s[i] = or_round_f16(rng_normal(&g));
}

/* ------------------------------------------------------------------------ */
/* Lloyd-Max codebook for the coordinate marginal of a uniform unit vector  */
/* [TQ discussion: Lloyd-Max boundaries and reconstruction values after the */
/* rotation].  f(x) = C_d (1-x^2)^((d-3)/2) on [-1, 1],                     */
/* C_d = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)).                            */
/* ------------------------------------------------------------------------ */
#define GL_N 24
static double gl_x[GL_N], gl_w[GL_N];
static int gl_ready = 0;

/* Gauss-Legendre nodes: roots of P_n by Newton's method, w = 2/((1-x^2)P_n'^2) */
static void gl_init(void) {
  if (gl_ready) return;
  int n = GL_N;
  for (int i = 0; i < n; ++i) {
    double x = cos(M_PI * (i + 0.75) / (n + 0.5));
    double dp = 0.0;
    for (int it = 0; it < 100; ++it) {
      double p0 = 1.0, p1 = x;
      for (int k = 2; k <= n; ++k) {
        double p2 = ((2.0 * k - 1.0) * x * p1 - (k - 1.0) * p0) / k;
        p0 = p1;
        p1 = p2;
      }
      dp = n * (x * p1 - p0) / (x * x - 1.0);
      double dx = p1 / dp;
      x -= dx;
      if (fabs(dx) < 1e-16) break;
    }
    /* recompute derivative at the converged node */
    double p0 = 1.0, p1 = x;
    for (int k = 2; k <= n; ++k) {
      double p2 = ((2.0 * k - 1.0) * x * p1 - (k - 1.0) * p0) / k;
      p0 = p1;
      p1 = p2;
    }
    dp = n * (x * p1 - p0) / (x * x - 1.0);
    gl_x[i] = x;
    gl_w[i] = 2.0 / ((1.0 - x * x) * dp * dp);
  }
  gl_ready = 1;
}

/* C_d = r(d)/sqrt(pi) with r(d) = Gamma(d/2)/Gamma((d-1)/2), from
 * r(2) = 1/sqrt(pi), r(3) = sqrt(pi)/2 and r(d+2) = r(d) d/(d-1). */
static double sphere_cd(int d) {
  double r = (d % 2 == 0) ? 1.0 / sqrt(M_PI) : sqrt(M_PI) / 2.0;
  for (int k = (d % 2 == 0) ? 2 : 3; k < d; k += 2) r *= (double)k / (double)(k - 1);
  return r / sqrt(M_PI);
}

static double sphere_pdf(int d, double cd, double x) {
  double t = 1.0 - x * x;
  if (t <= 0.0) return 0.0;
  return cd * pow(t, 0.5 * (d - 3));
}

static double gl_panel(int d, double cd, double a, double b) {
  double h = 0.5 * (b - a), c = 0.5 * (a + b), s = 0.0;
  for (int i = 0; i < GL_N; ++i) s += gl_w[i] * sphere_pdf(d, cd, c + h * gl_x[i]);
  return s * h;
}

/* probability mass of [a, b] under the sphere marginal: composite
 * Gauss-Legendre on panels no wider than a quarter of the density's scale
 * 1/sqrt(d); the range where the density is below ~1e-300 is skipped. */
OR_API double or_sphere_mass(int d, double a, double b) {
  gl_init();
  double cd = sphere_cd(d);
  double xmax = (d > 3) ? sqrt(1500.0 / (d - 3)) : 1.0;
  if (xmax > 1.0) xmax = 1.0;
  if (a < -xmax) a = -xmax;
  if (b > xmax) b = xmax;
  if (b <= a) return 0.0;
  double h = fmin(1.0 / 64.0, 0.25 / sqrt((double)d));
  int panels = (int)ceil((b - a) / h);
  double total = 0.0;
  for (int i = 0; i < panels; ++i) {
    double lo = a + (b - a) * i / panels, hi = a + (b - a) * (i + 1) / panels;
    total += gl_panel(d, cd, lo, hi);
  }
  return total;
}

/* first moment of [a, b] in closed form: int x f(x) dx */
OR_API double or_sphere_first_moment(int d, double a, double b) {
  double cd = sphere_cd(d);
  double e = 0.5 * (d - 1);
  return cd * (pow(1.0 - a * a, e) - pow(1.0 - b * b, e)) / (d - 1);
}

/*
 * Lloyd-Max on the positive half (the density is symmetric, so the
 * quantiser is too: levels +-c[k]).  L = 2^(bits-1) positive levels;
 * positive boundaries t[k] = (c[k] + c[k+1]) / 2, k < L-1; the cell of c[0]
 * is [0, t[0]], that of c[L-1] is [t[L-2], 1].  Start: quantiles of the
 * normal approximation N(0, 1/d); iterate centroid/boundary updates until
 * max |delta c| < 1e-15 (at most max_iter rounds).  Returns iterations used.
 */
static double norm_quantile(double p) { /* bisection on the normal CDF */
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 200; ++i) {
    double mid = 0.5 * (lo + hi);
    if (0.5 * erfc(-mid / sqrt(2.0)) < p) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

OR_API int or_lloyd_max(int d, int bits, int max_iter, double* c /* L */, double* t /* L-1 */,
                        double* mse_out) {
  int L = 1 << (bits - 1);
  for (int k = 0; k < L; ++k)
    c[k] = norm_quantile((L + k + 0.5) / (2.0 * L)) / sqrt((double)d);
  int it = 0;
  for (; it < max_iter; ++it) {
    for (int k = 0; k + 1 < L; ++k) t[k] = 0.5 * (c[k] + c[k + 1]);
    double delta = 0.0;
    for (int k = 0; k < L; ++k) {
      double a = (k == 0) ? 0.0 : t[k - 1];
      double b = (k == L - 1) ? 1.0 : t[k];
      double nc = or_sphere_first_moment(d, a, b) / or_sphere_mass(d, a, b);
      delta = fmax(delta, fabs(nc - c[k]));
      c[k] = nc;
    }
    if (delta < 1e-15) { ++it; break; }
  }
  for (int k = 0; k + 1 < L; ++k) t[k] = 0.5 * (c[k] + c[k + 1]);
  if (mse_out) {
    /* E[(X - Q(X))^2] = E[X^2] - sum over both signs of P(cell) c^2, valid
     * at a centroid fixed point; E[X^2] = 1/d for a unit-sphere coordinate */
    double s = 0.0;
    for (int k = 0; k < L; ++k) {
      double a = (k == 0) ? 0.0 : t[k - 1];
      double b = (k == L - 1) ? 1.0 : t[k];
      s += 2.0 * or_sphere_mass(d, a, b) * c[k] * c[k];
    }
    *mse_out = 1.0 / d - s;
  }
  return it;
}

/* ------------------------------------------------------------------------ */
/* Page format (storage layout of the cold tier; 128 token slots per page). */
/* The format is this library's own (the pages fix none).  Two kinds:       */
/*                                                                          */
/* Keys-only pages (a search database): the record layout.  Sections in     */
/* order, each starting on a 16-byte boundary:                              */
/*   KC key codes    128 x d/4 bytes   (2-bit codes: sign and magnitude)    */
/*   QS QJL signs    128 x m/8 bytes                                        */
/*   KN key norm     128 x fp16                                             */
/*   KG residual norm 128 x fp16                                            */
/* Key code word w (little-endian u32, w < d/16) of a token holds           */
/* coordinates j = 16w + 8h + r (h in {0,1}, r = 2i + e < 8): sign bit at   */
/* 16h + 15 - 4i - e, magnitude bit at 16h + 13 - 4i - e.                   */
/* QJL word w (w < m/32) holds sketch index i = 32w + 16h + r (r < 16) at   */
/* bit 16h + 15 - r.                                                        */
/*                                                                          */
/* Pages with values (the decode's cold tier): 8 blocks of 16 token slots   */
/* (block kb = slot/16, t = slot mod 16), each 12d + 2m + 96 bytes:         */
/*   KH key plane H  2d bytes   at 0                                        */
/*   KL key plane L  2d bytes   at 2d                                       */
/*   QS QJL signs    2m bytes   at 4d                                       */
/*   VC value codes  8d bytes   at 4d + 2m                                  */
/*   NK key norm n and residual norm, fp16 pairs (n, gamma) per token, at   */
/*      12d + 2m + 4t                                                       */
/*   VN value norm fp16 at 12d + 2m + 64 + 2t                               */
/* The key code is the index u = 2H + L of the level in ascending order     */
/* (-c1, -c0, +c0, +c1): H = 1 - sign, L = sign XOR magnitude.  In a plane  */
/* (index j < d for H and L, sketch index j < m for QS), the bit of token t */
/* is bit t mod 8 of the byte at                                           */
/*   16 (4 (j/32) + (j/4) mod 4) + 4 (2 ((j/16) mod 2) + t/8) + j mod 4     */
/* so that a 32-bit word holds 4 consecutive indices x 8 tokens.            */
/* Value codes (a code is sign<<3 | magnitude index, 0..7): one byte holds  */
/* two tokens of one coordinate, the even token in the low nibble.  With    */
/* i = j/16, g = j mod 8, jh = (j mod 16)/8, pair q = t/2, c = q mod 4,     */
/* th = q/4, the byte sits at                                               */
/*   (i/4)*512 + (4g + c)*16 + (i mod 4)*4 + jh + 2*th                      */
/* of the block's VC section, so that the 32-bit word at (4g + c)*16 +      */
/* (i mod 4)*4 holds, in its four bytes, coordinates (g, g+8) x token       */
/* pairs (c, c+4).                                                          */
/* ------------------------------------------------------------------------ */
#define PAGE_TOKENS 128
#define BLOCK_TOKENS 16

typedef struct {
  /* record layout: section offsets; block layout: offsets inside a block */
  size_t kc, kl, qs, vc, kn, kg, vn, block, bytes;
} or_layout;

static size_t up16(size_t x) { return (x + 15) & ~(size_t)15; }

static or_layout layout_of(int d, int m, int with_values) {
  or_layout L;
  memset(&L, 0, sizeof(L));
  if (with_values) {
    L.kc = 0;
    L.kl = (size_t)2 * d;
    L.qs = (size_t)4 * d;
    L.vc = (size_t)4 * d + (size_t)2 * m;
    L.kn = (size_t)12 * d + (size_t)2 * m;
    L.kg = L.kn + 2;
    L.vn = L.kn + 64;
    L.block = L.kn + 96;
    L.bytes = (PAGE_TOKENS / BLOCK_TOKENS) * L.block;
    return L;
  }
  size_t off = 0;
  L.kc = off; off = up16(off + (size_t)PAGE_TOKENS * d / 4);
  L.qs = off; off = up16(off + (size_t)PAGE_TOKENS * m / 8);
  L.kn = off; off = up16(off + 2 * PAGE_TOKENS);
  L.kg = off; off = up16(off + 2 * PAGE_TOKENS);
  L.bytes = off;
  return L;
}

/* offs (8 or NULL): kc, qs, vc, kn, kg, vn, block bytes (0: record layout),
 * kl.  Block layout: kc = KH, kn and kg the fields of token 0 of block 0. */
OR_API size_t or_page_layout(int d, int m, int with_values, size_t* offs) {
  or_layout L = layout_of(d, m, with_values);
  if (offs) {
    offs[0] = L.kc; offs[1] = L.qs; offs[2] = L.vc;
    offs[3] = L.kn; offs[4] = L.kg; offs[5] = L.vn;
    offs[6] = L.block; offs[7] = L.kl;
  }
  return L.bytes;
}

static uint32_t rd32(const uint8_t* p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
static void wr32(uint8_t* p, uint32_t v) {
  p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); p[2] = (uint8_t)(v >> 16); p[3] = (uint8_t)(v >> 24);
}
static uint16_t rd16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static void wr16(uint8_t* p, uint16_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }

static int kc_sign_bit(int j) { /* record layout: position inside word j/16 */
  int h = (j % 16) / 8, r = j % 8, i = r / 2, e = r % 2;
  return 16 * h + 15 - 4 * i - e;
}
static int kc_mag_bit(int j) { return kc_sign_bit(j) - 2; }
static int qs_bit(int i) { /* record layout: position inside word i/32 */
  int h = (i % 32) / 16, r = i % 16;
  return 16 * h + 15 - r;
}

/* block layout: byte of plane index j for token t (bit t mod 8) */
static size_t plane_byte(int j, int t) {
  return (size_t)16 * (4 * (j / 32) + (j / 4) % 4) + (size_t)4 * (2 * ((j / 16) % 2) + t / 8) +
         (size_t)(j % 4);
}
static void put_bit(uint8_t* p, int bit, int v) {
  *p = (uint8_t)(v ? (*p | (1u << bit)) : (*p & ~(1u << bit)));
}

/* block layout: offset, inside a block's value section, of the byte holding
 * token t (slot mod 16) of coordinate j */
static size_t vc_pos(int t, int j) {
  int q = t / 2, c = q % 4, th = q / 4;
  int i = j / 16, g = j % 8, jh = (j % 16) / 8;
  return (size_t)(i / 4) * 512 + (size_t)(4 * g + c) * 16 + (size_t)(i % 4) * 4 +
         (size_t)(jh + 2 * th);
}

/* write one key record into token slot `slot` of page `pg` */
OR_API void or_pack_key(uint8_t* pg, int d, int m, int with_values, int slot,
                        const int32_t* sign, const int32_t* mag, const int32_t* qbits,
                        double n, double gamma) {
  or_layout L = layout_of(d, m, with_values);
  if (with_values) {
    uint8_t* bk = pg + (size_t)(slot / BLOCK_TOKENS) * L.block;
    int t = slot % BLOCK_TOKENS;
    for (int j = 0; j < d; ++j) {
      put_bit(bk + L.kc + plane_byte(j, t), t % 8, !sign[j]);
      put_bit(bk + L.kl + plane_byte(j, t), t % 8, (sign[j] != 0) != (mag[j] != 0));
    }
    for (int i = 0; i < m; ++i) put_bit(bk + L.qs + plane_byte(i, t), t % 8, qbits[i] != 0);
    wr16(bk + L.kn + 4 * t, f16_bits(or_round_f16(n)));
    wr16(bk + L.kg + 4 * t, f16_bits(or_round_f16(gamma)));
    return;
  }
  uint8_t* kc = pg + L.kc + (size_t)slot * (d / 4);
  for (int w = 0; w < d / 16; ++w) {
    uint32_t word = 0;
    for (int j = 16 * w; j < 16 * w + 16; ++j) {
      if (sign[j]) word |= 1u << kc_sign_bit(j);
      if (mag[j]) word |= 1u << kc_mag_bit(j);
    }
    wr32(kc + 4 * w, word);
  }
  uint8_t* qs = pg + L.qs + (size_t)slot * (m / 8);
  for (int w = 0; w < m / 32; ++w) {
    uint32_t word = 0;
    for (int i = 32 * w; i < 32 * w + 32; ++i)
      if (qbits[i]) word |= 1u << qs_bit(i);
    wr32(qs + 4 * w, word);
  }
  wr16(pg + L.kn + 2 * slot, f16_bits(or_round_f16(n)));
  wr16(pg + L.kg + 2 * slot, f16_bits(or_round_f16(gamma)));
}

OR_API void or_unpack_key(const uint8_t* pg, int d, int m, int with_values, int slot,
                          int32_t* sign, int32_t* mag, int32_t* qbits, double* n, double* gamma) {
  or_layout L = layout_of(d, m, with_values);
  if (with_values) {
    const uint8_t* bk = pg + (size_t)(slot / BLOCK_TOKENS) * L.block;
    int t = slot % BLOCK_TOKENS;
    for (int j = 0; j < d; ++j) {
      int h = (bk[L.kc + plane_byte(j, t)] >> (t % 8)) & 1;
      int l = (bk[L.kl + plane_byte(j, t)] >> (t % 8)) & 1;
      sign[j] = 1 - h;
      mag[j] = l ^ sign[j];
    }
    for (int i = 0; i < m; ++i) qbits[i] = (bk[L.qs + plane_byte(i, t)] >> (t % 8)) & 1;
    *n = f16_value(rd16(bk + L.kn + 4 * t));
    *gamma = f16_value(rd16(bk + L.kg + 4 * t));
    return;
  }
  const uint8_t* kc = pg + L.kc + (size_t)slot * (d / 4);
  for (int j = 0; j < d; ++j) {
    uint32_t word = rd32(kc + 4 * (j / 16));
    sign[j] = (word >> kc_sign_bit(j)) & 1u;
    mag[j] = (word >> kc_mag_bit(j)) & 1u;
  }
  const uint8_t* qs = pg + L.qs + (size_t)slot * (m / 8);
  for (int i = 0; i < m; ++i) qbits[i] = (rd32(qs + 4 * (i / 32)) >> qs_bit(i)) & 1u;
  *n = f16_value(rd16(pg + L.kn + 2 * slot));
  *gamma = f16_value(rd16(pg + L.kg + 2 * slot));
}

/* value record (pages with values): code = sign<<3 | magnitude index */
OR_API void or_pack_value(uint8_t* pg, int d, int m, int slot, const int32_t* code, double n) {
  or_layout L = layout_of(d, m, 1);
  uint8_t* bk = pg + (size_t)(slot / BLOCK_TOKENS) * L.block;
  int t = slot % BLOCK_TOKENS, hi = t & 1;
  for (int j = 0; j < d; ++j) {
    uint8_t* bp = bk + L.vc + vc_pos(t, j);
    uint8_t c = (uint8_t)(code[j] & 0xF);
    *bp = hi ? (uint8_t)((*bp & 0x0F) | (c << 4)) : (uint8_t)((*bp & 0xF0) | c);
  }
  wr16(bk + L.vn + 2 * t, f16_bits(or_round_f16(n)));
}

OR_API void or_unpack_value(const uint8_t* pg, int d, int m, int slot, int32_t* code, double* n) {
  or_layout L = layout_of(d, m, 1);
  const uint8_t* bk = pg + (size_t)(slot / BLOCK_TOKENS) * L.block;
  int t = slot % BLOCK_TOKENS;
  for (int j = 0; j < d; ++j) {
    uint8_t b = bk[L.vc + vc_pos(t, j)];
    code[j] = (t & 1) ? (b >> 4) : (b & 0xF);
  }
  *n = f16_value(rd16(bk + L.vn + 2 * t));
}

/* batched forms: record v goes to page page_id[v], slot slot[v].
 * key arrays: sign/mag [N*d], qbits [N*m], n, gamma [N];
 * value arrays (with_values): vcode [N*d], vn [N]; may be NULL for keys-only. */
OR_API void or_pack_batch(uint8_t* pool, size_t page_bytes, int d, int m, int with_values,
                          int64_t N, const int32_t* page_id, const int32_t* slot,
                          const int32_t* sign, const int32_t* mag, const int32_t* qbits,
                          const double* n, const double* gamma, const int32_t* vcode,
                          const double* vn) {
  for (int64_t v = 0; v < N; ++v) {
    uint8_t* pg = pool + (size_t)page_id[v] * page_bytes;
    or_pack_key(pg, d, m, with_values, slot[v], sign + (size_t)v * d, mag + (size_t)v * d,
                qbits + (size_t)v * m, n[v], gamma[v]);
    if (with_values && vcode) or_pack_value(pg, d, m, slot[v], vcode + (size_t)v * d, vn[v]);
  }
}

OR_API void or_unpack_batch(const uint8_t* pool, size_t page_bytes, int d, int m,
                            int with_values, int64_t N, const int32_t* page_id,
                            const int32_t* slot, int32_t* sign, int32_t* mag, int32_t* qbits,
                            double* n, double* gamma, int32_t* vcode, double* vn) {
  for (int64_t v = 0; v < N; ++v) {
    const uint8_t* pg = pool + (size_t)page_id[v] * page_bytes;
    or_unpack_key(pg, d, m, with_values, slot[v], sign + (size_t)v * d, mag + (size_t)v * d,
                  qbits + (size_t)v * m, n + v, gamma + v);
    if (with_values && vcode) or_unpack_value(pg, d, m, slot[v], vcode + (size_t)v * d, vn + v);
  }
}

/* ------------------------------------------------------------------------ */
/* Encoding one vector [TQ "Funktionsweise" steps 1 and 2; EXP "Stufe 1/2"] */
/* ------------------------------------------------------------------------ */
/*
 * x_rot: the rotated vector as fp32 values (Pi x rounded to fp32, or the
 * caller's pre-rotated input); xnorm: the Euclidean norm of the vector.
 * n = fp16(xnorm).  Per coordinate, in fp32: T_k = fp32(n * t_k);
 * sign = [x_rot_j < 0]; magnitude index = #{k : |x_rot_j| >= T_k}.
 * Reconstruction c_hat_j = (+-) c[idx] in the normalised domain.
 * Keys only: residual r = x_rot / n - c_hat (double); gamma = fp16(|r|);
 * QJL bit i = [(S r)_i < 0] (double).
 */
static void encode_one(int d, int m, const double* S, const double* cpos, const double* tpos, int L,
                       const double* x_rot, double xnorm, int is_key, int32_t* sign, int32_t* mag,
                       int32_t* qbits, double* n_out, double* gamma_out, double* r_scratch) {
  double n = or_round_f16(xnorm);
  *n_out = n;
  if (gamma_out) *gamma_out = 0.0;
  if (n == 0.0 || !isfinite(n)) {
    for (int j = 0; j < d; ++j) { sign[j] = 0; mag[j] = 0; }
    if (is_key) for (int i = 0; i < m; ++i) qbits[i] = 0;
    return;
  }
  float nf = (float)n;
  for (int j = 0; j < d; ++j) {
    float xj = (float)x_rot[j];
    sign[j] = (xj < 0.0f) ? 1 : 0;
    float ax = fabsf(xj);
    int idx = 0;
    for (int k = 0; k + 1 < L; ++k) {
      float thr = nf * (float)tpos[k]; /* one fp32 product, rounded */
      if (ax >= thr) idx = k + 1;
    }
    mag[j] = idx;
  }
  if (!is_key) return;
  double rr = 0.0;
  for (int j = 0; j < d; ++j) {
    double ch = (sign[j] ? -1.0 : 1.0) * cpos[mag[j]];
    r_scratch[j] = x_rot[j] / n - ch;
    rr += r_scratch[j] * r_scratch[j];
  }
  *gamma_out = or_round_f16(sqrt(rr));
  for (int i = 0; i < m; ++i) {
    double p = 0.0;
    for (int j = 0; j < d; ++j) p += S[(size_t)i * d + j] * r_scratch[j];
    qbits[i] = (p < 0.0) ? 1 : 0;
  }
}

/*
 * Encode N vectors.  rotated = 0: x is the raw input (values exactly as
 * stored, e.g. bf16 widened), x_rot = fp32(Pi x) and xnorm = |x|.
 * rotated = 1: x already holds fp32 rotated values; xnorm = |x|.
 * Outputs: sign/mag [N*d], qbits [N*m] (keys), n [N], gamma [N] (keys),
 * xrot_out [N*d] (the fp32 rotated values used, may be NULL).
 */
OR_API void or_encode(int d, int m, const double* pi, const double* S, const double* cpos,
                      const double* tpos, int L, const double* x, int64_t N, int rotated,
                      int is_key, int32_t* sign, int32_t* mag, int32_t* qbits, double* n,
                      double* gamma, double* xrot_out, int threads) {
#ifdef _OPENMP
  const int nthreads = threads > 0 ? threads : omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
  {
    double* xr = (double*)malloc(sizeof(double) * d);
    double* rs = (double*)malloc(sizeof(double) * d);
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
    for (int64_t v = 0; v < N; ++v) {
      const double* xv = x + (size_t)v * d;
      double ss = 0.0;
      for (int j = 0; j < d; ++j) ss += xv[j] * xv[j];
      for (int j = 0; j < d; ++j) {
        if (rotated) {
          xr[j] = round_f32(xv[j]);
        } else {
          double acc = 0.0;
          for (int k = 0; k < d; ++k) acc += pi[(size_t)j * d + k] * xv[k];
          xr[j] = round_f32(acc);
        }
      }
      if (xrot_out) memcpy(xrot_out + (size_t)v * d, xr, sizeof(double) * d);
      encode_one(d, m, S, cpos, tpos, L, xr, sqrt(ss), is_key, sign + (size_t)v * d,
                 mag + (size_t)v * d, is_key ? qbits + (size_t)v * m : NULL, n + v,
                 is_key ? gamma + v : NULL, rs);
    }
    free(xr);
    free(rs);
  }
}

/* ------------------------------------------------------------------------ */
/* Estimators [TQ "QJL", EXP "Stufe 2"].                                     */
/* ------------------------------------------------------------------------ */
/* <q, r> ~ sqrt(pi/2)/m * gamma * sum_i (S q)_i * (1 - 2 bit_i) */
OR_API double or_qjl_estimate(int m, const double* sq /* S q, m */, const int32_t* qbits,
                              double gamma) {
  double acc = 0.0;
  for (int i = 0; i < m; ++i) acc += qbits[i] ? -sq[i] : sq[i];
  return sqrt(M_PI / 2.0) / m * gamma * acc;
}

/* Monte-Carlo check helper: for trial t, S_t = or_qjl_matrix(seed0 + t);
 * returns the sample mean and (unbiased) sample variance of the estimate of
 * <q, r> with the exact |r| as gamma. */
OR_API void or_qjl_montecarlo(int d, int m, const double* q, const double* r, int64_t trials,
                              uint64_t seed0, double* mean, double* var) {
  double* S = (double*)malloc(sizeof(double) * m * d);
  double* sq = (double*)malloc(sizeof(double) * m);
  int32_t* bits = (int32_t*)malloc(sizeof(int32_t) * m);
  double rn = 0.0;
  for (int j = 0; j < d; ++j) rn += r[j] * r[j];
  rn = sqrt(rn);
  double s1 = 0.0, s2 = 0.0;
  for (int64_t t = 0; t < trials; ++t) {
    or_qjl_matrix(m, d, seed0 + (uint64_t)t, S);
    for (int i = 0; i < m; ++i) {
      double a = 0.0, b = 0.0;
      for (int j = 0; j < d; ++j) {
        a += S[(size_t)i * d + j] * q[j];
        b += S[(size_t)i * d + j] * r[j];
      }
      sq[i] = a;
      bits[i] = (b < 0.0) ? 1 : 0;
    }
    double e = or_qjl_estimate(m, sq, bits, rn);
    s1 += e;
    s2 += e * e;
  }
  *mean = s1 / trials;
  *var = (s2 - s1 * s1 / trials) / (trials - 1);
  free(S); free(sq); free(bits);
}

/* estimated score of a stored key against a query (scale applied):
 * n * ( <q_rot, c_hat> + sqrt(pi/2)/m * gamma * <S q_rot, 1-2 bits> ) * scale */
static double key_score(int d, int m, const double* qrot, const double* sq, const double* cpos,
                        const int32_t* sign, const int32_t* mag, const int32_t* qbits, double n,
                        double gamma, double scale) {
  double ip = 0.0;
  for (int j = 0; j < d; ++j) ip += qrot[j] * (sign[j] ? -cpos[mag[j]] : cpos[mag[j]]);
  return n * (ip + or_qjl_estimate(m, sq, qbits, gamma)) * scale;
}

/* Estimated scores of the cold tokens of one (batch, kv head) group for G
 * query heads, exactly as the decode attention forms them (key_score with the
 * scale applied): q [G, d] (original domain), pages / cold_len as the group's
 * page table row and length; out [G, cold_len]. */
OR_API void or_cold_logits(int d, int m, const double* pi, const double* S, const double* kcpos,
                           int G, const double* q, double scale, const uint8_t* pool,
                           size_t page_bytes, const int32_t* pages, int cold_len, double* out) {
  double* qrot = (double*)malloc(sizeof(double) * (size_t)G * d);
  double* sq = (double*)malloc(sizeof(double) * (size_t)G * m);
  int32_t* sign = (int32_t*)malloc(sizeof(int32_t) * d);
  int32_t* mag = (int32_t*)malloc(sizeof(int32_t) * d);
  int32_t* qb = (int32_t*)malloc(sizeof(int32_t) * m);
  for (int h = 0; h < G; ++h) {
    for (int j = 0; j < d; ++j) {
      double a = 0.0;
      for (int k = 0; k < d; ++k) a += pi[(size_t)j * d + k] * q[(size_t)h * d + k];
      qrot[(size_t)h * d + j] = a;
    }
    for (int i = 0; i < m; ++i) {
      double a = 0.0;
      for (int j = 0; j < d; ++j) a += S[(size_t)i * d + j] * qrot[(size_t)h * d + j];
      sq[(size_t)h * m + i] = a;
    }
  }
  for (int t = 0; t < cold_len; ++t) {
    const uint8_t* pg = pool + (size_t)pages[t / PAGE_TOKENS] * page_bytes;
    double n, gamma;
    or_unpack_key(pg, d, m, 1, t % PAGE_TOKENS, sign, mag, qb, &n, &gamma);
    for (int h = 0; h < G; ++h)
      out[(size_t)h * cold_len + t] = key_score(d, m, qrot + (size_t)h * d, sq + (size_t)h * m,
                                                 kcpos, sign, mag, qb, n, gamma, scale);
  }
  free(qrot); free(sq); free(sign); free(mag); free(qb);
}

/* ------------------------------------------------------------------------ */
/* Decode attention over one (batch, kv head) group [MON "Vereinfachte      */
/* Decode-Schleife": hot scores, cold scores, softmax, aggregation].         */
/* One softmax over cold tokens (estimated scores, reconstructed values      */
/* v_hat = n_v Pi^T c_hat_v) followed by hot tokens (exact fp16 keys and     */
/* values).  Two-pass softmax.  q: [G, d]; out: [G, d].                      */
/* ------------------------------------------------------------------------ */
/*
 * Threshold gate [MON "Vereinfachte Decode-Schleife": the cold pages are
 * decompressed and scored only if max(scores_hot) < threshold].  Reading: the
 * test is taken per query head on the raw hot scores <q, k_t> (the product
 * q @ kv_hot.T as written, no softmax scale); with no hot tokens the maximum
 * is -inf.  A head whose test fails attends to its hot tokens alone.  With
 * gated = 0 every head reads the cold tokens.  open (may be NULL) receives
 * per head the gate's decision: 1 if the head reads its cold tokens (whether
 * or not there are any), else 0.
 */
OR_API int or_attention_group(int d, int m, const double* pi, const double* S,
                              const double* kcpos, const double* vcpos, int G,
                              const double* q, double scale, const double* k_hot,
                              const double* v_hot, int hot_len, const uint8_t* pool,
                              size_t page_bytes, const int32_t* pages, int cold_len,
                              int gated, double threshold, int32_t* open, double* out) {
  int nt = cold_len + hot_len;
  double* logits = (double*)malloc(sizeof(double) * (size_t)G * (nt > 0 ? nt : 1));
  double* vals = (double*)malloc(sizeof(double) * (size_t)(nt > 0 ? nt : 1) * d);
  double* qrot = (double*)malloc(sizeof(double) * (size_t)G * d);
  double* sq = (double*)malloc(sizeof(double) * (size_t)G * m);
  int32_t* sign = (int32_t*)malloc(sizeof(int32_t) * d);
  int32_t* mag = (int32_t*)malloc(sizeof(int32_t) * d);
  int32_t* qb = (int32_t*)malloc(sizeof(int32_t) * m);
  int32_t* vcode = (int32_t*)malloc(sizeof(int32_t) * d);
  double* chat = (double*)malloc(sizeof(double) * d);
  if (!logits || !vals || !qrot || !sq || !sign || !mag || !qb || !vcode || !chat) return -1;

  for (int h = 0; h < G; ++h) {
    for (int j = 0; j < d; ++j) {
      double a = 0.0;
      for (int k = 0; k < d; ++k) a += pi[(size_t)j * d + k] * q[(size_t)h * d + k];
      qrot[(size_t)h * d + j] = a;
    }
    for (int i = 0; i < m; ++i) {
      double a = 0.0;
      for (int j = 0; j < d; ++j) a += S[(size_t)i * d + j] * qrot[(size_t)h * d + j];
      sq[(size_t)h * m + i] = a;
    }
  }
  for (int t = 0; t < cold_len; ++t) {
    const uint8_t* pg = pool + (size_t)pages[t / PAGE_TOKENS] * page_bytes;
    int slot = t % PAGE_TOKENS;
    double n, gamma, nv;
    or_unpack_key(pg, d, m, 1, slot, sign, mag, qb, &n, &gamma);
    for (int h = 0; h < G; ++h)
      logits[(size_t)h * nt + t] = key_score(d, m, qrot + (size_t)h * d, sq + (size_t)h * m,
                                             kcpos, sign, mag, qb, n, gamma, scale);
    or_unpack_value(pg, d, m, slot, vcode, &nv);
    for (int j = 0; j < d; ++j) {
      int c = vcode[j];
      chat[j] = ((c >> 3) ? -1.0 : 1.0) * vcpos[c & 7];
    }
    for (int k = 0; k < d; ++k) { /* v_hat = n_v * Pi^T c_hat */
      double a = 0.0;
      for (int j = 0; j < d; ++j) a += pi[(size_t)j * d + k] * chat[j];
      vals[(size_t)t * d + k] = nv * a;
    }
  }
  for (int t = 0; t < hot_len; ++t) {
    for (int h = 0; h < G; ++h) {
      double a = 0.0;
      for (int j = 0; j < d; ++j) a += q[(size_t)h * d + j] * k_hot[(size_t)t * d + j];
      logits[(size_t)h * nt + cold_len + t] = a * scale;
    }
    memcpy(vals + (size_t)(cold_len + t) * d, v_hot + (size_t)t * d, sizeof(double) * d);
  }
  for (int h = 0; h < G; ++h) {
    double* o = out + (size_t)h * d;
    for (int j = 0; j < d; ++j) o[j] = 0.0;
    int is_open = 1;
    if (gated) {
      double hmax = -INFINITY;
      for (int t = 0; t < hot_len; ++t) {
        double a = 0.0;
        for (int j = 0; j < d; ++j) a += q[(size_t)h * d + j] * k_hot[(size_t)t * d + j];
        hmax = fmax(hmax, a);
      }
      is_open = hmax < threshold;
    }
    if (open) open[h] = is_open; /* the gate's decision, also when there is no cold token */
    const int first = is_open ? 0 : cold_len; /* first token of the softmax */
    if (nt - first == 0) continue; /* no tokens: output defined as zero */
    double mx = -INFINITY;
    for (int t = first; t < nt; ++t) mx = fmax(mx, logits[(size_t)h * nt + t]);
    double den = 0.0;
    for (int t = first; t < nt; ++t) den += exp(logits[(size_t)h * nt + t] - mx);
    for (int t = first; t < nt; ++t) {
      double p = exp(logits[(size_t)h * nt + t] - mx) / den;
      for (int j = 0; j < d; ++j) o[j] += p * vals[(size_t)t * d + j];
    }
  }
  free(logits); free(vals); free(qrot); free(sq);
  free(sign); free(mag); free(qb); free(vcode); free(chat);
  return 0;
}

/*
 * Batched driver: groups listed in sel (pairs b, kv_head); the q heads of
 * kv head h are h*G .. h*G+G-1 (contiguous grouping).  Layouts:
 * q [B, Hq, d]; k_hot, v_hot [B, Hkv, W, d]; page_table [B, Hkv, max_pages];
 * out [nsel, G, d]; open (may be NULL) [nsel, G].  gated, threshold: the
 * threshold gate of or_attention_group.
 */
OR_API int or_attention_gated(int d, int m, const double* pi, const double* S,
                              const double* kcpos, const double* vcpos, int B, int Hq, int Hkv,
                              const double* q, double scale, const double* k_hot,
                              const double* v_hot, int W, const int32_t* hot_len,
                              const uint8_t* pool, size_t page_bytes, const int32_t* page_table,
                              int max_pages, const int32_t* cold_len, const int32_t* sel, int nsel,
                              int gated, double threshold, int32_t* open, double* out,
                              int threads) {
  int G = Hq / Hkv;
  int err = 0;
#ifdef _OPENMP
  const int nthreads = threads > 0 ? threads : omp_get_max_threads();
#pragma omp parallel for num_threads(nthreads) schedule(dynamic) reduction(| : err)
#endif
  for (int s = 0; s < nsel; ++s) {
    int b = sel[2 * s], h = sel[2 * s + 1];
    const double* kh = k_hot ? k_hot + ((size_t)b * Hkv + h) * (size_t)W * d : NULL;
    const double* vh = v_hot ? v_hot + ((size_t)b * Hkv + h) * (size_t)W * d : NULL;
    int hl = hot_len ? hot_len[b] : 0;
    int cl = cold_len ? cold_len[b] : 0;
    err |= or_attention_group(d, m, pi, S, kcpos, vcpos, G, q + ((size_t)b * Hq + (size_t)h * G) * d,
                              scale, kh, vh, hl, pool, page_bytes,
                              page_table + ((size_t)b * Hkv + h) * max_pages, cl, gated,
                              threshold, open ? open + (size_t)s * G : NULL,
                              out + (size_t)s * G * d);
  }
  return err;
}

/* The ungated form: every head reads hot and cold tokens. */
OR_API int or_attention(int d, int m, const double* pi, const double* S, const double* kcpos,
                        const double* vcpos, int B, int Hq, int Hkv, const double* q,
                        double scale, const double* k_hot, const double* v_hot, int W,
                        const int32_t* hot_len, const uint8_t* pool, size_t page_bytes,
                        const int32_t* page_table, int max_pages, const int32_t* cold_len,
                        const int32_t* sel, int nsel, double* out, int threads) {
  return or_attention_gated(d, m, pi, S, kcpos, vcpos, B, Hq, Hkv, q, scale, k_hot, v_hot, W,
                            hot_len, pool, page_bytes, page_table, max_pages, cold_len, sel, nsel,
                            0, 0.0, NULL, out, threads);
}

/* ------------------------------------------------------------------------ */
/* Compressed top-k search [TQ "Leistung bei der Vektorsuche"].             */
/* Score of DB vector i: n_i ( <q_rot, c_hat_i> + sqrt(pi/2)/m gamma_i      */
/* <S q_rot, 1-2 bits_i> ), scale 1.  Result: the k largest, ties to the    */
/* lower id.  DB vector i sits in keys-only page i/128, slot i%128.          */
/* ------------------------------------------------------------------------ */
static int better(double sa, int32_t ia, double sb, int32_t ib) {
  return (sa > sb) || (sa == sb && ia < ib);
}

OR_API void or_topk(int d, int m, const double* pi, const double* S, const double* kcpos,
                    const double* queries, int Q, const uint8_t* db, size_t page_bytes, int64_t N,
                    int k, int32_t* out_ids, double* out_scores, int threads) {
#ifdef _OPENMP
  const int nthreads = threads > 0 ? threads : omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
  {
    double* qrot = (double*)malloc(sizeof(double) * d);
    double* sq = (double*)malloc(sizeof(double) * m);
    int32_t* sign = (int32_t*)malloc(sizeof(int32_t) * d);
    int32_t* mag = (int32_t*)malloc(sizeof(int32_t) * d);
    int32_t* qb = (int32_t*)malloc(sizeof(int32_t) * m);
#ifdef _OPENMP
#pragma omp for schedule(dynamic)
#endif
    for (int qi = 0; qi < Q; ++qi) {
      const double* qv = queries + (size_t)qi * d;
      for (int j = 0; j < d; ++j) {
        double a = 0.0;
        for (int kk = 0; kk < d; ++kk) a += pi[(size_t)j * d + kk] * qv[kk];
        qrot[j] = a;
      }
      for (int i = 0; i < m; ++i) {
        double a = 0.0;
        for (int j = 0; j < d; ++j) a += S[(size_t)i * d + j] * qrot[j];
        sq[i] = a;
      }
      int32_t* ids = out_ids + (size_t)qi * k;
      double* sc = out_scores + (size_t)qi * k;
      int filled = 0;
      for (int64_t v = 0; v < N; ++v) {
        double n, gamma;
        or_unpack_key(db + (size_t)(v / PAGE_TOKENS) * page_bytes, d, m, 0,
                      (int)(v % PAGE_TOKENS), sign, mag, qb, &n, &gamma);
        double s = key_score(d, m, qrot, sq, kcpos, sign, mag, qb, n, gamma, 1.0);
        int32_t id = (int32_t)v;
        /* keep the list sorted best-first: insertion into k slots */
        if (filled < k) {
          int pos = filled++;
          while (pos > 0 && better(s, id, sc[pos - 1], ids[pos - 1])) {
            sc[pos] = sc[pos - 1]; ids[pos] = ids[pos - 1]; --pos;
          }
          sc[pos] = s; ids[pos] = id;
        } else if (better(s, id, sc[k - 1], ids[k - 1])) {
          int pos = k - 1;
          while (pos > 0 && better(s, id, sc[pos - 1], ids[pos - 1])) {
            sc[pos] = sc[pos - 1]; ids[pos] = ids[pos - 1]; --pos;
          }
          sc[pos] = s; ids[pos] = id;
        }
      }
      for (int i = filled; i < k; ++i) { ids[i] = -1; sc[i] = -INFINITY; }
    }
    free(qrot); free(sq); free(sign); free(mag); free(qb);
  }
}

OR_API int or_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Stage-1 variant: PolarQuant [TQ "PolarQuant: Ein neuer Winkel auf        */
/* Kompression": pairs of coordinates go to polar form, the radii are       */
/* paired again and the transform repeats until one radius and a set of     */
/* angles remain; the angles, whose distribution is known and concentrated, */
/* are quantised on a fixed grid].                                          */
/*                                                                           */
/* Applied to the rotated vector.  Level 1 pairs coordinates (2i, 2i+1):    */
/* angle theta in [0, 2 pi), uniform for a rotated vector, quantised on     */
/* 2^b1 equal bins with the bin centres as levels (the Lloyd-Max quantiser  */
/* of a uniform angle).  Level l >= 2 pairs the radii (r_e, r_o) of two      */
/* blocks of k = 2^(l-1) coordinates: phi = atan(r_o / r_e) in [0, pi/2]    */
/* has density proportional to sin^(k-1)(2 phi) (cos^2 phi is Beta(k/2,     */
/* k/2) for a uniform direction), quantised with its own 2^b2-level          */
/* Lloyd-Max codebook.  The last radius is stored as fp16.                   */
/*                                                                           */
/* Every decision is taken in fp32 exactly as stated here, so that a GPU    */
/* encoder given the same fp32 inputs takes the same ones: radii            */
/* sqrtf(fmaf(u, u, v * v)); level 1 reduces (a, b) to the first quadrant   */
/* by exact swaps and negations and counts the boundaries tan(2 pi j / M)   */
/* (fp32) with b' >= a' * t; level l counts the boundaries tan(t_j) (fp32)   */
/* with r_o >= r_e * T (only when r_o > 0).  A zero pair has angle 0.        */
/* ------------------------------------------------------------------------ */

/* int_a^b phi^order sin^(k-1)(2 phi) dphi, composite Gauss-Legendre */
static double angle_moment(int k, double a, double b, int order) {
  gl_init();
  if (b <= a) return 0.0;
  int panels = (int)ceil((b - a) / 0.01);
  double h = (b - a) / panels, s = 0.0;
  for (int p = 0; p < panels; ++p) {
    double lo = a + p * h, hh = 0.5 * h, c = lo + hh, ps = 0.0;
    for (int i = 0; i < GL_N; ++i) {
      double x = c + hh * gl_x[i];
      double f = pow(sin(2.0 * x), k - 1);
      ps += gl_w[i] * (order ? x * f : f);
    }
    s += ps * hh;
  }
  return s;
}

/* Lloyd-Max codebook of the level angle for blocks of k coordinates:
 * 2^bits levels c (increasing) and 2^bits - 1 boundaries t on [0, pi/2]. */
OR_API int or_angle_lloyd_max(int k, int bits, int max_iter, double* c, double* t) {
  int L = 1 << bits;
  for (int j = 0; j < L; ++j) c[j] = (j + 0.5) * (M_PI / 2.0) / L;
  int it = 0;
  for (; it < max_iter; ++it) {
    for (int j = 0; j + 1 < L; ++j) t[j] = 0.5 * (c[j] + c[j + 1]);
    double delta = 0.0;
    for (int j = 0; j < L; ++j) {
      double a = (j == 0) ? 0.0 : t[j - 1];
      double b = (j == L - 1) ? M_PI / 2.0 : t[j];
      double nc = angle_moment(k, a, b, 1) / angle_moment(k, a, b, 0);
      delta = fmax(delta, fabs(nc - c[j]));
      c[j] = nc;
    }
    if (delta < 1e-15) { ++it; break; }
  }
  for (int j = 0; j + 1 < L; ++j) t[j] = 0.5 * (c[j] + c[j + 1]);
  return it;
}

static int polar_levels(int d) { /* levels >= 2: log2(d) - 1 */
  int n = 0;
  for (int v = d / 2; v > 1; v >>= 1) ++n;
  return n;
}

static void put_bits(uint8_t* dst, size_t bitpos, int nbits, uint32_t v) {
  for (int i = 0; i < nbits; ++i)
    if ((v >> i) & 1u) dst[(bitpos + i) >> 3] |= (uint8_t)(1u << ((bitpos + i) & 7));
}

static uint32_t get_bits(const uint8_t* src, size_t bitpos, int nbits) {
  uint32_t v = 0;
  for (int i = 0; i < nbits; ++i)
    v |= (uint32_t)((src[(bitpos + i) >> 3] >> ((bitpos + i) & 7)) & 1u) << i;
  return v;
}

/* bytes of one vector's angle codes */
OR_API size_t or_polar_code_bytes(int d, int b1, int b2) {
  size_t bits = (size_t)b1 * (d / 2) + (size_t)b2 * (d / 2 - 1);
  return (bits + 7) / 8;
}

/* level-1 bin of the pair (a, b) among M = 2^b1 equal bins of [0, 2 pi) */
static int level1_bin(float a, float b, int M, const float* tq /* M/4 - 1 */) {
  int q;
  float u, v; /* the pair turned into the first quadrant [0, pi/2) */
  if (a > 0.0f && b >= 0.0f) { q = 0; u = a; v = b; }
  else if (a <= 0.0f && b > 0.0f) { q = 1; u = b; v = -a; }
  else if (a < 0.0f && b <= 0.0f) { q = 2; u = -a; v = -b; }
  else if (a >= 0.0f && b < 0.0f) { q = 3; u = -b; v = a; }
  else { return 0; } /* zero pair */
  int j = 0;
  for (int i = 0; i < M / 4 - 1; ++i)
    if (v >= u * tq[i]) j = i + 1;
  return q * (M / 4) + j;
}

/* x: N rotated vectors (fp32); codes: N * or_polar_code_bytes bytes
 * (zeroed here); radius: fp16 bits of the final radius.  b1 >= 2. */
OR_API void or_polar_encode(int d, const float* x, int64_t N, int b1, int b2, uint8_t* codes,
                            uint16_t* radius) {
  int M = 1 << b1, L = 1 << b2, nl = polar_levels(d);
  size_t cb = or_polar_code_bytes(d, b1, b2);
  float tq[64];
  for (int i = 0; i < M / 4 - 1; ++i) tq[i] = (float)tan(2.0 * M_PI * (i + 1) / M);
  float T[16][16];
  double c[64], t[64];
  for (int l = 0; l < nl; ++l) {
    or_angle_lloyd_max(1 << (l + 1), b2, 100000, c, t);
    for (int j = 0; j < L - 1; ++j) T[l][j] = (float)tan(t[j]);
  }
  float* r = (float*)malloc(sizeof(float) * (d / 2));
  for (int64_t n = 0; n < N; ++n) {
    const float* v = x + (size_t)n * d;
    uint8_t* out = codes + (size_t)n * cb;
    memset(out, 0, cb);
    size_t pos = 0;
    for (int i = 0; i < d / 2; ++i) {
      float a = v[2 * i], b = v[2 * i + 1];
      put_bits(out, pos, b1, (uint32_t)level1_bin(a, b, M, tq));
      pos += b1;
      r[i] = sqrtf(fmaf(a, a, b * b));
    }
    int nodes = d / 2;
    for (int l = 0; l < nl; ++l) {
      nodes /= 2;
      for (int i = 0; i < nodes; ++i) {
        float re = r[2 * i], ro = r[2 * i + 1];
        int j = 0;
        if (ro > 0.0f)
          for (int s = 0; s < L - 1; ++s)
            if (ro >= re * T[l][s]) j = s + 1;
        put_bits(out, pos, b2, (uint32_t)j);
        pos += b2;
        r[i] = sqrtf(fmaf(re, re, ro * ro));
      }
    }
    radius[n] = f16_bits(or_round_f16((double)r[0]));
  }
  free(r);
}

/* reconstruction (fp64) from the codes and the fp16 radius */
OR_API void or_polar_decode(int d, const uint8_t* codes, const uint16_t* radius, int64_t N, int b1,
                            int b2, double* xhat) {
  int M = 1 << b1, L = 1 << b2, nl = polar_levels(d);
  size_t cb = or_polar_code_bytes(d, b1, b2);
  double cl[16][16], t[64];
  for (int l = 0; l < nl; ++l) or_angle_lloyd_max(1 << (l + 1), b2, 100000, cl[l], t);
  double* r = (double*)malloc(sizeof(double) * (d / 2));
  double* rn = (double*)malloc(sizeof(double) * (d / 2));
  for (int64_t n = 0; n < N; ++n) {
    const uint8_t* in = codes + (size_t)n * cb;
    r[0] = f16_value(radius[n]);
    /* level-l codes start after the level-1 codes and the lower levels' */
    size_t base = (size_t)b1 * (d / 2);
    size_t off[16];
    int cnt = d / 2;
    for (int l = 0; l < nl; ++l) {
      cnt /= 2;
      off[l] = base;
      base += (size_t)b2 * cnt;
    }
    int nodes = 1;
    for (int l = nl - 1; l >= 0; --l) {
      for (int i = 0; i < nodes; ++i) {
        double phi = cl[l][get_bits(in, off[l] + (size_t)b2 * i, b2)];
        rn[2 * i] = r[i] * cos(phi);
        rn[2 * i + 1] = r[i] * sin(phi);
      }
      nodes *= 2;
      memcpy(r, rn, sizeof(double) * nodes);
    }
    double* o = xhat + (size_t)n * d;
    for (int i = 0; i < d / 2; ++i) {
      double th = 2.0 * M_PI * (get_bits(in, (size_t)b1 * i, b1) + 0.5) / M;
      o[2 * i] = r[i] * cos(th);
      o[2 * i + 1] = r[i] * sin(th);
    }
  }
  free(r);
  free(rn);
}

/* the exact transform (no quantisation), fp64: final radius and the angles
 * (level 1 first, then levels 2, 3, ...), and its inverse */
OR_API void or_polar_transform(int d, const double* x, double* radius, double* angles) {
  double* r = (double*)malloc(sizeof(double) * (d / 2));
  int k = 0;
  for (int i = 0; i < d / 2; ++i) {
    double th = atan2(x[2 * i + 1], x[2 * i]);
    angles[k++] = th < 0.0 ? th + 2.0 * M_PI : th;
    r[i] = hypot(x[2 * i], x[2 * i + 1]);
  }
  for (int nodes = d / 4; nodes >= 1; nodes /= 2)
    for (int i = 0; i < nodes; ++i) {
      angles[k++] = atan2(r[2 * i + 1], r[2 * i]);
      r[i] = hypot(r[2 * i], r[2 * i + 1]);
    }
  *radius = r[0];
  free(r);
}

OR_API void or_polar_inverse(int d, double radius, const double* angles, double* x) {
  double* r = (double*)malloc(sizeof(double) * d);
  double* rn = (double*)malloc(sizeof(double) * d);
  int nl = polar_levels(d);
  size_t off[16];
  size_t base = (size_t)(d / 2);
  int cnt = d / 2;
  for (int l = 0; l < nl; ++l) {
    cnt /= 2;
    off[l] = base;
    base += cnt;
  }
  r[0] = radius;
  int nodes = 1;
  for (int l = nl - 1; l >= 0; --l) {
    for (int i = 0; i < nodes; ++i) {
      rn[2 * i] = r[i] * cos(angles[off[l] + i]);
      rn[2 * i + 1] = r[i] * sin(angles[off[l] + i]);
    }
    nodes *= 2;
    memcpy(r, rn, sizeof(double) * nodes);
  }
  for (int i = 0; i < d / 2; ++i) {
    x[2 * i] = r[i] * cos(angles[i]);
    x[2 * i + 1] = r[i] * sin(angles[i]);
  }
  free(r);
  free(rn);
}
