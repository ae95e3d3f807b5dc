// Host-side math of the OrbitQuant layer: the seeded permutation, the
// Lloyd-Max codebook design and the fp16 decode scale.  Offline work, run once
// per layer; nothing here is on the per-token path.
#include "oq_internal.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

namespace oq {

// ---------------------------------------------------------------------------
// SplitMix64 (Steele, Lea, Flood 2014) and the Fisher-Yates shuffle that
// draws the RPBH permutation pi (gecl notes Method 4: a uniform random
// permutation scatters outlier channels across blocks; the pages fix no
// generator, so a seeded one shared by weights and activations is used).
// ---------------------------------------------------------------------------
struct SplitMix64 {
  uint64_t state;
  explicit SplitMix64(uint64_t seed) : state(seed) {}
  uint64_t next() {
    state += 0x9E3779B97F4A7C15ull;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
};

void make_permutation(int d, uint64_t seed, std::vector<uint32_t>& perm,
                      std::vector<int8_t>* signs) {
  perm.resize(d);
  for (int i = 0; i < d; ++i) perm[i] = (uint32_t)i;
  SplitMix64 g(seed);
  for (int i = d - 1; i >= 1; --i) {
    // j uniform in [0, i]: high 64 bits of the 128-bit product next() * (i+1)
    unsigned __int128 prod = (unsigned __int128)g.next() * (unsigned __int128)(uint64_t)(i + 1);
    uint32_t j = (uint32_t)(prod >> 64);
    std::swap(perm[i], perm[j]);
  }
  if (signs) {
    // Rademacher D_j of pith Supplementary A, by rotated position, drawn after
    // the shuffle: -1 when bit 63 is set.
    signs->resize(d);
    for (int i = 0; i < d; ++i) (*signs)[i] = (g.next() >> 63) ? -1 : 1;
  }
}

// ---------------------------------------------------------------------------
// Lloyd-Max design.  Symmetric log-concave density, so the optimal quantizer
// is symmetric with a threshold at 0; solve on the positive half-line for the
// positive thresholds tau_1 < ... < tau_{n-1} (n = L/2 cells, tau_0 = 0,
// tau_n = top) by Newton's method on
//   F_k = tau_k - (c_{k-1} + c_k) / 2 = 0,   c_k = centroid of [tau_k, tau_{k+1}]
// (Max's conditions: each threshold the midpoint of its levels, each level the
// conditional mean of its cell).  The Jacobian is tridiagonal.
// ---------------------------------------------------------------------------
namespace {

struct GaussLegendre {
  std::vector<double> x, w;  // nodes and weights on [-1, 1]
  explicit GaussLegendre(int n) : x(n), w(n) {
    for (int i = 0; i < n; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = z;  // Legendre recurrence
        for (int k = 2; k <= n; ++k) {
          double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
          p0 = p1;
          p1 = p2;
        }
        double dp = n * (z * p1 - p0) / (z * z - 1.0);
        double dz = p1 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) {
          // final derivative at the converged node
          double q0 = 1.0, q1 = z;
          for (int k = 2; k <= n; ++k) {
            double q2 = ((2.0 * k - 1.0) * z * q1 - (k - 1.0) * q0) / k;
            q0 = q1;
            q1 = q2;
          }
          dp = n * (z * q1 - q0) / (z * z - 1.0);
          x[i] = z;
          w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
          break;
        }
      }
    }
  }
};

const GaussLegendre& gl24() {
  static GaussLegendre g(24);
  return g;
}

struct Marginal {
  int d;
  bool gaussian;
  double log_c;   // log normaliser of the sphere density
  double m;       // exponent (d-3)/2
  double sigma;   // 1/sqrt(d)
  double top;     // upper end of the support (1, or +inf)
  double width;   // panel scale for quadrature

  Marginal(int d_, bool g) : d(d_), gaussian(g) {
    m = (d - 3) / 2.0;
    log_c = std::lgamma(d / 2.0) - std::lgamma((d - 1) / 2.0) - 0.5 * std::log(M_PI);
    sigma = 1.0 / std::sqrt((double)d);
    top = g ? INFINITY : 1.0;
    width = 1.0 / std::sqrt(std::max(d - 3, 1) * 1.0);
  }
  double pdf(double t) const {
    if (gaussian) return std::exp(-0.5 * d * t * t) * std::sqrt(d / (2.0 * M_PI));
    if (std::fabs(t) >= 1.0) return 0.0;
    return std::exp(log_c + m * std::log1p(-t * t));
  }
  // mass and first moment of [a, b], 0 <= a < b <= top
  void cell(double a, double b, double& P, double& M) const {
    if (gaussian) {
      const double r = std::sqrt(d / 2.0);
      P = 0.5 * (std::erfc(a * r) - (std::isinf(b) ? 0.0 : std::erfc(b * r)));
      const double ga = std::exp(-0.5 * d * a * a);
      const double gb = std::isinf(b) ? 0.0 : std::exp(-0.5 * d * b * b);
      M = (ga - gb) / std::sqrt(2.0 * M_PI * d);
      return;
    }
    // composite 24-point Gauss-Legendre; beyond 45 widths past `a` the
    // density has fallen by more than exp(-1000) and is dropped
    const double hi = std::min(b, a + 45.0 * width);
    const int panels = std::max(1, (int)std::ceil((hi - a) / (0.2 * width)));
    const GaussLegendre& g = gl24();
    P = 0.0;
    M = 0.0;
    for (int p = 0; p < panels; ++p) {
      const double lo_p = a + (hi - a) * p / panels;
      const double hi_p = a + (hi - a) * (p + 1) / panels;
      const double c = 0.5 * (lo_p + hi_p), h = 0.5 * (hi_p - lo_p);
      for (size_t i = 0; i < g.x.size(); ++i) {
        const double t = c + h * g.x[i];
        const double f = h * g.w[i] * pdf(t);
        P += f;
        M += f * t;
      }
    }
  }
  double survival(double x) const {  // P(T > x), x >= 0, for the initial guess
    if (gaussian) return 0.5 * std::erfc(x * std::sqrt(d / 2.0));
    double P, M;
    cell(x, 1.0, P, M);
    return P;
  }
};

// levels and their derivatives for given positive thresholds
void centroids(const Marginal& f, const std::vector<double>& tau, std::vector<double>& c,
               std::vector<double>& P, std::vector<double>* dlo, std::vector<double>* dhi) {
  const int n = (int)tau.size() - 1;  // tau[0] = 0, tau[n] = top
  c.resize(n);
  P.resize(n);
  if (dlo) dlo->resize(n), dhi->resize(n);
  for (int k = 0; k < n; ++k) {
    double Pk, Mk;
    f.cell(tau[k], tau[k + 1], Pk, Mk);
    P[k] = Pk;
    c[k] = Mk / Pk;
    if (dlo) {
      (*dlo)[k] = f.pdf(tau[k]) * (c[k] - tau[k]) / Pk;
      (*dhi)[k] = std::isinf(tau[k + 1]) ? 0.0 : f.pdf(tau[k + 1]) * (tau[k + 1] - c[k]) / Pk;
    }
  }
}

}  // namespace

oq_status design_codebook(int d, int bits, int flags, oq_codebook* out) {
  const bool gaussian = (flags & OQ_FLAG_GAUSSIAN_MARGINAL) != 0;
  const Marginal f(d, gaussian);
  const int L = 1 << bits, n = L / 2;
  std::vector<double> tau(n + 1), c, P, dlo, dhi;
  tau[0] = 0.0;
  tau[n] = f.top;
  // initial thresholds: midpoints of levels placed at the quantiles of the
  // f^(1/3) point density, approximated by N(0, 3/d), found by bisection
  std::vector<double> c0(n);
  for (int k = 0; k < n; ++k) {
    const double target = (n - k - 0.5) / L;  // P(X > c0_k) for X ~ N(0, 3/d)
    double lo = 0.0, hi = 40.0 * f.sigma;
    for (int it = 0; it < 200; ++it) {
      const double mid = 0.5 * (lo + hi);
      (0.5 * std::erfc(mid / (std::sqrt(6.0) * f.sigma)) > target ? lo : hi) = mid;
    }
    c0[k] = std::min(0.5 * (lo + hi), 0.999 * (1.0 - 1e-3 * (n - k)));
  }
  for (int k = 1; k < n; ++k) tau[k] = 0.5 * (c0[k - 1] + c0[k]);

  int iters = 0;
  if (n >= 2) {
    // a few plain Lloyd sweeps bring the start into Newton's basin
    for (int it = 0; it < 30; ++it, ++iters) {
      centroids(f, tau, c, P, nullptr, nullptr);
      for (int k = 1; k < n; ++k) tau[k] = 0.5 * (c[k - 1] + c[k]);
    }
    std::vector<double> F(n), a(n), b(n), cc(n), dx(n), newtau(n + 1);
    auto residual = [&](const std::vector<double>& t, std::vector<double>& Fo) {
      std::vector<double> cl, Pl;
      centroids(f, t, cl, Pl, nullptr, nullptr);
      double mx = 0.0;
      for (int k = 1; k < n; ++k) {
        Fo[k] = t[k] - 0.5 * (cl[k - 1] + cl[k]);
        mx = std::max(mx, std::fabs(Fo[k]));
      }
      return mx;
    };
    for (int it = 0; it < 200; ++it, ++iters) {
      centroids(f, tau, c, P, &dlo, &dhi);
      double fmax = 0.0;
      for (int k = 1; k < n; ++k) {
        F[k] = tau[k] - 0.5 * (c[k - 1] + c[k]);
        fmax = std::max(fmax, std::fabs(F[k]));
        // tridiagonal Jacobian row k (unknowns tau_1..tau_{n-1})
        a[k] = (k > 1) ? -0.5 * dlo[k - 1] : 0.0;          // d/d tau_{k-1}
        b[k] = 1.0 - 0.5 * (dhi[k - 1] + dlo[k]);           // d/d tau_k
        cc[k] = (k < n - 1) ? -0.5 * dhi[k] : 0.0;          // d/d tau_{k+1}
      }
      if (fmax < 1e-17 * f.sigma) break;
      // Thomas algorithm
      std::vector<double> cp(n), dp(n);
      for (int k = 1; k < n; ++k) {
        const double den = b[k] - (k > 1 ? a[k] * cp[k - 1] : 0.0);
        cp[k] = cc[k] / den;
        dp[k] = (F[k] - (k > 1 ? a[k] * dp[k - 1] : 0.0)) / den;
      }
      for (int k = n - 1; k >= 1; --k) dx[k] = dp[k] - (k < n - 1 ? cp[k] * dx[k + 1] : 0.0);
      // damped step that keeps the thresholds ordered and lowers |F|
      double step = 1.0;
      std::vector<double> Fn(n);
      for (int tries = 0; tries < 40; ++tries, step *= 0.5) {
        newtau = tau;
        bool ok = true;
        for (int k = 1; k < n; ++k) newtau[k] = tau[k] - step * dx[k];
        for (int k = 1; k <= n; ++k) ok = ok && newtau[k] > newtau[k - 1];
        if (ok && residual(newtau, Fn) <= fmax) break;
        if (tries == 39) newtau = tau;
      }
      double move = 0.0;
      for (int k = 1; k < n; ++k) move = std::max(move, std::fabs(newtau[k] - tau[k]));
      tau = newtau;
      if (move < 1e-16 * f.sigma) break;
    }
  }
  centroids(f, tau, c, P, nullptr, nullptr);

  std::memset(out, 0, sizeof(*out));
  out->d = d;
  out->bits = bits;
  out->flags = flags & OQ_FLAG_GAUSSIAN_MARGINAL;
  out->iterations = iters;
  for (int k = 0; k < n; ++k) {
    out->levels[n + k] = c[k];
    out->levels[n - 1 - k] = -c[k];
  }
  for (int j = 0; j < L - 1; ++j) out->thresholds[j] = 0.5 * (out->levels[j] + out->levels[j + 1]);
  out->thresholds[n - 1] = 0.0;
  double sum = 0.0;
  for (int k = 0; k < n; ++k) sum += P[k] * c[k] * c[k];
  out->mse = 1.0 / d - 2.0 * sum;
  return OQ_OK;
}

oq_status get_codebook(int d, int bits, int flags, oq_codebook* out) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int>, oq_codebook> cache;
  const auto key = std::make_tuple(d, bits, flags & OQ_FLAG_GAUSSIAN_MARGINAL);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *out = it->second;
      return OQ_OK;
    }
  }
  oq_status st = design_codebook(d, bits, flags, out);
  if (st == OQ_OK) {
    std::lock_guard<std::mutex> lock(mu);
    cache[key] = *out;
  }
  return st;
}

// ---------------------------------------------------------------------------
// fp16 decode tables.  Both operands of the contraction are decoded to fp16
// levels; a per-codebook scale alpha is chosen so that alpha * level lands as
// close as possible to fp16-representable values (the epilogue divides by
// alpha_a * alpha_w).  fp16 rounding is written out here: round to nearest,
// ties to even, normal range only (levels are scaled into [2^-10, 2^4)).
// ---------------------------------------------------------------------------
uint16_t f64_to_f16_bits(double v) {
  const uint16_t sign = v < 0 ? 0x8000 : 0;
  double a = std::fabs(v);
  if (a == 0.0) return sign;
  int e;
  double m = std::frexp(a, &e);          // a = m * 2^e, m in [0.5, 1)
  // fp16 normal: value = (1 + f/1024) * 2^(E-15), E in [1, 30]
  int E = e - 1 + 15;
  double scaled = m * 2048.0;            // in [1024, 2048): 11 significant bits
  double r = std::nearbyint(scaled);     // ties to even under the default mode
  if (r >= 2048.0) {
    r = 1024.0;
    ++E;
  }
  if (E <= 0 || E >= 31) return sign;    // out of range: not produced for our levels
  return (uint16_t)(sign | (E << 10) | ((int)r - 1024));
}

double f16_bits_to_f64(uint16_t h) {
  const int E = (h >> 10) & 31, f = h & 1023;
  double v = (E == 0) ? f / 1024.0 * std::ldexp(1.0, -14) : (1.0 + f / 1024.0) * std::ldexp(1.0, E - 15);
  return (h & 0x8000) ? -v : v;
}

// e4m3 (4 exponent bits, bias 7, 3 mantissa bits, largest finite 448) for
// the lower-precision contraction mode: round to nearest, ties to even,
// normal range only (levels are scaled into [2^-6, 448)).
uint8_t f64_to_e4m3_bits(double v) {
  const uint8_t sign = v < 0 ? 0x80 : 0;
  const double a = std::fabs(v);
  if (a == 0.0) return sign;
  int e;
  const double m = std::frexp(a, &e);    // a = m * 2^e, m in [0.5, 1)
  int E = e - 1 + 7;
  double r = std::nearbyint(m * 16.0);   // 4 significant bits, in [8, 16]
  if (r >= 16.0) {
    r = 8.0;
    ++E;
  }
  if (E <= 0 || E > 15 || (E == 15 && r == 15.0)) return sign;   // not produced for our levels
  return (uint8_t)(sign | (E << 3) | ((int)r - 8));
}

double e4m3_bits_to_f64(uint8_t b) {
  const int E = (b >> 3) & 15, f = b & 7;
  const double v = (E == 0) ? f / 8.0 * std::ldexp(1.0, -6) : (1.0 + f / 8.0) * std::ldexp(1.0, E - 7);
  return (b & 0x80) ? -v : v;
}

// the scale that brings the positive levels closest to e4m3 values (largest
// relative error over the levels), searched in [8, 16) / max level so that the
// largest level lands in [8, 16)
double choose_fp8_scale(const oq_codebook& cb, double* worst) {
  const int L = 1 << cb.bits;
  const double base = 8.0 / cb.levels[L - 1];
  double best = base, best_err = 1e30;
  for (int j = 0; j < 4096; ++j) {
    const double alpha = base * (1.0 + j / 4096.0);
    double err = 0.0;
    for (int i = L / 2; i < L; ++i) {
      const double v = alpha * cb.levels[i];
      err = std::max(err, std::fabs(e4m3_bits_to_f64(f64_to_e4m3_bits(v)) - v) / v);
    }
    if (err < best_err) {
      best_err = err;
      best = alpha;
    }
  }
  if (worst) *worst = best_err;
  return best;
}

double choose_fp16_scale(const oq_codebook& cb) {
  const int L = 1 << cb.bits;
  const double base = std::sqrt((double)cb.d);
  double best = base, best_err = 1e30;
  for (int j = 0; j < 4096; ++j) {
    const double alpha = base * (1.0 + j / 4096.0);
    double err = 0.0;
    for (int i = L / 2; i < L; ++i) {
      const double v = alpha * cb.levels[i];
      err = std::max(err, std::fabs(f16_bits_to_f64(f64_to_f16_bits(v)) - v) / v);
    }
    if (err < best_err) {
      best_err = err;
      best = alpha;
    }
  }
  return best;
}


// Threshold search table (see oq_bin_table): the smallest power of two K for
// which consecutive scaled thresholds (as fp32, the values the kernel compares
// against) lie more than one bin apart, then per bin the number of thresholds
// in earlier bins and the one threshold inside it (+inf if none).  With
// full_range the bins cover every g a finite token can produce: |u| <= 1, so
// |g| <= K sqrt(d), plus a margin for fp32 rounding of z and s; a kernel can
// then index it without clamping.
oq_status build_bin_table(const oq_codebook& cb, int d, int h, const uint16_t* lv16, float* kscale, int* b0, int* nb,
                          std::vector<uint32_t>& codes, std::vector<uint32_t>& levels, bool full_range) {
  const int L = 1 << cb.bits;
  const double sd = std::sqrt((double)d);
  auto bits_of = [](float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return u;
  };
  for (int lk = 0; lk <= 16; ++lk) {
    const double K = std::ldexp(1.0, lk);
    std::vector<float> tk(L - 1);
    for (int j = 0; j < L - 1; ++j) tk[j] = (float)(K * sd * cb.thresholds[j]);
    bool apart = true;
    for (int j = 1; j < L - 1 && apart; ++j) apart = (double)tk[j] - (double)tk[j - 1] > 1.0;
    if (!apart) continue;
    int lo = (int)std::nearbyint(tk[0]) - 1, hi = (int)std::nearbyint(tk[L - 2]) + 1;
    if (full_range) {
      const int bound = (int)std::ceil(K * sd * (1.0 + 1e-4)) + 2;
      lo = std::min(lo, -bound);
      hi = std::max(hi, bound);
    }
    const int n = hi - lo + 1;
    if (n > OQ_MAX_BINS) break;
    codes.assign(2 * (size_t)n, 0u);
    levels.assign(2 * (size_t)n, 0u);
    int j = 0;
    for (int b = 0; b < n; ++b) {
      const int m = lo + b;
      while (j < L - 1 && (int)std::nearbyint(tk[j]) < m) ++j;
      const bool has = j < L - 1 && (int)std::nearbyint(tk[j]) == m;
      const uint32_t t = bits_of(has ? tk[j] : INFINITY);
      codes[2 * b] = t;
      codes[2 * b + 1] = (uint32_t)j;
      levels[2 * b] = t;
      levels[2 * b + 1] = (uint32_t)lv16[j] | ((uint32_t)lv16[has ? j + 1 : j] << 16);
    }
    *kscale = (float)(K * sd / std::sqrt((double)h));
    *b0 = -lo;
    *nb = n;
    return OQ_OK;
  }
  set_error("threshold table: codebook thresholds too close for a bin table");
  return OQ_ERR_UNSUPPORTED;
}

}  // namespace oq
