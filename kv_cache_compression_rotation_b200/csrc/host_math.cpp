// Host-side math of libtq: Lloyd-Max codebooks, integer water-filling, spectral
// calibration.  Plain double-precision C++; no CUDA.
//
// Codebook (TurboQuant review, "Method"): the coordinate law after a random rotation is
// the marginal of a uniform point on S^{d-1},
//     f(t) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) * (1 - t^2)^((d-3)/2),
// converging to N(0, 1/d); the codebook is the fixed point of the continuous 1-D
// k-means (Lloyd-Max) iteration.  Cell masses use composite Gauss-Legendre quadrature
// of f for d >= 16 and the regularized incomplete beta function (t^2 ~ Beta(1/2,
// (d-1)/2), continued fraction by the modified Lentz method) for smaller d; first
// moments have the closed form
//     int_a^b t f(t) dt = C_d / (d-1) * ((1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "tq_internal.h"

namespace tq {
namespace {

// Continued fraction of the regularized incomplete beta (Lentz's method): returns
// I_x(a, b) for x < (a + 1) / (a + b + 2), where the fraction converges quickly.
double ibeta_cf(double a, double b, double x) {
  const double tiny = 1e-300;
  double c = 1.0;
  double dd = 1.0 - (a + b) * x / (a + 1.0);
  if (std::fabs(dd) < tiny) dd = tiny;
  dd = 1.0 / dd;
  double h = dd;
  for (int m = 1; m <= 100000; ++m) {
    const double m2 = 2.0 * m;
    double num = m * (b - m) * x / ((a + m2 - 1.0) * (a + m2));
    dd = 1.0 + num * dd;
    if (std::fabs(dd) < tiny) dd = tiny;
    c = 1.0 + num / c;
    if (std::fabs(c) < tiny) c = tiny;
    dd = 1.0 / dd;
    h *= dd * c;
    num = -(a + m) * (a + b + m) * x / ((a + m2) * (a + m2 + 1.0));
    dd = 1.0 + num * dd;
    if (std::fabs(dd) < tiny) dd = tiny;
    c = 1.0 + num / c;
    if (std::fabs(c) < tiny) c = tiny;
    dd = 1.0 / dd;
    const double del = dd * c;
    h *= del;
    if (std::fabs(del - 1.0) < 1e-16) break;
  }
  const double lfront = a * std::log(x) + b * std::log1p(-x) - (std::lgamma(a) + std::lgamma(b) - std::lgamma(a + b));
  return std::exp(lfront) * h / a;
}

// I_x(a,b) and 1 - I_x(a,b), each computed without cancellation.
void ibeta_pair(double a, double b, double x, double* lo, double* hi) {
  if (x <= 0.0) { *lo = 0.0; *hi = 1.0; return; }
  if (x >= 1.0) { *lo = 1.0; *hi = 0.0; return; }
  if (x < (a + 1.0) / (a + b + 2.0)) {
    *lo = ibeta_cf(a, b, x);
    *hi = 1.0 - *lo;
  } else {
    *hi = ibeta_cf(b, a, 1.0 - x);
    *lo = 1.0 - *hi;
  }
}

struct Law {
  int dist;      // 0 beta-sphere, 1 gaussian
  int d;
  double sigma;
  double lo, hi;  // support
  double scale;   // coordinate standard deviation
};

// P(T <= t) and P(T > t).
void cdf_parts(const Law& L, double t, double* below, double* above) {
  if (L.dist == TQ_DIST_GAUSSIAN) {
    const double z = t / L.sigma;
    *below = 0.5 * std::erfc(-z / std::sqrt(2.0));
    *above = 0.5 * std::erfc(z / std::sqrt(2.0));
    return;
  }
  if (t <= -1.0) { *below = 0.0; *above = 1.0; return; }
  if (t >= 1.0) { *below = 1.0; *above = 0.0; return; }
  const double beta = 0.5 * (L.d - 1);
  double in, out;  // P(|T| <= |t|), P(|T| > |t|)
  ibeta_pair(0.5, beta, t * t, &in, &out);
  if (t >= 0) { *below = 0.5 + 0.5 * in; *above = 0.5 * out; }
  else        { *below = 0.5 * out;      *above = 0.5 + 0.5 * in; }
}

// Gauss-Legendre nodes and weights on [-1, 1] (Newton iteration on P_n).
struct GaussLegendre {
  static constexpr int n = 12;
  double x[n], w[n];
  GaussLegendre() {
    for (int i = 0; i < n; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (n + 0.5)), dp = 0.0;
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = 0.0;
        for (int k = 1; k <= n; ++k) {
          const double p2 = p1;
          p1 = p0;
          p0 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p2) / k;
        }
        dp = n * (z * p0 - p1) / (z * z - 1.0);
        const double dz = p0 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) break;
      }
      x[i] = z;
      w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

// Mass of the sphere marginal on (a, b] by composite Gauss-Legendre quadrature of
// C_d (1 - t^2)^((d-3)/2).  Used for d >= 16, where the density is smooth on [-1, 1];
// unlike differences of incomplete-beta values it has no switch between two
// evaluation branches, so the Lloyd map stays smooth to rounding level and the
// iteration converges for large d.
double beta_mass_quad(const Law& L, double a, double b) {
  static const GaussLegendre gl;
  const double nu = 0.5 * (L.d - 3);
  const double lc = std::lgamma(0.5 * L.d) - 0.5 * std::log(M_PI) - std::lgamma(0.5 * (L.d - 1));
  double lo = std::max(a, std::max(-1.0, -60.0 * L.scale));
  double hi = std::min(b, std::min(1.0, 60.0 * L.scale));
  if (!(hi > lo)) return 0.0;
  const int nsub = std::max(1, static_cast<int>(std::ceil((hi - lo) / (0.5 * L.scale))));
  const double h = (hi - lo) / nsub;
  double total = 0.0;
  for (int s = 0; s < nsub; ++s) {
    const double c0 = lo + (s + 0.5) * h;
    double part = 0.0;
    for (int i = 0; i < GaussLegendre::n; ++i) {
      const double t = c0 + 0.5 * h * gl.x[i];
      if (std::fabs(t) < 1.0) part += gl.w[i] * std::exp(lc + nu * std::log1p(-t * t));
    }
    total += 0.5 * h * part;
  }
  return total;
}

double cell_mass(const Law& L, double a, double b) {
  if (L.dist == TQ_DIST_BETA_SPHERE && L.d >= 16) return beta_mass_quad(L, a, b);
  double ba, aa, bb, ab;
  cdf_parts(L, a, &ba, &aa);
  cdf_parts(L, b, &bb, &ab);
  return a >= 0 ? aa - ab : bb - ba;
}

// int_a^b t f(t) dt
double cell_first(const Law& L, double a, double b) {
  if (L.dist == TQ_DIST_GAUSSIAN) {
    auto phi = [&](double t) {
      if (!std::isfinite(t)) return 0.0;
      const double z = t / L.sigma;
      return std::exp(-0.5 * z * z) / std::sqrt(2.0 * M_PI);
    };
    return L.sigma * (phi(a) - phi(b));
  }
  const double beta = 0.5 * (L.d - 1);
  const double lc = std::lgamma(0.5 * L.d) - 0.5 * std::log(M_PI) - std::lgamma(0.5 * (L.d - 1));
  auto g = [&](double t) {
    t = std::min(1.0, std::max(-1.0, t));
    return std::fabs(t) >= 1.0 ? 0.0 : std::exp(beta * std::log1p(-t * t));
  };
  return std::exp(lc) / (L.d - 1) * (g(a) - g(b));
}

double quantile(const Law& L, double p) {
  double lo = L.dist == TQ_DIST_GAUSSIAN ? -40.0 * L.sigma : -1.0;
  double hi = -lo;
  for (int it = 0; it < 200; ++it) {
    const double mid = 0.5 * (lo + hi);
    double below, above;
    cdf_parts(L, mid, &below, &above);
    if (below < p) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

}  // namespace

tq_status codebook_build(int d, int bits, int dist, double sigma, double* c_out, double* t_out,
                         int* iters_out) {
  if (bits < 1 || bits > 8) return fail(TQ_ERR_INVALID_ARG, "codebook: bits must be 1..8");
  if (!c_out || !t_out) return fail(TQ_ERR_INVALID_ARG, "codebook: null output");
  Law L{};
  L.dist = dist;
  if (dist == TQ_DIST_BETA_SPHERE) {
    if (d < 2 || d > (1 << 20)) return fail(TQ_ERR_INVALID_ARG, "codebook: beta law needs d >= 2");
    L.d = d; L.lo = -1.0; L.hi = 1.0; L.scale = 1.0 / std::sqrt((double)d);
  } else if (dist == TQ_DIST_GAUSSIAN) {
    if (!(sigma > 0.0) || !std::isfinite(sigma)) return fail(TQ_ERR_INVALID_ARG, "codebook: sigma must be > 0");
    L.sigma = sigma; L.lo = -INFINITY; L.hi = INFINITY; L.scale = sigma;
  } else {
    return fail(TQ_ERR_INVALID_ARG, "codebook: unknown dist");
  }
  const int K = 1 << bits;
  std::vector<double> c(K), cn(K), edge(K + 1);
  for (int k = 0; k < K; ++k) c[k] = quantile(L, (k + 0.5) / K);
  const long max_iter = 10000000;
  for (long it = 1; it <= max_iter; ++it) {
    edge[0] = L.lo;
    edge[K] = L.hi;
    for (int k = 1; k < K; ++k) edge[k] = 0.5 * (c[k - 1] + c[k]);
    double move = 0.0;
    for (int k = 0; k < K; ++k) {
      const double m = cell_mass(L, edge[k], edge[k + 1]);
      const double f = cell_first(L, edge[k], edge[k + 1]);
      cn[k] = m > 0 ? f / m : 0.5 * (edge[k] + edge[k + 1]);
      move = std::max(move, std::fabs(cn[k] - c[k]));
    }
    c.swap(cn);
    // both laws are symmetric: keep the codebook exactly odd so the middle boundary is 0
    for (int k = 0; k < K / 2; ++k) {
      const double v = 0.5 * (c[K - 1 - k] - c[k]);
      c[k] = -v;
      c[K - 1 - k] = v;
    }
    if (move < 1e-13 * L.scale) {
      for (int k = 0; k < K; ++k) c_out[k] = c[k];
      for (int k = 0; k + 1 < K; ++k) t_out[k] = 0.5 * (c[k] + c[k + 1]);
      if (iters_out) *iters_out = (int)it;
      return TQ_OK;
    }
  }
  return fail(TQ_ERR_NOT_CONVERGED, "codebook: Lloyd-Max did not converge");
}

tq_status waterfill(const double* lambda, int k, int budget, int max_bits, int32_t* out) {
  if (!lambda || !out || k < 1 || budget < 0 || max_bits < 0)
    return fail(TQ_ERR_INVALID_ARG, "waterfill: bad arguments");
  for (int j = 0; j < k; ++j) out[j] = 0;
  for (int s = 0; s < budget; ++s) {
    int best = -1;
    double gain = -1.0;
    for (int j = 0; j < k; ++j) {
      if (out[j] >= max_bits) continue;
      const double g = lambda[j] * std::ldexp(1.0, -2 * out[j]);
      if (g > gain) { gain = g; best = j; }
    }
    if (best < 0) break;
    out[best] += 1;
  }
  return TQ_OK;
}

tq_status spectral_calibrate(const float* X, int64_t n, int d, double* vecs, double* vals) {
  if (!X || !vecs || !vals || n < 1 || d < 1 || d > 1024)
    return fail(TQ_ERR_INVALID_ARG, "calibrate: bad arguments");
  std::vector<double> A((size_t)d * d, 0.0), V((size_t)d * d, 0.0);
  std::vector<double> row(d);
  for (int64_t i = 0; i < n; ++i) {
    for (int j = 0; j < d; ++j) row[j] = X[i * d + j];
    for (int a = 0; a < d; ++a) {
      const double ra = row[a];
      double* Ar = &A[(size_t)a * d];
      for (int b = a; b < d; ++b) Ar[b] += ra * row[b];
    }
  }
  for (int a = 0; a < d; ++a)
    for (int b = a; b < d; ++b) {
      A[(size_t)a * d + b] /= (double)n;
      A[(size_t)b * d + a] = A[(size_t)a * d + b];
    }
  for (int a = 0; a < d; ++a) V[(size_t)a * d + a] = 1.0;
  // Cyclic Jacobi: annihilate each off-diagonal pair with a plane rotation.
  double total = 0.0;
  for (int a = 0; a < d; ++a)
    for (int b = 0; b < d; ++b) total += A[(size_t)a * d + b] * A[(size_t)a * d + b];
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0;
    for (int a = 0; a < d; ++a)
      for (int b = a + 1; b < d; ++b) off += A[(size_t)a * d + b] * A[(size_t)a * d + b];
    if (off <= 1e-30 * total) break;
    for (int p = 0; p < d; ++p) {
      for (int q = p + 1; q < d; ++q) {
        const double apq = A[(size_t)p * d + q];
        if (std::fabs(apq) < 1e-300) continue;
        const double app = A[(size_t)p * d + p], aqq = A[(size_t)q * d + q];
        const double theta = (aqq - app) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        for (int k = 0; k < d; ++k) {  // columns p, q
          const double akp = A[(size_t)k * d + p], akq = A[(size_t)k * d + q];
          A[(size_t)k * d + p] = c * akp - s * akq;
          A[(size_t)k * d + q] = s * akp + c * akq;
        }
        for (int k = 0; k < d; ++k) {  // rows p, q
          const double apk = A[(size_t)p * d + k], aqk = A[(size_t)q * d + k];
          A[(size_t)p * d + k] = c * apk - s * aqk;
          A[(size_t)q * d + k] = s * apk + c * aqk;
        }
        for (int k = 0; k < d; ++k) {  // eigenvector columns
          const double vkp = V[(size_t)k * d + p], vkq = V[(size_t)k * d + q];
          V[(size_t)k * d + p] = c * vkp - s * vkq;
          V[(size_t)k * d + q] = s * vkp + c * vkq;
        }
      }
    }
  }
  std::vector<int> order(d);
  for (int j = 0; j < d; ++j) order[j] = j;
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) {
    return A[(size_t)x * d + x] > A[(size_t)y * d + y];
  });
  for (int r = 0; r < d; ++r) {
    const int j = order[r];
    vals[r] = A[(size_t)j * d + j];
    int arg = 0;
    double best = -1.0;
    for (int k = 0; k < d; ++k) {
      const double v = std::fabs(V[(size_t)k * d + j]);
      if (v > best) { best = v; arg = k; }
    }
    const double sgn = V[(size_t)arg * d + j] < 0 ? -1.0 : 1.0;
    for (int k = 0; k < d; ++k) vecs[(size_t)r * d + k] = sgn * V[(size_t)k * d + j];
  }
  return TQ_OK;
}

tq_status lut_scale(const double* values, int count, float* scale_out) {
  if (!values || !scale_out || count < 1) return fail(TQ_ERR_INVALID_ARG, "lut_scale: bad arguments");
  std::vector<double> mags;
  for (int i = 0; i < count; ++i) {
    const double a = std::fabs(values[i]);
    if (a > 0.0 && std::isfinite(a)) mags.push_back(a);
  }
  std::sort(mags.begin(), mags.end());
  mags.erase(std::unique(mags.begin(), mags.end()), mags.end());
  if (mags.empty()) { *scale_out = 1.0f; return TQ_OK; }
  // relative rounding error of v to the nearest half-precision value (normal range)
  auto rel_err = [](double v) {
    int e;
    std::frexp(v, &e);                       // v = f * 2^e, f in [0.5, 1)
    const double ulp = std::ldexp(1.0, e - 11);
    const double r = std::nearbyint(v / ulp) * ulp;
    return std::fabs(r - v) / v;
  };
  const int steps = 1 << 22;
  double best_s = 1.0, best = 1e9;
  for (int i = 0; i < steps; ++i) {
    const double sc = 1.0 + static_cast<double>(i) / steps;
    double worst = 0.0;
    for (double m : mags) {
      worst = std::max(worst, rel_err(m / sc));
      if (worst >= best) break;
    }
    if (worst < best) { best = worst; best_s = sc; }
  }
  *scale_out = static_cast<float>(best_s);
  return TQ_OK;
}

tq_status spectral_unit_codebooks(double* c_out, double* t_out) {
  if (!c_out || !t_out) return fail(TQ_ERR_INVALID_ARG, "unit codebooks: null output");
  for (int b = 1; b <= 8; ++b) {
    const tq_status s = codebook_build(0, b, TQ_DIST_GAUSSIAN, 1.0, c_out + ((1 << b) - 2),
                                       t_out + ((1 << b) - b - 1), nullptr);
    if (s != TQ_OK) return s;
  }
  return TQ_OK;
}

tq_status spectral_descriptor(const double* vecs, const double* vals, int d, int k_top, int budget, int tail_bits,
                              int max_bits, float* rot_out, float* sigma_out, float* unit_c_out, float* unit_t_out,
                              int32_t* top_bits_out, float* lut_scale_out) {
  if (!vecs || !vals || !rot_out || !sigma_out || !unit_c_out || !unit_t_out || !top_bits_out || !lut_scale_out)
    return fail(TQ_ERR_INVALID_ARG, "spectral descriptor: null argument");
  if (d < 2 || d > 1024 || k_top < 1 || k_top > TQ_MAX_TOP || k_top > d || budget < 0 || tail_bits < 1 ||
      tail_bits > 4 || max_bits < 1 || max_bits > 8)
    return fail(TQ_ERR_INVALID_ARG, "spectral descriptor: size out of range");
  // bits of the signal dims: reverse water-filling over their eigenvalues (negative sample
  // eigenvalues of a rank-deficient calibration count as zero variance)
  std::vector<double> lam(d);
  for (int j = 0; j < d; ++j) lam[j] = std::isfinite(vals[j]) ? std::max(vals[j], 0.0) : 0.0;
  tq_status s = waterfill(lam.data(), k_top, budget, max_bits, top_bits_out);
  if (s != TQ_OK) return s;
  int top_sum = 0;
  for (int j = 0; j < k_top; ++j) top_sum += top_bits_out[j];
  if (top_sum + k_top > 32) return fail(TQ_ERR_UNSUPPORTED, "spectral descriptor: top bits + signs exceed one word");
  // dim j's codebook is sqrt(lambda_j) times the unit-normal Lloyd-Max codebook
  for (int j = 0; j < d; ++j) sigma_out[j] = static_cast<float>(std::sqrt(lam[j]));
  for (size_t i = 0; i < static_cast<size_t>(d) * d; ++i) rot_out[i] = static_cast<float>(vecs[i]);
  std::vector<double> uc(510), ut(502);
  if ((s = spectral_unit_codebooks(uc.data(), ut.data())) != TQ_OK) return s;
  for (int i = 0; i < 510; ++i) unit_c_out[i] = static_cast<float>(uc[i]);
  for (int i = 0; i < 502; ++i) unit_t_out[i] = static_cast<float>(ut[i]);
  // half-precision table of the tail codebook (the top dims are decoded in fp32)
  return lut_scale(uc.data() + ((1 << tail_bits) - 2), 1 << tail_bits, lut_scale_out);
}

}  // namespace tq
