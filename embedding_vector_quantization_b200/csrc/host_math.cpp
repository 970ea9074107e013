// Host-side math of the library: the seeded Gaussian stream, the Householder QR
// that turns it into the rotation Pi, and the Lloyd-Max codebook builder.
//
// "Google TurboQuant: 6x KV-cache compression" (ebisuda.net), section
// "Stage 1: PolarQuant (MSE-optimal compression)": the rotation is the
// orthogonal factor of a QR decomposition of a Gaussian matrix; each rotated
// coordinate then follows a known law, on which a Lloyd-Max quantizer
// (continuous k-means) is precomputed per bit width, independent of the data.
//
// Choices the pages leave open (shared with the test oracle only as a written
// spec, never as code):
//  * generator: SplitMix64 (Steele, Lea & Flood 2014), uniforms from the top 53
//    bits, Box-Muller pairs with u1 = 1 - a, u2 = b, cosine output first; G is
//    filled row-major, then S continues the stream;
//  * QR sign convention: diag(R) > 0 (Haar-distributed Q);
//  * coordinate law: (1 - t^2)^((d-3)/2) on [-1, 1]; cell masses by composite
//    Gauss-Legendre quadrature in theta = asin(t), where the integrand
//    cos(theta)^(d-2) is smooth for every d >= 3; cell first moments from the
//    closed form of int t (1 - t^2)^k dt;
//  * Lloyd start at the quantiles (i + 1/2) / L, stop when no centroid moves by
//    1e-15 (or 1e5 iterations), then force exact odd symmetry.
//
// The angle codebooks of the recursive polar transform ("PolarQuant explainer"
// (aibr.jp), sections 1 and 3: angles quantized with codebooks designed from their
// analytic distribution) follow the same Lloyd iteration on each level's law.

#include "host_math.h"

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <vector>

namespace tqhost {

// ---------------------------------------------------------------- generator

namespace {
inline uint64_t splitmix_next(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ULL;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}
inline double unit53(uint64_t v) { return static_cast<double>(v >> 11) * 0x1.0p-53; }
}  // namespace

void gaussian_stream(uint64_t seed, size_t count, double* out) {
  uint64_t state = seed;
  const double two_pi = 6.283185307179586476925286766559;
  for (size_t i = 0; i < count; i += 2) {
    const double a = unit53(splitmix_next(state));
    const double b = unit53(splitmix_next(state));
    const double r = std::sqrt(-2.0 * std::log(1.0 - a));
    out[i] = r * std::cos(two_pi * b);
    if (i + 1 < count) out[i + 1] = r * std::sin(two_pi * b);
  }
}

// ---------------------------------------------------------------- rotation

// In-place Householder QR of the row-major n x n matrix A. On return Q (n x n,
// row-major) holds the orthogonal factor with every column multiplied by the
// sign of the matching diagonal entry of R, so that A = Q R with diag(R) > 0.
static void householder_q(int n, std::vector<double>& A, std::vector<double>& Q) {
  std::vector<double> V(static_cast<size_t>(n) * n, 0.0);  // reflector k in column k, rows k..n-1
  std::vector<double> rdiag(n), w(n);
  for (int k = 0; k < n; ++k) {
    double norm2 = 0.0;
    for (int i = k; i < n; ++i) norm2 += A[(size_t)i * n + k] * A[(size_t)i * n + k];
    const double norm = std::sqrt(norm2);
    const double x0 = A[(size_t)k * n + k];
    const double alpha = (x0 >= 0.0) ? -norm : norm;   // reflect away from x0 (no cancellation)
    // v = x - alpha e1, normalised
    double vnorm2 = 0.0;
    for (int i = k; i < n; ++i) {
      const double vi = A[(size_t)i * n + k] - (i == k ? alpha : 0.0);
      V[(size_t)i * n + k] = vi;
      vnorm2 += vi * vi;
    }
    rdiag[k] = alpha;
    if (vnorm2 == 0.0) continue;  // column already reduced
    const double inv = 1.0 / std::sqrt(vnorm2);
    for (int i = k; i < n; ++i) V[(size_t)i * n + k] *= inv;
    // A[k:, k:] -= 2 v (v^T A[k:, k:])
    std::fill(w.begin() + k, w.end(), 0.0);
    for (int i = k; i < n; ++i) {
      const double vi = V[(size_t)i * n + k];
      const double* row = &A[(size_t)i * n];
      for (int j = k; j < n; ++j) w[j] += vi * row[j];
    }
    for (int i = k; i < n; ++i) {
      const double s = 2.0 * V[(size_t)i * n + k];
      double* row = &A[(size_t)i * n];
      for (int j = k; j < n; ++j) row[j] -= s * w[j];
    }
  }
  // Q = H_0 H_1 ... H_{n-1}: apply the reflectors in reverse order to I.
  Q.assign(static_cast<size_t>(n) * n, 0.0);
  for (int i = 0; i < n; ++i) Q[(size_t)i * n + i] = 1.0;
  for (int k = n - 1; k >= 0; --k) {
    std::fill(w.begin() + k, w.end(), 0.0);
    for (int i = k; i < n; ++i) {
      const double vi = V[(size_t)i * n + k];
      if (vi == 0.0) continue;
      const double* row = &Q[(size_t)i * n];
      for (int j = k; j < n; ++j) w[j] += vi * row[j];
    }
    for (int i = k; i < n; ++i) {
      const double s = 2.0 * V[(size_t)i * n + k];
      if (s == 0.0) continue;
      double* row = &Q[(size_t)i * n];
      for (int j = k; j < n; ++j) row[j] -= s * w[j];
    }
  }
  // Sign fix: column k of Q times sign(R_kk) makes diag(R) positive.
  for (int k = 0; k < n; ++k) {
    if (rdiag[k] < 0.0)
      for (int i = 0; i < n; ++i) Q[(size_t)i * n + k] = -Q[(size_t)i * n + k];
  }
}

void rotation(int d, int m, uint64_t seed, double* Pi, double* S) {
  const size_t dd = static_cast<size_t>(d) * d;
  std::vector<double> g(dd + static_cast<size_t>(m) * d);
  gaussian_stream(seed, g.size(), g.data());
  std::vector<double> A(g.begin(), g.begin() + dd), Q;
  householder_q(d, A, Q);
  std::copy(Q.begin(), Q.end(), Pi);
  if (m > 0 && S != nullptr) std::copy(g.begin() + dd, g.end(), S);
}

// ---------------------------------------------------------------- codebook

namespace {

// 20-point Gauss-Legendre nodes/weights on [-1, 1] (computed once by Newton's
// method on the Legendre recurrence).
struct GaussLegendre {
  static constexpr int kN = 20;
  double x[kN], w[kN];
  GaussLegendre() {
    for (int i = 0; i < kN; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (kN + 0.5));
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = z;
        for (int k = 2; k <= kN; ++k) {
          const double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
          p0 = p1;
          p1 = p2;
        }
        const double dp = kN * (z * p1 - p0) / (z * z - 1.0);
        const double dz = p1 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-17) break;
      }
      double p0 = 1.0, p1 = z;
      for (int k = 2; k <= kN; ++k) {
        const double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
        p0 = p1;
        p1 = p2;
      }
      const double dp = kN * (z * p1 - p0) / (z * z - 1.0);
      x[i] = z;
      w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

const GaussLegendre& gl() {
  static const GaussLegendre g;
  return g;
}

// The coordinate law of a uniform unit vector in R^d, through theta = asin(t):
// P(a < T <= b) = int_{asin a}^{asin b} cos^(d-2)(theta) dtheta / Z.
struct CoordLaw {
  int d;
  double p;          // exponent d - 2
  double k1;         // (d - 1) / 2 = k + 1
  double theta_max;  // beyond this the mass is below 1e-300 relative
  double panel;      // quadrature panel width in theta
  double logZ;

  explicit CoordLaw(int dim) : d(dim), p(dim - 2.0), k1((dim - 1) / 2.0) {
    const double tmax = std::min(1.0, 40.0 / std::sqrt(static_cast<double>(d)));
    theta_max = std::asin(tmax);
    panel = std::min(0.05, 0.25 / std::sqrt(static_cast<double>(d)));
    logZ = std::log(raw_integral(-theta_max, theta_max));
  }
  // cos^p(theta) with log(cos theta) = log1p(-2 sin^2(theta/2)): no cancellation near 0,
  // where p * log(cos theta) would otherwise lose ~1e-13 relative for large d.
  double integrand(double th) const {
    if (p == 0.0) return 1.0;
    const double s = std::sin(0.5 * th);
    const double arg = -2.0 * s * s;
    if (arg <= -1.0) return 0.0;
    return std::exp(p * std::log1p(arg));
  }
  double raw_integral(double lo, double hi) const {
    if (hi <= lo) return 0.0;
    const int panels = std::max(1, static_cast<int>(std::ceil((hi - lo) / panel)));
    const double h = (hi - lo) / panels;
    const GaussLegendre& g = gl();
    double sum = 0.0;
    for (int pi = 0; pi < panels; ++pi) {
      const double mid = lo + (pi + 0.5) * h;
      double s = 0.0;
      for (int i = 0; i < GaussLegendre::kN; ++i) s += g.w[i] * integrand(mid + 0.5 * h * g.x[i]);
      sum += 0.5 * h * s;
    }
    return sum;
  }
  double clip_theta(double t) const {
    const double th = std::asin(std::max(-1.0, std::min(1.0, t)));
    return std::max(-theta_max, std::min(theta_max, th));
  }
  double mass(double a, double b) const {
    return raw_integral(clip_theta(a), clip_theta(b)) / std::exp(logZ);
  }
  // int_a^b t (1-t^2)^k dt / Z = [(1-a^2)^(k+1) - (1-b^2)^(k+1)] / (2 (k+1) Z)
  double moment(double a, double b) const {
    auto g = [&](double t) {
      t = std::max(-1.0, std::min(1.0, t));
      if (t * t >= 1.0) return 0.0;
      return std::exp(k1 * std::log1p(-t * t) - logZ);
    };
    return (g(a) - g(b)) / (2.0 * k1);
  }
  double cdf(double t) const { return mass(-1.0, t); }
};

}  // namespace

int codebook(int d, int bits, double* centroids, double* bounds) {
  if (d < 3 || bits < 1 || bits > 8) return -1;
  const int L = 1 << bits;
  CoordLaw law(d);
  std::vector<double> c(L), nc(L), edge(L + 1);
  // start at the quantiles (i + 1/2)/L, found by bisection on the CDF
  for (int i = 0; i < L; ++i) {
    const double target = (i + 0.5) / L;
    double lo = -1.0, hi = 1.0;
    for (int it = 0; it < 200 && hi - lo > 1e-16; ++it) {
      const double mid = 0.5 * (lo + hi);
      (law.cdf(mid) < target ? lo : hi) = mid;
    }
    c[i] = 0.5 * (lo + hi);
  }
  for (int it = 0; it < 100000; ++it) {
    edge[0] = -1.0;
    edge[L] = 1.0;
    for (int i = 0; i + 1 < L; ++i) edge[i + 1] = 0.5 * (c[i] + c[i + 1]);
    double step = 0.0;
    for (int i = 0; i < L; ++i) {
      const double ms = law.mass(edge[i], edge[i + 1]);
      nc[i] = law.moment(edge[i], edge[i + 1]) / ms;
      step = std::max(step, std::fabs(nc[i] - c[i]));
    }
    c.swap(nc);
    if (step < 1e-15) break;
  }
  for (int i = 0; i < L; ++i) centroids[i] = 0.5 * (c[i] - c[L - 1 - i]);
  for (int i = 0; i + 1 < L; ++i) bounds[i] = 0.5 * (centroids[i] + centroids[i + 1]);
  return 0;
}

// ---------------------------------------------------------------- polar angle codebooks

namespace {

// Law of a level-l angle of the recursive polar transform of a uniform direction, l >= 2:
// density proportional to (sin psi cos psi)^(k-1) = (sin(2 psi) / 2)^(k-1) on [0, pi/2],
// k = 2^(l-1). Masses and first moments by composite Gauss-Legendre quadrature of the
// integrand scaled to 1 at its peak, sin(2 psi)^(k-1).
struct AngleLaw {
  double p;      // exponent k - 1
  double panel;  // quadrature panel width
  double Z;      // total mass of the scaled integrand

  explicit AngleLaw(int k) : p(k - 1.0) {
    panel = std::min(0.05, 0.3 / std::sqrt(static_cast<double>(k)));
    Z = raw(0.0, 0.5 * M_PI, false);
  }
  double integrand(double psi) const {
    const double s = std::sin(2.0 * psi);
    if (p == 0.0) return 1.0;
    if (s <= 0.0) return 0.0;
    return std::exp(p * std::log(s));
  }
  double raw(double lo, double hi, bool first_moment) const {
    if (hi <= lo) return 0.0;
    const int panels = std::max(1, static_cast<int>(std::ceil((hi - lo) / panel)));
    const double h = (hi - lo) / panels;
    const GaussLegendre& g = gl();
    double sum = 0.0;
    for (int pi = 0; pi < panels; ++pi) {
      const double mid = lo + (pi + 0.5) * h;
      double acc = 0.0;
      for (int i = 0; i < GaussLegendre::kN; ++i) {
        const double t = mid + 0.5 * h * g.x[i];
        acc += g.w[i] * integrand(t) * (first_moment ? t : 1.0);
      }
      sum += 0.5 * h * acc;
    }
    return sum;
  }
  double mass(double a, double b) const { return raw(a, b, false) / Z; }
  double moment(double a, double b) const { return raw(a, b, true) / Z; }
};

}  // namespace

int polar_codebook(int level, int bits, double* centroids, double* bounds) {
  if (level < 1 || level > 16 || bits < 1 || bits > 8) return -1;
  const int L = 1 << bits;
  if (level == 1) {
    // uniform on (-pi, pi]: the Lloyd fixed point is the uniform grid of L cells
    for (int i = 0; i < L; ++i) centroids[i] = -M_PI + (2.0 * i + 1.0) * M_PI / L;
    for (int i = 0; i + 1 < L; ++i) bounds[i] = -M_PI + 2.0 * (i + 1) * M_PI / L;
    return 0;
  }
  const AngleLaw law(1 << (level - 1));
  const double top = 0.5 * M_PI;
  std::vector<double> c(L), nc(L), edge(L + 1);
  for (int i = 0; i < L; ++i) {   // start at the quantiles (i + 1/2) / L
    const double target = (i + 0.5) / L;
    double lo = 0.0, hi = top;
    for (int it = 0; it < 200 && hi - lo > 1e-16; ++it) {
      const double mid = 0.5 * (lo + hi);
      (law.mass(0.0, mid) < target ? lo : hi) = mid;
    }
    c[i] = 0.5 * (lo + hi);
  }
  for (int it = 0; it < 100000; ++it) {
    edge[0] = 0.0;
    edge[L] = top;
    for (int i = 0; i + 1 < L; ++i) edge[i + 1] = 0.5 * (c[i] + c[i + 1]);
    double step = 0.0;
    for (int i = 0; i < L; ++i) {
      nc[i] = law.moment(edge[i], edge[i + 1]) / law.mass(edge[i], edge[i + 1]);
      step = std::max(step, std::fabs(nc[i] - c[i]));
    }
    c.swap(nc);
    if (step < 1e-15) break;
  }
  // the law is symmetric about pi/4
  for (int i = 0; i < L; ++i) centroids[i] = 0.5 * (c[i] + (top - c[L - 1 - i]));
  for (int i = 0; i + 1 < L; ++i) bounds[i] = 0.5 * (centroids[i] + centroids[i + 1]);
  return 0;
}

}  // namespace tqhost
