// Host-side method setup: the Lloyd-Max codebook of the rotated coordinate and
// the Haar orthogonal matrix. Both run once per (d, bits) / per rotation draw,
// in fp64, on the CPU; neither is on the per-token path.
#include <cmath>
#include <cstring>
#include <vector>

#include "tq_internal.h"

namespace tq {
namespace {

// Gauss-Legendre nodes and weights on [-1, 1] by Newton's method on P_n, with
// P_n and P_n' from Bonnet's three-term recurrence (the classical construction).
struct GaussLegendre {
  std::vector<double> x, w;
  explicit GaussLegendre(int n) : x(n), w(n) {
    for (int i = 0; i < n; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
      double dp = 1.0;
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = z;
        for (int k = 2; k <= n; ++k) {
          double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
          p0 = p1;
          p1 = p2;
        }
        // p1 = P_n(z), p0 = P_{n-1}(z)
        dp = n * (z * p1 - p0) / (z * z - 1.0);
        double dz = p1 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) break;
      }
      x[i] = z;
      w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

// Law of one coordinate of a uniform random unit vector in R^d:
// f(x) = C_d (1 - x^2)^((d-3)/2) on [-1, 1].
struct SphereCoordinate {
  int d;
  double log_c, alpha;
  explicit SphereCoordinate(int d_) : d(d_) {
    log_c = std::lgamma(d / 2.0) - 0.5 * std::log(M_PI) - std::lgamma((d - 1) / 2.0);
    alpha = (d - 3) / 2.0;
  }
  double pdf(double x) const {
    double s = 1.0 - x * x;
    if (s <= 0.0) return 0.0;
    return std::exp(log_c + alpha * std::log(s));
  }
  // int_a^b x f(x) dx from the antiderivative -(1-x^2)^(alpha+1) / (2 (alpha+1)).
  double first_moment(double a, double b) const {
    auto g = [&](double x) {
      double s = 1.0 - x * x;
      return s <= 0.0 ? 0.0 : std::exp(log_c + (alpha + 1.0) * std::log(s));
    };
    return (g(a) - g(b)) / (2.0 * (alpha + 1.0));
  }
};

double integrate_mass(const SphereCoordinate& f, const GaussLegendre& gl, double a, double b,
                      int panels) {
  double h = (b - a) / panels, total = 0.0;
  for (int p = 0; p < panels; ++p) {
    double lo = a + p * h, mid = lo + 0.5 * h, sum = 0.0;
    for (size_t i = 0; i < gl.x.size(); ++i) sum += gl.w[i] * f.pdf(mid + 0.5 * h * gl.x[i]);
    total += 0.5 * h * sum;
  }
  return total;
}

}  // namespace

// Returns 0 on success, 1 if the iteration did not converge.
int lloyd_max_sphere(int d, int bits, double* centroids, double* boundaries) {
  const int L = 1 << bits;
  SphereCoordinate f(d);
  GaussLegendre gl(24);
  std::vector<double> c(L), next(L), edges(L + 1);
  const double spread = 2.0 / std::sqrt((double)d);
  for (int k = 0; k < L; ++k) c[k] = (L == 1) ? 0.0 : -spread + 2.0 * spread * k / (L - 1);
  for (int it = 0; it < 20000; ++it) {
    edges[0] = -1.0;
    edges[L] = 1.0;
    for (int k = 1; k < L; ++k) edges[k] = 0.5 * (c[k - 1] + c[k]);
    double moved = 0.0;
    for (int k = 0; k < L; ++k) {
      double mass = integrate_mass(f, gl, edges[k], edges[k + 1], 96);
      next[k] = f.first_moment(edges[k], edges[k + 1]) / mass;
      moved = std::fmax(moved, std::fabs(next[k] - c[k]));
    }
    c.swap(next);
    if (moved < 1e-15) {
      // The density is even, so the optimal codebook is odd; impose it exactly.
      for (int k = 0; k < L; ++k) next[k] = 0.5 * (c[k] - c[L - 1 - k]);
      c.swap(next);
      for (int k = 0; k < L; ++k) centroids[k] = c[k];
      for (int k = 1; k < L; ++k) boundaries[k - 1] = 0.5 * (c[k - 1] + c[k]);
      return 0;
    }
  }
  return 1;
}

// Householder QR of the row-major d x d matrix g; writes Q with diag(R) > 0.
// Returns 0 on success, 1 if a column is exactly dependent.
int haar_from_gaussian(int d, const double* g, double* q) {
  std::vector<double> a(g, g + (size_t)d * d), v(d), qv(d);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) q[(size_t)i * d + j] = (i == j) ? 1.0 : 0.0;
  std::vector<double> rdiag(d);
  for (int k = 0; k < d; ++k) {
    double norm2 = 0.0;
    for (int i = k; i < d; ++i) norm2 += a[(size_t)i * d + k] * a[(size_t)i * d + k];
    double norm = std::sqrt(norm2);
    if (norm == 0.0) return 1;
    double x0 = a[(size_t)k * d + k];
    double alpha = (x0 >= 0.0) ? -norm : norm;
    double vnorm2 = 0.0;
    for (int i = k; i < d; ++i) {
      v[i] = a[(size_t)i * d + k] - (i == k ? alpha : 0.0);
      vnorm2 += v[i] * v[i];
    }
    rdiag[k] = alpha;
    if (vnorm2 == 0.0) continue;  // column already in place (alpha = x0)
    double beta = 2.0 / vnorm2;
    // A[k:, k:] -= beta v (v^T A[k:, k:])
    for (int j = k; j < d; ++j) {
      double s = 0.0;
      for (int i = k; i < d; ++i) s += v[i] * a[(size_t)i * d + j];
      s *= beta;
      for (int i = k; i < d; ++i) a[(size_t)i * d + j] -= s * v[i];
    }
    // Q[:, k:] -= beta (Q[:, k:] v) v^T
    for (int i = 0; i < d; ++i) {
      double s = 0.0;
      for (int j = k; j < d; ++j) s += q[(size_t)i * d + j] * v[j];
      s *= beta;
      for (int j = k; j < d; ++j) q[(size_t)i * d + j] -= s * v[j];
    }
  }
  for (int k = 0; k < d; ++k) {
    if (rdiag[k] < 0.0)
      for (int i = 0; i < d; ++i) q[(size_t)i * d + k] = -q[(size_t)i * d + k];
  }
  return 0;
}

}  // namespace tq
