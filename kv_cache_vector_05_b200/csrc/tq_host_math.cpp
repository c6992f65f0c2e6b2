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

// Initial boundaries from the high-resolution optimal point density, proportional to
// f^(1/3) (Panter and Dite): the (i/L)-quantiles of that density, tabulated on a grid.
void point_density_edges(const SphereCoordinate& f, int L, std::vector<double>& e) {
  const int n = 200000;
  std::vector<double> cdf(n + 1, 0.0);
  const double h = 2.0 / n;
  double prev = std::cbrt(f.pdf(-1.0));
  for (int i = 1; i <= n; ++i) {
    const double cur = std::cbrt(f.pdf(-1.0 + i * h));
    cdf[i] = cdf[i - 1] + 0.5 * h * (prev + cur);
    prev = cur;
  }
  int j = 0;
  for (int k = 1; k < L; ++k) {
    const double target = cdf[n] * k / L;
    while (j < n && cdf[j + 1] < target) ++j;
    const double span = cdf[j + 1] - cdf[j];
    e[k - 1] = -1.0 + h * (j + (span > 0.0 ? (target - cdf[j]) / span : 0.0));
  }
}

// The Lloyd-Max conditions solved by Newton's method on the L - 1 boundaries: residual
// R_i = t_i - (c_i + c_{i+1}) / 2, where a cell mean moves with its right edge b as
// f(b)(b - c)/M0 and with its left edge a as f(a)(c - a)/M0, so the Jacobian is
// tridiagonal (Thomas algorithm). Steps are halved until the boundaries stay ordered.
// Returns 0 and the cell means in c on convergence.
int lloyd_max_newton(const SphereCoordinate& f, const GaussLegendre& gl, int L, std::vector<double>& c) {
  std::vector<double> e(L - 1), m0(L), edges(L + 1), res(L - 1), right(L - 1), left(L - 1), diag(L - 1),
      step(L - 1), cp(L - 1), dp(L - 1), cand(L - 1);
  point_density_edges(f, L, e);
  auto cells = [&]() {
    edges[0] = -1.0;
    edges[L] = 1.0;
    for (int k = 1; k < L; ++k) edges[k] = e[k - 1];
    for (int k = 0; k < L; ++k) {
      m0[k] = integrate_mass(f, gl, edges[k], edges[k + 1], 96);
      c[k] = f.first_moment(edges[k], edges[k + 1]) / m0[k];
    }
  };
  for (int it = 0; it < 60; ++it) {
    cells();
    for (int i = 0; i < L - 1; ++i) {
      const double fe = f.pdf(e[i]);
      res[i] = e[i] - 0.5 * (c[i] + c[i + 1]);
      right[i] = fe * (e[i] - c[i]) / m0[i];         // d c_i / d t_i
      left[i] = fe * (c[i + 1] - e[i]) / m0[i + 1];  // d c_{i+1} / d t_i
      diag[i] = 1.0 - 0.5 * (right[i] + left[i]);
    }
    // rows i: -left[i-1]/2 x_{i-1} + diag[i] x_i - right[i+1]/2 x_{i+1} = res[i]
    const int n = L - 1;
    cp[0] = n > 1 ? -0.5 * right[1] / diag[0] : 0.0;
    dp[0] = res[0] / diag[0];
    for (int i = 1; i < n; ++i) {
      const double lo = -0.5 * left[i - 1];
      const double den = diag[i] - lo * cp[i - 1];
      cp[i] = i < n - 1 ? -0.5 * right[i + 1] / den : 0.0;
      dp[i] = (res[i] - lo * dp[i - 1]) / den;
    }
    step[n - 1] = dp[n - 1];
    for (int i = n - 2; i >= 0; --i) step[i] = dp[i] - cp[i] * step[i + 1];
    double lam = 1.0;
    for (int tries = 0; tries < 60; ++tries) {
      bool ok = true;
      for (int i = 0; i < n; ++i) {
        cand[i] = e[i] - lam * step[i];
        if (cand[i] <= -1.0 || cand[i] >= 1.0 || (i > 0 && cand[i] <= cand[i - 1])) ok = false;
      }
      if (ok) break;
      lam *= 0.5;
    }
    double moved = 0.0;
    for (int i = 0; i < n; ++i) moved = std::fmax(moved, std::fabs(cand[i] - e[i]));
    e.swap(cand);
    if (moved < 1e-12) {  // the cell moments' rounding in the far tails floors the steps near 1e-13
      cells();
      return 0;
    }
  }
  return 1;
}

}  // namespace

// Returns 0 on success, 1 if the iteration did not converge.
int lloyd_max_sphere(int d, int bits, double* centroids, double* boundaries) {
  const int L = 1 << bits;
  SphereCoordinate f(d);
  GaussLegendre gl(24);
  std::vector<double> c(L), next(L), edges(L + 1);
  if (bits >= 5) {  // many levels: Newton's method on the same two conditions
    if (lloyd_max_newton(f, gl, L, c)) return 1;
    for (int k = 0; k < L; ++k) next[k] = 0.5 * (c[k] - c[L - 1 - k]);  // odd by symmetry, exactly
    for (int k = 0; k < L; ++k) centroids[k] = next[k];
    for (int k = 1; k < L; ++k) boundaries[k - 1] = 0.5 * (next[k - 1] + next[k]);
    return 0;
  }
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
