// Host-side Lloyd-Max fitter for the coordinate law of a random unit vector.
//
// zubnet.ai news, "Google's TurboQuant quantizes LLM KV cache to 3.5 bits per
// channel", paragraph 2: after a random rotation each coordinate follows a Beta
// law, and an optimal scalar quantizer is applied per coordinate. The law of one
// coordinate y of a uniform point on S^{d-1} has density proportional to
// (1 - y^2)^((d-3)/2). With y = sin(theta) the mass of [0, y] is
//   C * W_{d-2}(asin y),  W_n(theta) = int_0^theta cos^n(t) dt,
// and W_n follows the Wallis recurrence
//   W_n = cos^{n-1}(theta) sin(theta) / n + (n-1)/n * W_{n-2},
//   W_0 = theta, W_1 = sin(theta),
// whose terms are all non-negative on [0, pi/2] (no cancellation). The
// normaliser is C = 1 / (2 W_{d-2}(pi/2)). The first moment of a cell has the
// elementary antiderivative -(1-y^2)^((d-1)/2) / (d-1). Lloyd's iteration
// (thresholds at centroid midpoints, centroids at cell means) has a unique
// fixed point because the density is log-concave, so the starting point only
// affects the number of sweeps.
#include <cmath>
#include <cstdint>
#include <vector>

namespace tq {

namespace {

double wallis(int n, double theta) {
  const double s = std::sin(theta), c = std::cos(theta);
  double w = (n % 2 == 0) ? theta : s;
  double cpow = (n % 2 == 0) ? c : c * c;   // cos^{k-1} for the first step k = 2 or 3
  for (int k = (n % 2 == 0) ? 2 : 3; k <= n; k += 2) {
    w = cpow * s / k + (double)(k - 1) / k * w;
    cpow *= c * c;
  }
  return w;
}

struct Law {
  int d;
  double norm;   // C
  explicit Law(int d_) : d(d_) { norm = 1.0 / (2.0 * wallis(d - 2, M_PI / 2)); }
  // P(Y <= y)
  double cdf(double y) const {
    if (y <= -1.0) return 0.0;
    if (y >= 1.0) return 1.0;
    const double half = norm * wallis(d - 2, std::asin(std::fabs(y)));
    return y >= 0 ? 0.5 + half : 0.5 - half;
  }
  // int_a^b y f(y) dy
  double moment(double a, double b) const {
    auto g = [&](double y) {
      if (std::fabs(y) >= 1.0) return 0.0;
      return std::pow(1.0 - y * y, 0.5 * (d - 1));
    };
    return norm / (d - 1) * (g(a) - g(b));
  }
};

}  // namespace

// Returns false if the iteration produced a non-finite value.
bool fit_lloyd_max(int d, int bits, float *out) {
  const int L = 1 << bits;
  const Law law(d);
  std::vector<double> c(L), nc(L), edge(L + 1);
  const double spread = std::fmin(2.5 / std::sqrt((double)d), 0.9);
  for (int j = 0; j < L; ++j) c[j] = spread * (2.0 * j + 1 - L) / L;
  for (int sweep = 0; sweep < 400000; ++sweep) {
    edge[0] = -1.0;
    edge[L] = 1.0;
    for (int j = 1; j < L; ++j) edge[j] = 0.5 * (c[j - 1] + c[j]);
    double move = 0.0;
    for (int j = 0; j < L; ++j) {
      const double mass = law.cdf(edge[j + 1]) - law.cdf(edge[j]);
      // an empty cell (possible only far in the tails) keeps its midpoint
      nc[j] = mass > 1e-300 ? law.moment(edge[j], edge[j + 1]) / mass : 0.5 * (edge[j] + edge[j + 1]);
      move = std::fmax(move, std::fabs(nc[j] - c[j]));
    }
    c.swap(nc);
    if (move < 1e-15) break;
  }
  for (int j = 0; j < L; ++j) {
    const double v = 0.5 * (c[j] - c[L - 1 - j]);
    if (!std::isfinite(v)) return false;
    out[j] = (float)v;
  }
  return true;
}

}  // namespace tq
