// Host-side parts of libtq: error reporting and the Lloyd-Max codebook.
//
// Codebook (aiboss88 page, "TurboQuant technical principles": Beta-distributed coordinates after a
// random rotation, Lloyd-Max / continuous 1-D k-means codebook computed once; techblog-plum page,
// step 1: precomputed, no inference-time cost).
//
// One coordinate X of a uniform unit vector in R^d has density proportional to (1 - x^2)^((d-3)/2)
// on [-1, 1]. With x = sin(theta) this becomes cos(theta)^(d-2) d(theta) on [-pi/2, pi/2], which is
// smooth for every d >= 3, so the cell probabilities are computed by composite Gauss-Legendre
// quadrature in theta. The first moment has a closed form,
//   int_{theta_a}^{theta_b} sin(theta) cos(theta)^(d-2) d(theta) = (cos^(d-1) theta_a - cos^(d-1) theta_b)/(d-1),
// and the normalising constant cancels in every centroid (first moment / probability).
// Lloyd-Max alternates midpoint boundaries and conditional-mean centroids on the positive half
// (the density is symmetric, so t_{L/2} = 0 exactly and the negative half is the mirror image).
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "tq_internal.h"

namespace tq {

static thread_local std::string g_last_error;

tq_status fail(tq_status code, const std::string& msg) {
  g_last_error = msg;
  return code;
}
void clear_error() { g_last_error.clear(); }

bool valid_dim(int d) { return d >= 32 && d <= 4096 && d % 32 == 0; }

namespace {

// Gauss-Legendre nodes / weights on [-1, 1] by Newton's method on P_n (three-term recurrence).
struct GaussLegendre {
  std::vector<double> x, w;
  explicit GaussLegendre(int n) : x(n), w(n) {
    for (int i = 0; i < (n + 1) / 2; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
      double dp = 0;
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = 0.0;
        for (int j = 1; j <= n; ++j) {
          double p2 = p1;
          p1 = p0;
          p0 = ((2.0 * j - 1.0) * z * p1 - (j - 1.0) * p2) / j;
        }
        dp = n * (z * p0 - p1) / (z * z - 1.0);
        double dz = p0 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) break;
      }
      x[i] = -z;
      x[n - 1 - i] = z;
      w[i] = w[n - 1 - i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

const GaussLegendre& gl() {
  static const GaussLegendre g(48);
  return g;
}

// integral of cos(theta)^(d-2) over [ta, tb] (0 <= ta <= tb <= pi/2), panels no wider than
// a quarter of the standard deviation of theta (about 1/sqrt(d)).
double cell_mass(double ta, double tb, int d) {
  if (tb <= ta) return 0.0;
  const double e = d - 2.0;
  const double hmax = 0.25 / std::sqrt((double)d);
  // beyond theta_cut the integrand is below 1e-320 of its peak
  double cut = std::acos(std::exp(-745.0 / std::max(e, 1.0)));
  if (e < 1.0) cut = M_PI / 2;
  tb = std::min(tb, std::max(cut, ta));
  if (tb <= ta) return 0.0;
  int panels = std::max(1, (int)std::ceil((tb - ta) / hmax));
  double h = (tb - ta) / panels, acc = 0.0;
  const GaussLegendre& g = gl();
  for (int p = 0; p < panels; ++p) {
    double a = ta + p * h, mid = a + 0.5 * h, s = 0.0;
    for (size_t k = 0; k < g.x.size(); ++k) {
      const double sn = std::sin(mid + 0.5 * h * g.x[k]);
      // cos^e = exp(e/2 log(1 - sin^2)): log1p keeps full relative accuracy near theta = 0,
      // where log(cos) would lose it (its absolute error is multiplied by e ~ d)
      s += g.w[k] * std::exp(0.5 * e * std::log1p(-sn * sn));
    }
    acc += 0.5 * h * s;
  }
  return acc;
}

// integral of sin cos^(d-2) over [asin xa, asin xb] in closed form: ((1-xa^2)^((d-1)/2) - (1-xb^2)^((d-1)/2)) / (d-1)
double cell_moment(double xa, double xb, int d) {
  auto cpow = [d](double x) { return x >= 1.0 ? 0.0 : std::exp(0.5 * (d - 1.0) * std::log1p(-x * x)); };
  return (cpow(xa) - cpow(xb)) / (d - 1.0);
}

}  // namespace

}  // namespace tq

using namespace tq;

extern "C" TQ_API const char* tq_last_error(void) { return g_last_error.c_str(); }

extern "C" TQ_API const char* tq_version(void) { return "libtq 0.1 (sm_100a)"; }

extern "C" TQ_API tq_status tq_codebook_init(int32_t d, int32_t bits, tq_codebook* out) {
  clear_error();
  if (!out) return fail(TQ_ERR_INVALID_ARG, "tq_codebook_init: out is NULL");
  if (d < 3 || d > (1 << 20)) return fail(TQ_ERR_UNSUPPORTED, "tq_codebook_init: need 3 <= d <= 2^20");
  if (bits < 1 || bits > 4) return fail(TQ_ERR_UNSUPPORTED, "tq_codebook_init: need 1 <= bits <= 4");
  const int L = 1 << bits, H = L / 2;
  std::vector<double> c(H), nc(H), edge(H + 1);
  // start: evenly spread over three standard deviations
  for (int k = 0; k < H; ++k) c[k] = std::min(0.999, (k + 0.5) / H * 3.0 / std::sqrt((double)d));
  bool converged = false;
  double best = INFINITY;
  int stale = 0, it = 0;
  const double tol = 1e-14;
  for (it = 1; it <= 200000; ++it) {
    edge[0] = 0.0;
    for (int k = 1; k < H; ++k) edge[k] = 0.5 * (c[k - 1] + c[k]);
    edge[H] = 1.0;
    double delta = 0.0;
    for (int k = 0; k < H; ++k) {
      double ta = std::asin(edge[k]), tb = std::asin(edge[k + 1]);
      double m = cell_mass(ta, tb, d);
      nc[k] = (m > 0) ? cell_moment(edge[k], edge[k + 1], d) / m : 0.5 * (edge[k] + edge[k + 1]);
      delta = std::max(delta, std::fabs(nc[k] - c[k]));
    }
    c.swap(nc);
    if (delta <= tol * c[H - 1]) converged = true;
    if (delta < best) {
      best = delta;
      stale = 0;
    } else {
      ++stale;
    }
    if (converged && (stale >= 50 || delta == 0.0)) break;
  }
  if (!converged) return fail(TQ_ERR_NOT_CONVERGED, "tq_codebook_init: Lloyd-Max iteration did not converge");
  std::memset(out, 0, sizeof(*out));
  out->d = d;
  out->bits = bits;
  out->levels = L;
  out->iterations = it;
  for (int k = 0; k < H; ++k) {
    out->c64[H + k] = c[k];
    out->c64[H - 1 - k] = -c[k];
  }
  for (int k = 0; k + 1 < L; ++k) out->t64[k] = 0.5 * (out->c64[k] + out->c64[k + 1]);
  out->t64[H - 1] = 0.0;
  for (int k = 0; k < L; ++k) out->c[k] = (float)out->c64[k];
  for (int k = 0; k + 1 < L; ++k) out->t[k] = (float)out->t64[k];
  // distortion E|u - Q(u)|^2 = 1 - d sum_k c_k^2 P_k; by symmetry the sum is twice the positive
  // half, and a positive cell's P_k is its mass over twice the half-range mass, so the factors cancel
  double total = cell_mass(0.0, M_PI / 2, d), acc = 0.0;
  for (int k = 0; k < H; ++k) {
    double e0 = k == 0 ? 0.0 : 0.5 * (c[k - 1] + c[k]);
    double e1 = k == H - 1 ? 1.0 : 0.5 * (c[k] + c[k + 1]);
    acc += c[k] * c[k] * cell_mass(std::asin(e0), std::asin(e1), d) / total;
  }
  out->distortion = 1.0 - d * acc;
  return TQ_OK;
}

namespace tq {

int walsh_planes(const tq_codebook* cb, int* mask, float* beta) {
  const int L = cb->levels, bits = cb->bits;
  int n = 0;
  for (int m = 1; m < (1 << bits); ++m) {
    if (!(__builtin_popcount(m) & 1)) continue;
    double acc = 0.0;
    for (int idx = 0; idx < L; ++idx) {
      const int par = __builtin_popcount(idx & m) & 1;      // XOR of the planes in the subset
      acc += (double)cb->c[idx] * (par ? -1.0 : 1.0);       // prod (1 - 2 bit) = 1 - 2 parity
    }
    mask[n] = m;
    beta[n] = (float)(acc / L);
    ++n;
  }
  return n;
}

}  // namespace tq
