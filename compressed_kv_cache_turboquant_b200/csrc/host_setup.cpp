// Host-side setup of a TurboQuant instance: the Lloyd-Max codebook of the
// rotated-coordinate law and the Haar rotation from a Gaussian matrix.
// Plain C++ in float64; no CUDA.
//
// Pages:
//   [ttakun]  "KV缓存52GB瞬间爆内存？TurboQuant随机旋转+标量量化如何把LLM长上下文推理成本
//             砍到1/16且失真逼近理论极限" (ttakun.com/news/45354)
//   [tq.net]  turboquant.net/zh, "TurboQuant 最近的进展和外溢影响"
#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "tq_internal.h"

namespace tqi {

// ---------------------------------------------------------------------------
// Coordinate law f(x) = C (1 - x^2)^((d-3)/2) on [-1, 1]
// [tq.net, "TurboQuant 两阶段算法", 坐标分布公式].
//
// C = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) is evaluated through the ratio
// R(n) = Gamma(n + 1/2) / Gamma(n) = (sqrt(pi)/2) prod_{k=1}^{n-1} (k + 1/2)/k,
// a product of well-conditioned factors; a difference of two lgamma values
// near 4e3 (d = 1536) would lose ~12 digits of the first decimal places.
//   d odd  (d = 2n+1): C = R(n) / sqrt(pi)
//   d even (d = 2n)  : C = (n-1) / (sqrt(pi) R(n-1))
// With x = sin(theta) the law becomes C cos^(d-2)(theta) d(theta), smooth on
// the whole interval, so Gauss-Legendre in theta converges fast even at the
// ends; the first moment has the closed form
//   int_a^b x f(x) dx = C/(d-1) [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)].
// ---------------------------------------------------------------------------

static double gamma_ratio_half(int n) {  // R(n) for n >= 1
  double r = std::sqrt(M_PI) / 2.0;
  for (int k = 1; k < n; ++k) r *= (k + 0.5) / k;
  return r;
}

static double law_constant(int d) {
  if (d % 2 == 1) {
    int n = (d - 1) / 2;
    return gamma_ratio_half(n) / std::sqrt(M_PI);
  }
  int n = d / 2;
  return (n - 1) / (std::sqrt(M_PI) * gamma_ratio_half(n - 1));
}

struct GaussLegendre {
  std::vector<double> x, w;
  explicit GaussLegendre(int n) : x(n), w(n) {
    // Newton iteration on P_n from the Tricomi-style initial guesses
    for (int i = 0; i < n; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = z;
        for (int k = 2; k <= n; ++k) {
          double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
          p0 = p1;
          p1 = p2;
        }
        double dp = n * (z * p1 - p0) / (z * z - 1.0);
        double dz = p1 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) {
          // recompute the derivative at the converged node
          p0 = 1.0;
          p1 = z;
          for (int k = 2; k <= n; ++k) {
            double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
            p0 = p1;
            p1 = p2;
          }
          dp = n * (z * p1 - p0) / (z * z - 1.0);
          x[i] = z;
          w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
          break;
        }
      }
    }
  }
};

struct Law {
  int d;
  double C;
  double piece;  // theta step of the quadrature pieces
  const GaussLegendre* gl;

  // P[a < X <= b] = C int_{asin a}^{asin b} cos^(d-2)(theta) d(theta)
  double mass(double a, double b) const {
    double ta = std::asin(std::max(-1.0, std::min(1.0, a)));
    double tb = std::asin(std::max(-1.0, std::min(1.0, b)));
    if (tb <= ta) return 0.0;
    int pieces = std::max(1, (int)std::ceil((tb - ta) / piece));
    double h = (tb - ta) / pieces, s = 0.0;
    for (int p = 0; p < pieces; ++p) {
      double lo = ta + p * h, mid = lo + 0.5 * h, acc = 0.0;
      for (size_t i = 0; i < gl->x.size(); ++i) {
        double th = mid + 0.5 * h * gl->x[i];
        acc += gl->w[i] * std::pow(std::cos(th), d - 2);
      }
      s += 0.5 * h * acc;
    }
    return C * s;
  }

  // int_a^b x f(x) dx by the closed form; the power difference is taken as
  // e^B * -expm1(A - B) of the logs, which keeps relative accuracy when the
  // two powers are nearly equal
  double first_moment(double a, double b) const {
    double p = 0.5 * (d - 1);
    auto lg = [&](double v) {
      double s = std::min(v * v, 1.0);
      return s >= 1.0 ? -INFINITY : p * std::log1p(-s);
    };
    double A = lg(a), B = lg(b);
    double big = std::max(A, B), small = std::min(A, B);
    if (std::isinf(big)) return 0.0;
    double diff = std::isinf(small) ? std::exp(big) : std::exp(big) * -std::expm1(small - big);
    double sgn = (A >= B) ? 1.0 : -1.0;
    return C / (d - 1) * sgn * diff;
  }
};

}  // namespace tqi

using namespace tqi;

extern "C" int tq_make_codebook(int b, int d, double* centroids, double* thresholds) {
  TQ_TRACE("tq_make_codebook");
  if (!centroids) return set_error(TQ_EINVAL, "tq_make_codebook: centroids is NULL");
  if (b < 1 || b > 4 || d < 3 || d > TQ_MAX_DIM)
    return set_error(TQ_EUNSUPPORTED, "tq_make_codebook: need 1 <= b <= 4 and 3 <= d <= %d",
                     TQ_MAX_DIM);
  static const GaussLegendre gl(32);
  Law law{d, law_constant(d), 0.5 / std::sqrt((double)d), &gl};
  const int K = 1 << b;
  // outer cells carry no mass beyond 16 standard deviations (1/sqrt(d)) of the law
  const double reach = 16.0 / std::sqrt((double)d);
  std::vector<double> c(K), t(K - 1), cn(K);
  double s = std::min(3.0 / std::sqrt((double)d), 1.0);
  for (int k = 0; k < K; ++k) c[k] = ((2.0 * k + 1.0) / K - 1.0) * s;
  double best = INFINITY;
  int since_best = 0;
  for (int it = 0; it < 20000; ++it) {
    for (int k = 0; k + 1 < K; ++k) t[k] = 0.5 * (c[k] + c[k + 1]);
    for (int k = 0; k < K; ++k) {
      // quadrature range of the mass (outer cells clipped at `reach`), exact
      // range of the closed-form first moment
      double lo = (k == 0) ? std::max(-1.0, t[0] - reach) : t[k - 1];
      double hi = (k == K - 1) ? std::min(1.0, t[K - 2] + reach) : t[k];
      double m0 = law.mass(lo, hi);
      double m1 = law.first_moment(k == 0 ? -1.0 : t[k - 1], k == K - 1 ? 1.0 : t[k]);
      cn[k] = m1 / m0;
    }
    // the law is even: keep the codebook exactly symmetric
    double step = 0.0;
    for (int k = 0; k < K / 2; ++k) {
      const double v = 0.5 * (cn[K - 1 - k] - cn[k]);  // positive half
      step = std::max(step, std::fabs(v - c[K - 1 - k]));
      cn[K - 1 - k] = v;
      cn[k] = -v;
    }
    c.swap(cn);
    if (step < best) {
      best = step;
      since_best = 0;
    } else {
      ++since_best;
    }
    if (step == 0.0 || since_best >= 200) break;
  }
  for (int k = 0; k < K; ++k) centroids[k] = c[k];
  if (thresholds)
    for (int k = 0; k + 1 < K; ++k) thresholds[k] = 0.5 * (c[k] + c[k + 1]);
  return clear_error();
}

// ---------------------------------------------------------------------------
// Rotation: G = Q R by Householder reflections; Pi = Q diag(sign(diag R))
// [ttakun, "为什么随机旋转是整个算法的底层杠杆"]; [tq.net, "实现步骤草图", 生成随机旋转矩阵].
// The sign fix makes Pi Haar distributed (R gets a positive diagonal).
// ---------------------------------------------------------------------------
extern "C" int tq_make_rotation(int d, const double* G, double* Pi) {
  TQ_TRACE("tq_make_rotation");
  if (!G || !Pi) return set_error(TQ_EINVAL, "tq_make_rotation: NULL pointer");
  if (d < 1 || d > TQ_MAX_DIM)
    return set_error(TQ_EUNSUPPORTED, "tq_make_rotation: need 1 <= d <= %d", TQ_MAX_DIM);
  const size_t n = (size_t)d;
  std::vector<double> A;  // column-major working copy: A[j*n + i] = G[i][j]
  std::vector<double> V;  // Householder vectors, column k in V[k*n ...]
  std::vector<double> beta(n), rdiag(n);
  try {
    A.resize(n * n);
    V.assign(n * n, 0.0);
  } catch (...) {
    return set_error(TQ_ENOMEM, "tq_make_rotation: out of host memory");
  }
  for (size_t i = 0; i < n; ++i)
    for (size_t j = 0; j < n; ++j) A[j * n + i] = G[i * n + j];
  for (size_t k = 0; k < n; ++k) {
    double* a = &A[k * n];
    double norm = 0.0;
    for (size_t i = k; i < n; ++i) norm += a[i] * a[i];
    norm = std::sqrt(norm);
    double alpha = (a[k] >= 0.0) ? -norm : norm;  // R_kk = alpha
    double* v = &V[k * n];
    for (size_t i = k; i < n; ++i) v[i] = a[i];
    v[k] -= alpha;
    double vv = 0.0;
    for (size_t i = k; i < n; ++i) vv += v[i] * v[i];
    beta[k] = (vv > 0.0) ? 2.0 / vv : 0.0;
    rdiag[k] = alpha;
    // apply H_k = I - beta v v^T to the remaining columns
    for (size_t j = k + 1; j < n; ++j) {
      double* c = &A[j * n];
      double s = 0.0;
      for (size_t i = k; i < n; ++i) s += v[i] * c[i];
      s *= beta[k];
      for (size_t i = k; i < n; ++i) c[i] -= s * v[i];
    }
  }
  // Q = H_0 H_1 ... H_{n-1}: apply the reflections in reverse to the identity,
  // column by column (Q stored column-major in A)
  for (size_t j = 0; j < n; ++j) {
    double* q = &A[j * n];
    for (size_t i = 0; i < n; ++i) q[i] = (i == j) ? 1.0 : 0.0;
    for (size_t kk = n; kk-- > 0;) {
      const double* v = &V[kk * n];
      double s = 0.0;
      for (size_t i = kk; i < n; ++i) s += v[i] * q[i];
      s *= beta[kk];
      for (size_t i = kk; i < n; ++i) q[i] -= s * v[i];
    }
  }
  for (size_t j = 0; j < n; ++j) {
    double sg = (rdiag[j] < 0.0) ? -1.0 : 1.0;
    for (size_t i = 0; i < n; ++i) Pi[i * n + j] = sg * A[j * n + i];
  }
  return clear_error();
}

namespace tqi {

// Law of a level-l angle of the polar tree of a uniform point on the sphere
// (l >= 2): sin^2(theta) ~ Beta(m/2, m/2) with m = 2^(l-1) coordinates on each
// side of the pair, i.e. f(theta) proportional to (sin theta cos theta)^(m-1)
// on [0, pi/2].  Cell mass and first moment by composite Gauss-Legendre in
// theta (the normalising constant cancels in the Lloyd-Max centroids).
struct AngleLaw {
  int m;
  const GaussLegendre* gl;
  void integrals(double a, double b, double* mass, double* mom) const {
    *mass = 0.0;
    *mom = 0.0;
    if (b <= a) return;
    const int pieces = std::max(1, (int)std::ceil((b - a) / 0.01));
    const double h = (b - a) / pieces;
    for (int p = 0; p < pieces; ++p) {
      const double mid = a + (p + 0.5) * h;
      for (size_t i = 0; i < gl->x.size(); ++i) {
        const double th = mid + 0.5 * h * gl->x[i];
        const double f = std::pow(0.5 * std::sin(2.0 * th), m - 1);
        *mass += 0.5 * h * gl->w[i] * f;
        *mom += 0.5 * h * gl->w[i] * f * th;
      }
    }
  }
};

}  // namespace tqi

extern "C" int tq_polar_codebook(int b, int level, double* centroids, double* thresholds) {
  TQ_TRACE("tq_polar_codebook");
  if (!centroids) return set_error(TQ_EINVAL, "tq_polar_codebook: NULL centroids");
  if (b < 1 || b > 8 || level < 1 || level > 12)
    return set_error(TQ_EUNSUPPORTED, "tq_polar_codebook: b = %d, level = %d", b, level);
  const int K = 1 << b;
  std::vector<double> c(K);
  if (level == 1) {
    // the uniform law on the circle: cells [k, k+1) 2 pi / K, centroids in the middle
    for (int k = 0; k < K; ++k) c[k] = (k + 0.5) * 2.0 * M_PI / K;
  } else {
    static const GaussLegendre gl(16);
    const AngleLaw law{1 << (level - 1), &gl};
    const double sd = 0.5 / std::sqrt((double)law.m);
    for (int k = 0; k < K; ++k) {
      const double q = K > 1 ? -2.0 + 4.0 * k / (K - 1) : 0.0;
      c[k] = std::min(M_PI / 2 - 1e-6, std::max(1e-6, M_PI / 4 + sd * q));
    }
    for (int it = 0; it < 2000; ++it) {
      double change = 0.0;
      std::vector<double> next(K);
      for (int k = 0; k < K; ++k) {
        const double lo = k == 0 ? 0.0 : 0.5 * (c[k - 1] + c[k]);
        const double hi = k == K - 1 ? M_PI / 2 : 0.5 * (c[k] + c[k + 1]);
        double mass, mom;
        law.integrals(lo, hi, &mass, &mom);
        next[k] = mass > 0.0 ? mom / mass : 0.5 * (lo + hi);
        change = std::max(change, std::fabs(next[k] - c[k]));
      }
      c = next;
      if (change < 1e-15) break;
    }
  }
  for (int k = 0; k < K; ++k) centroids[k] = c[k];
  if (thresholds)
    for (int k = 0; k + 1 < K; ++k)
      thresholds[k] = level == 1 ? (k + 1) * 2.0 * M_PI / K : 0.5 * (c[k] + c[k + 1]);
  return clear_error();
}
