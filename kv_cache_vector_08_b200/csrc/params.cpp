// Host-side parameter generation for a TurboQuant context, in float64.
//
// turboquant.net, "伪代码实现步骤": the rotation is the Q factor of a seeded Gaussian
// d x d matrix ("生成随机旋转矩阵") and the codebook is a Lloyd-Max quantizer of the
// Beta-type coordinate density, computed once offline ("预计算 Lloyd-Max 质心",
// "PolarQuant：极坐标变换 / 坐标分布公式").  The QJL matrix S is Gaussian with m = d rows
// (admirer.cn article, QJL paragraph).  The random stream is SplitMix64 (Steele, Lea,
// Flood 2014) with Box-Muller, so any implementation of those published definitions
// draws the same matrices from the same seed.
#include "params.h"

#include <algorithm>
#include <cmath>
#include <cstring>

namespace tq {

namespace {
constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
}  // namespace

void splitmix64(uint64_t seed, uint64_t start, uint64_t count, uint64_t* out) {
  for (uint64_t i = 0; i < count; ++i) out[i] = mix64(seed + (start + i + 1) * kGolden);
}

void gaussian_stream(uint64_t seed, uint64_t count, double* out) {
  const double two_pi = 6.283185307179586476925286766559;
  uint64_t pairs = (count + 1) / 2;
  for (uint64_t j = 0; j < pairs; ++j) {
    uint64_t w[2];
    splitmix64(seed, 2 * j, 2, w);
    double u1 = (double)((w[0] >> 11) + 1) * 0x1.0p-53;
    double u2 = (double)((w[1] >> 11) + 1) * 0x1.0p-53;
    double rad = std::sqrt(-2.0 * std::log(u1));
    double ang = two_pi * u2;
    out[2 * j] = rad * std::cos(ang);
    if (2 * j + 1 < count) out[2 * j + 1] = rad * std::sin(ang);
  }
}

// Householder QR of G (row-major d x d).  Works on a column-major copy so that every
// reflector update runs down contiguous columns.  Q is accumulated backwards
// (Q = H_0 H_1 ... H_{d-1} applied to I from the last reflector), then its columns are
// multiplied by sign(R_jj) so that R has a positive diagonal.
void haar_rotation(int d, const double* G, double* Pi) {
  const size_t n = (size_t)d;
  std::vector<double> A(n * n), Q(n * n, 0.0), V(n * n, 0.0), beta(n, 0.0), rdiag(n, 0.0);
  for (size_t i = 0; i < n; ++i)
    for (size_t j = 0; j < n; ++j) A[j * n + i] = G[i * n + j];
  for (size_t j = 0; j < n; ++j) {
    double* a = &A[j * n];
    double nrm2 = 0.0;
    for (size_t i = j; i < n; ++i) nrm2 += a[i] * a[i];
    double nrm = std::sqrt(nrm2);
    double* v = &V[j * n];
    if (nrm == 0.0) {  // zero column: no reflection
      beta[j] = 0.0;
      rdiag[j] = 0.0;
      continue;
    }
    double alpha = a[j] >= 0.0 ? -nrm : nrm;
    for (size_t i = j; i < n; ++i) v[i] = a[i];
    v[j] -= alpha;
    double vv = 0.0;
    for (size_t i = j; i < n; ++i) vv += v[i] * v[i];
    beta[j] = vv > 0.0 ? 2.0 / vv : 0.0;
    rdiag[j] = alpha;
    const double bj = beta[j];
#pragma omp parallel for schedule(static) if (n - j > 128)
    for (long long c = (long long)j + 1; c < (long long)n; ++c) {
      double* col = &A[(size_t)c * n];
      double s = 0.0;
      for (size_t i = j; i < n; ++i) s += v[i] * col[i];
      s *= bj;
      for (size_t i = j; i < n; ++i) col[i] -= s * v[i];
    }
  }
  for (size_t i = 0; i < n; ++i) Q[i * n + i] = 1.0;
  for (long long jj = (long long)n - 1; jj >= 0; --jj) {
    const size_t j = (size_t)jj;
    const double* v = &V[j * n];
    const double bj = beta[j];
    if (bj == 0.0) continue;
#pragma omp parallel for schedule(static) if (n - j > 128)
    for (long long c = (long long)j; c < (long long)n; ++c) {
      double* col = &Q[(size_t)c * n];
      double s = 0.0;
      for (size_t i = j; i < n; ++i) s += v[i] * col[i];
      s *= bj;
      for (size_t i = j; i < n; ++i) col[i] -= s * v[i];
    }
  }
  for (size_t j = 0; j < n; ++j) {
    double sgn = rdiag[j] < 0.0 ? -1.0 : 1.0;
    for (size_t i = 0; i < n; ++i) Pi[i * n + j] = Q[j * n + i] * sgn;
  }
}

namespace {
// Continued fraction of I_x(a, b) (DLMF 8.17.22), evaluated by the modified Lentz method;
// valid for x < (a+1)/(a+b+2).  y = 1 - x is passed separately to keep log(1-x) accurate.
double ibeta_cf(double a, double b, double x, double y) {
  const double tiny = 1e-300, eps = 1e-16;
  double f = 1.0, C = 1.0, D = 0.0;
  for (int n = 1; n < 100000; ++n) {
    int m = n / 2;
    double dn;
    if (n & 1)
      dn = -(a + m) * (a + b + m) * x / ((a + 2 * m) * (a + 2 * m + 1));
    else
      dn = m * (b - m) * x / ((a + 2 * m - 1) * (a + 2 * m));
    D = 1.0 + dn * D;
    if (std::fabs(D) < tiny) D = tiny;
    C = 1.0 + dn / C;
    if (std::fabs(C) < tiny) C = tiny;
    D = 1.0 / D;
    double delta = C * D;
    f *= delta;
    if (std::fabs(delta - 1.0) < eps) break;
  }
  double lbeta = std::lgamma(a) + std::lgamma(b) - std::lgamma(a + b);
  double logpre = a * std::log(x) + b * std::log(y) - std::log(a) - lbeta;
  return std::exp(logpre) / f;
}

double ibeta_xy(double a, double b, double x, double y) {
  if (x <= 0.0) return 0.0;
  if (y <= 0.0) return 1.0;
  if (x < (a + 1.0) / (a + b + 2.0)) return ibeta_cf(a, b, x, y);
  return 1.0 - ibeta_cf(b, a, y, x);
}

// P(X > x) for x >= 0 with X ~ f_d:  X^2 ~ Beta(1/2, (d-1)/2), so
// P(X > x) = P(X^2 > x^2)/2 = I_{1-x^2}((d-1)/2, 1/2) / 2.
double upper_tail(double x, int d) {
  if (x <= 0.0) return 0.5;
  if (x >= 1.0) return 0.0;
  return 0.5 * ibeta_xy(0.5 * (d - 1), 0.5, 1.0 - x * x, x * x);
}

double mass(double a, double b, int d) {
  if (a >= 0.0) return upper_tail(a, d) - upper_tail(b, d);
  if (b <= 0.0) return upper_tail(-b, d) - upper_tail(-a, d);
  return 1.0 - upper_tail(-a, d) - upper_tail(b, d);
}

// int_a^b x f_d(x) dx = C_d/(d-1) [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)]
double first_moment(double a, double b, int d) {
  auto g = [d](double t) {
    if (std::fabs(t) >= 1.0) return 0.0;
    return std::exp(0.5 * (d - 1) * std::log1p(-t * t));
  };
  double logc = std::lgamma(0.5 * d) - std::lgamma(0.5 * (d - 1)) - 0.5 * std::log(M_PI);
  return std::exp(logc) / (d - 1) * (g(a) - g(b));
}

double cdf(double x, int d) { return x <= 0.0 ? upper_tail(-x, d) : 1.0 - upper_tail(x, d); }
}  // namespace

double incomplete_beta(double a, double b, double x) { return ibeta_xy(a, b, x, 1.0 - x); }

void lloyd_max_beta(int d, int levels, double* centroids, double* boundaries) {
  const int K = levels;
  std::vector<double> t(K + 1), c(K), cn(K);
  t[0] = -1.0;
  t[K] = 1.0;
  for (int j = 1; j < K; ++j) {  // equal-probability start, by bisection on the CDF
    double p = (double)j / K, lo = -1.0, hi = 1.0;
    for (int it = 0; it < 200; ++it) {
      double mid = 0.5 * (lo + hi);
      if (cdf(mid, d) < p) lo = mid; else hi = mid;
    }
    t[j] = 0.5 * (lo + hi);
  }
  for (int j = 0; j < K; ++j) c[j] = first_moment(t[j], t[j + 1], d) / mass(t[j], t[j + 1], d);
  for (int it = 0; it < 200000; ++it) {
    for (int j = 1; j < K; ++j) t[j] = 0.5 * (c[j - 1] + c[j]);
    double delta = 0.0;
    for (int j = 0; j < K; ++j) {
      cn[j] = first_moment(t[j], t[j + 1], d) / mass(t[j], t[j + 1], d);
      delta = std::max(delta, std::fabs(cn[j] - c[j]));
    }
    c.swap(cn);
    if (delta <= 1e-15) break;
  }
  // f_d is even: the exact quantizer is odd-symmetric, so make the computed one exactly so
  for (int j = 0; j < K; ++j) cn[j] = 0.5 * (c[j] - c[K - 1 - j]);
  for (int j = 0; j < K; ++j) centroids[j] = cn[j];
  for (int j = 0; j + 1 < K; ++j) boundaries[j] = 0.5 * (cn[j] + cn[j + 1]);
}

bool build_params(int d, int bits, uint64_t seed, int mode, HostParams* p) {
  if (d < 3 || d > 4096) return false;
  int k = mode == 0 ? bits - 1 : bits;
  if (mode != 0 && mode != 1) return false;
  if (mode == 0 && (bits < 2 || bits > 5)) return false;
  if (mode == 1 && (bits < 1 || bits > 4)) return false;
  p->d = d;
  p->bits = bits;
  p->k = k;
  p->mode = mode;
  p->m = mode == 0 ? d : 0;
  p->seed = seed;
  const size_t n = (size_t)d;
  std::vector<double> g(2 * n * n);
  gaussian_stream(seed, 2 * n * n, g.data());
  p->Pi.assign(n * n, 0.0);
  haar_rotation(d, g.data(), p->Pi.data());
  if (mode == 0) {
    p->S.assign(g.begin() + n * n, g.end());
    p->M.assign(n * n, 0.0);
    // M = S Pi^T:  M[j][i] = sum_l S[j][l] Pi[i][l]
#pragma omp parallel for schedule(static) if (n > 128)
    for (long long j = 0; j < (long long)n; ++j)
      for (size_t i = 0; i < n; ++i) {
        const double* s = &p->S[(size_t)j * n];
        const double* r = &p->Pi[i * n];
        double acc = 0.0;
        for (size_t l = 0; l < n; ++l) acc += s[l] * r[l];
        p->M[(size_t)j * n + i] = acc;
      }
  } else {
    p->S.clear();
    p->M.clear();
  }
  const int K = 1 << k;
  p->centroids.assign(K, 0.0);
  p->boundaries.assign(K - 1, 0.0);
  lloyd_max_beta(d, K, p->centroids.data(), p->boundaries.data());
  return true;
}

}  // namespace tq
