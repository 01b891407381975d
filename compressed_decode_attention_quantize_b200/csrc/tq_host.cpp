// Host-side table construction for libtq, in fp64.
//
// Builds, from (d, bit widths, qjl_m, seed):
//   * Pi, the random orthogonal rotation: Householder QR of a Gaussian d x d
//     matrix G, sign-fixed so that R has a positive diagonal ("What is
//     TurboQuant?", "How TurboQuant works", stage 1 step 1);
//   * S, the m x d QJL matrix of i.i.d. N(0,1) entries rounded to fp16
//     (stage 2);
//   * the Lloyd-Max codebooks (centroids and decision boundaries) for the law
//     of one coordinate of a uniform unit vector, f(t) ~ (1 - t^2)^((d-3)/2)
//     on [-1, 1], i.e. Beta((d-1)/2, (d-1)/2) mapped to [-1, 1] (stage 1
//     steps 1-2; "How to implement" part 1: one codebook per dimension and
//     bit width).
//
// Random numbers: SplitMix64 (Steele, Lea & Flood, 2014).  Stream s of a seed
// starts from state0 = mix(seed + (s+1) * gamma) and its i-th draw (i >= 0) is
// mix(state0 + (i+1) * gamma).  A uniform is ((z >> 11) + 0.5) * 2^-53 and a
// normal is sqrt(-2 ln u1) * cos(2 pi u2) (Box-Muller, two draws each).
// Stream 0 fills G and stream 1 fills S, both row-major.
//
// The cell integrals of the Lloyd-Max iteration use the substitution
// t = sin(theta), under which f(t) dt = K cos^(d-2)(theta) dtheta, a smooth
// integrand for every d; each cell is integrated by composite Gauss-Legendre
// quadrature (nodes from Newton's method on the Legendre recurrence).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "tq_internal.h"

namespace tqh {

static constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Fills `out` with `count` N(0,1) draws of stream `stream` of `seed`.
static void stream_normals(uint64_t seed, int stream, size_t count, double* out) {
  const uint64_t state0 = mix64(seed + (uint64_t)(stream + 1) * kGamma);
  const double two_pi = 6.283185307179586476925286766559;
  for (size_t k = 0; k < count; ++k) {
    const uint64_t z1 = mix64(state0 + (uint64_t)(2 * k + 1) * kGamma);
    const uint64_t z2 = mix64(state0 + (uint64_t)(2 * k + 2) * kGamma);
    const double u1 = ((double)(z1 >> 11) + 0.5) * 0x1.0p-53;
    const double u2 = ((double)(z2 >> 11) + 0.5) * 0x1.0p-53;
    out[k] = std::sqrt(-2.0 * std::log(u1)) * std::cos(two_pi * u2);
  }
}

// Nearest fp16 value of x (ties to even), returned as a double.
double round_to_half(double x) {
  if (x == 0.0 || !std::isfinite(x)) return x;
  const double ax = std::fabs(x);
  if (ax >= 65520.0) return std::copysign(INFINITY, x);
  int e = 0;
  std::frexp(ax, &e);                       // ax in [2^(e-1), 2^e)
  const int qexp = std::max(e - 11, -24);   // 11 significant bits; subnormal quantum 2^-24
  const double q = std::ldexp(1.0, qexp);
  return std::copysign(std::nearbyint(ax / q) * q, x);
}

// Householder QR of the row-major d x d matrix A; returns Q (row-major) and
// the diagonal of R.
static void householder_qr(int d, const std::vector<double>& A_in,
                           std::vector<double>& Q, std::vector<double>& rdiag) {
  std::vector<double> A(A_in);
  std::vector<std::vector<double>> vs(d);
  std::vector<double> betas(d, 0.0);
  rdiag.assign(d, 0.0);
  for (int k = 0; k < d; ++k) {
    double norm2 = 0.0;
    for (int i = k; i < d; ++i) norm2 += A[i * d + k] * A[i * d + k];
    const double norm = std::sqrt(norm2);
    const double x0 = A[k * d + k];
    const double alpha = (x0 >= 0.0) ? -norm : norm;   // R_kk after reflection
    std::vector<double> v(d - k);
    for (int i = k; i < d; ++i) v[i - k] = A[i * d + k];
    v[0] -= alpha;
    double vnorm2 = 0.0;
    for (double t : v) vnorm2 += t * t;
    const double beta = vnorm2 > 0.0 ? 2.0 / vnorm2 : 0.0;
    // A <- (I - beta v v^T) A on rows k.., columns k..
    for (int j = k; j < d; ++j) {
      double dot = 0.0;
      for (int i = k; i < d; ++i) dot += v[i - k] * A[i * d + j];
      dot *= beta;
      for (int i = k; i < d; ++i) A[i * d + j] -= dot * v[i - k];
    }
    rdiag[k] = A[k * d + k];
    vs[k] = std::move(v);
    betas[k] = beta;
  }
  // Q = H_0 H_1 ... H_{d-1}: apply the reflections to I from the right end.
  Q.assign((size_t)d * d, 0.0);
  for (int i = 0; i < d; ++i) Q[i * d + i] = 1.0;
  for (int k = d - 1; k >= 0; --k) {
    const std::vector<double>& v = vs[k];
    const double beta = betas[k];
    if (beta == 0.0) continue;
    for (int j = 0; j < d; ++j) {
      double dot = 0.0;
      for (int i = k; i < d; ++i) dot += v[i - k] * Q[i * d + j];
      dot *= beta;
      for (int i = k; i < d; ++i) Q[i * d + j] -= dot * v[i - k];
    }
  }
}

void rotation(int d, uint64_t seed, std::vector<double>& Pi) {
  std::vector<double> G((size_t)d * d);
  stream_normals(seed, 0, G.size(), G.data());
  std::vector<double> Q, rdiag;
  householder_qr(d, G, Q, rdiag);
  Pi.resize((size_t)d * d);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j)
      Pi[i * d + j] = Q[i * d + j] * (rdiag[j] >= 0.0 ? 1.0 : -1.0);
}

void qjl_matrix(int m, int d, uint64_t seed, std::vector<double>& S) {
  S.resize((size_t)m * d);
  if (m == 0) return;
  stream_normals(seed, 1, S.size(), S.data());
  for (double& s : S) s = round_to_half(s);
}

// Gauss-Legendre nodes/weights on [-1, 1].
static void gauss_legendre(int n, std::vector<double>& x, std::vector<double>& w) {
  x.resize(n);
  w.resize(n);
  const double pi = 3.14159265358979323846264338327950288;
  for (int i = 0; i < n; ++i) {
    double z = std::cos(pi * (i + 0.75) / (n + 0.5));
    double dp = 0.0;
    for (int it = 0; it < 100; ++it) {
      double p0 = 1.0, p1 = z;
      for (int k = 2; k <= n; ++k) {
        const double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
        p0 = p1;
        p1 = p2;
      }
      dp = n * (z * p1 - p0) / (z * z - 1.0);
      const double dz = p1 / dp;
      z -= dz;
      if (std::fabs(dz) < 1e-17) break;
    }
    double p0 = 1.0, p1 = z;
    for (int k = 2; k <= n; ++k) {
      const double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
      p0 = p1;
      p1 = p2;
    }
    dp = n * (z * p1 - p0) / (z * z - 1.0);
    x[i] = z;
    w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
  }
}

// Integrals over theta in [a, b] of cos^(d-2)(theta) (mass, up to K) and
// sin(theta) cos^(d-2)(theta) (first moment, up to K).
static void cell_integrals(int d, double a, double b, const std::vector<double>& gx,
                           const std::vector<double>& gw, int panels, double* mass,
                           double* moment) {
  double m0 = 0.0, m1 = 0.0;
  const double h = (b - a) / panels;
  for (int p = 0; p < panels; ++p) {
    const double lo = a + p * h;
    const double mid = lo + 0.5 * h;
    for (size_t i = 0; i < gx.size(); ++i) {
      const double th = mid + 0.5 * h * gx[i];
      const double c = std::cos(th);
      const double wt = 0.5 * h * gw[i] * (c > 0.0 ? std::pow(c, d - 2) : 0.0);
      m0 += wt;
      m1 += wt * std::sin(th);
    }
  }
  *mass = m0;
  *moment = m1;
}

// One Lloyd-Max step on the upper-half centroids c (boundary 0 in the
// middle): edges at the midpoints, each centroid the mean of its cell.  Also
// returns the cells' (unnormalised) masses and edges.  Panels of at most 0.02
// rad in theta = asin t keep the 24-point rule exact to rounding for every
// supported d.
static void lloyd_step(int d, const std::vector<double>& c, const std::vector<double>& gx,
                       const std::vector<double>& gw, std::vector<double>& u, std::vector<double>& mass,
                       std::vector<double>& edge) {
  const int half = (int)c.size();
  edge.resize(half + 1);
  edge[0] = 0.0;
  for (int i = 1; i < half; ++i) edge[i] = 0.5 * (c[i - 1] + c[i]);
  edge[half] = 1.0;
  u.resize(half);
  mass.resize(half);
  for (int i = 0; i < half; ++i) {
    const double a = std::asin(edge[i]), b = std::asin(edge[i + 1]);
    const int panels = std::max(1, (int)std::ceil((b - a) / 0.02));
    double m0, m1;
    cell_integrals(d, a, b, gx, gw, panels, &m0, &m1);
    u[i] = m1 / m0;
    mass[i] = m0;
  }
}

// Lloyd-Max centroids (2^bits, increasing) and interior boundaries for f_d.
// The plain alternation of the two optimality conditions converges slowly
// with many levels (8 bits), so once its steps fall below 1e-7 (or after 4000
// of them) Newton steps on c - U(c) finish the same fixed point: U_i depends
// on c_{i-1}, c_i, c_{i+1} through the two midpoints, with
// dU_i/dhi = f(hi) (hi - U_i) / P_i and dU_i/dlo = f(lo) (U_i - lo) / P_i, so
// each step is a tridiagonal solve.  Newton stops at 1e-15 or, after eight
// steps, below 1e-12 (the rounding floor of the cell masses).
static void lloyd_max_solve(int d, int bits, std::vector<double>& cen, std::vector<double>& bnd) {
  const int L = 1 << bits, half = L / 2;
  std::vector<double> gx, gw;
  gauss_legendre(24, gx, gw);
  std::vector<double> c(half), u, mass, edge;
  for (int i = 0; i < half; ++i) c[i] = (i + 0.5) / half * 3.0 / std::sqrt((double)d);
  double delta = 1.0;
  for (int it = 0; it < 4000; ++it) {
    lloyd_step(d, c, gx, gw, u, mass, edge);
    delta = 0.0;
    for (int i = 0; i < half; ++i) delta = std::max(delta, std::fabs(u[i] - c[i]));
    c = u;
    if (delta < 1e-15 || (delta < 1e-7 && half > 1)) break;
  }
  const double ex = 0.5 * (d - 3);
  auto dens = [&](double t) { return t >= 1.0 ? 0.0 : std::pow(1.0 - t * t, ex); };
  std::vector<double> lo(half), di(half), up(half), r(half), step(half), cand(half);
  for (int newton = 1; delta >= 1e-15 && half > 1 && newton <= 200; ++newton) {
    lloyd_step(d, c, gx, gw, u, mass, edge);
    for (int i = 0; i < half; ++i) {
      const double dh = i + 1 < half ? dens(edge[i + 1]) * (edge[i + 1] - u[i]) / mass[i] : 0.0;
      const double dl = i > 0 ? dens(edge[i]) * (u[i] - edge[i]) / mass[i] : 0.0;
      lo[i] = -0.5 * dl;              // (I - J)_{i,i-1}
      up[i] = -0.5 * dh;              // (I - J)_{i,i+1}
      di[i] = 1.0 - 0.5 * (dl + dh);
      r[i] = u[i] - c[i];
    }
    // Thomas algorithm for (I - J) step = r.
    for (int i = 1; i < half; ++i) {
      const double w = lo[i] / di[i - 1];
      di[i] -= w * up[i - 1];
      r[i] -= w * r[i - 1];
    }
    step[half - 1] = r[half - 1] / di[half - 1];
    for (int i = half - 2; i >= 0; --i) step[i] = (r[i] - up[i] * step[i + 1]) / di[i];
    double scale = 1.0;
    for (int tries = 0; tries < 60; ++tries, scale *= 0.5) {   // keep the centroids increasing in (0, 1)
      bool ok = true;
      for (int i = 0; i < half; ++i) {
        cand[i] = c[i] + scale * step[i];
        if (cand[i] <= (i ? cand[i - 1] : 0.0) || cand[i] >= 1.0) ok = false;
      }
      if (ok) break;
    }
    delta = 0.0;
    for (int i = 0; i < half; ++i) delta = std::max(delta, std::fabs(cand[i] - c[i]));
    c = cand;
    if (newton >= 8 && delta < 1e-12) break;
  }
  cen.resize(L);
  for (int i = 0; i < half; ++i) {
    cen[half + i] = c[i];
    cen[half - 1 - i] = -c[i];
  }
  bnd.resize(L - 1);
  for (int i = 0; i + 1 < L; ++i) bnd[i] = 0.5 * (cen[i] + cen[i + 1]);
  bnd[half - 1] = 0.0;
}

// Codebooks depend only on (d, bits); solve each once per process.
void lloyd_max(int d, int bits, std::vector<double>& cen, std::vector<double>& bnd) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, std::pair<std::vector<double>, std::vector<double>>> cache;
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find({d, bits});
    if (it != cache.end()) {
      cen = it->second.first;
      bnd = it->second.second;
      return;
    }
  }
  lloyd_max_solve(d, bits, cen, bnd);
  std::lock_guard<std::mutex> lk(mu);
  cache[{d, bits}] = {cen, bnd};
}

}  // namespace tqh
