// Polar Express coefficient schedule (host code).
//
// Amsel, Persson, Musco and Gower, "The Polar Express: Optimal Matrix Sign
// Methods and Their Application to the Muon Algorithm" (2025), build the
// per-step polynomials of a Newton-Schulz-type iteration greedily: if after
// t steps every singular value of the normalized input lies in [lo_t, hi_t],
// step t applies the odd quintic p_t(x) = a x + b x^3 + c x^5 that minimizes
//   max_{x in [lo_t, hi_t]} |1 - p_t(x)|,
// and the singular values then lie in the image of [lo_t, hi_t] under p_t.
// The first interval is [lower, 1] (Frobenius normalization puts every
// singular value at or below 1; `lower` bounds the smallest one).
//
// Once the interval is narrower than 1e-3 the 4 x 4 Remez system loses its
// conditioning; the minimax quintic there tends to the one with p(1) = 1,
// p'(1) = p''(1) = 0, i.e. (15/8, -5/4, 3/8), whose error on [1 - d, 1 + d]
// is below 3 d^3 (< 1e-8), so that polynomial is used instead.
//
// The minimax quintic equioscillates: 1 - p takes the values +E, -E, +E, -E
// at lo, at the two interior critical points of p and at hi.  Remez
// exchange finds it: solve the 4 x 4 system for (a, b, c, E) on the current
// points, move the interior points to the roots of p'(x) = a + 3 b x^2 +
// 5 c x^4, repeat until they stop moving.
//
// `safety` >= 1 applies p_t(x / safety) instead of p_t (coefficients a/s,
// b/s^3, c/s^5), which keeps a value slightly above the tracked interval
// (rounding) from being amplified; the tracked interval is then the image
// under the polynomial actually applied.
#pragma once
#include <cmath>
#include <algorithm>

namespace muon {
namespace polar_express {

struct Quintic {
  double a, b, c;
  double eval(double x) const {
    const double x2 = x * x;
    return x * (a + x2 * (b + x2 * c));
  }
};

// Solves the 4 x 4 system M z = r by Gaussian elimination with partial pivoting.
inline bool solve4(double M[4][4], double r[4], double z[4]) {
  for (int col = 0; col < 4; ++col) {
    int piv = col;
    for (int i = col + 1; i < 4; ++i)
      if (std::fabs(M[i][col]) > std::fabs(M[piv][col])) piv = i;
    if (M[piv][col] == 0.0) return false;
    if (piv != col) {
      for (int j = 0; j < 4; ++j) std::swap(M[col][j], M[piv][j]);
      std::swap(r[col], r[piv]);
    }
    for (int i = col + 1; i < 4; ++i) {
      const double f = M[i][col] / M[col][col];
      for (int j = col; j < 4; ++j) M[i][j] -= f * M[col][j];
      r[i] -= f * r[col];
    }
  }
  for (int i = 3; i >= 0; --i) {
    double s = r[i];
    for (int j = i + 1; j < 4; ++j) s -= M[i][j] * z[j];
    z[i] = s / M[i][i];
  }
  return true;
}

// Roots x in (lo, hi) of p'(x) = a + 3 b x^2 + 5 c x^4, ascending; returns their count.
inline int critical_points(const Quintic& p, double lo, double hi, double out[2]) {
  int n = 0;
  const double A = 5.0 * p.c, B = 3.0 * p.b, C = p.a;   // A y^2 + B y + C = 0, y = x^2
  double ys[2];
  int ny = 0;
  if (A == 0.0) {
    if (B != 0.0) ys[ny++] = -C / B;
  } else {
    const double disc = B * B - 4.0 * A * C;
    if (disc >= 0.0) {
      const double sq = std::sqrt(disc);
      // Numerically stable pair of roots.
      const double q = -0.5 * (B + (B >= 0.0 ? sq : -sq));
      if (q != 0.0) ys[ny++] = C / q;
      ys[ny++] = q / A;
    }
  }
  for (int i = 0; i < ny; ++i) {
    if (!(ys[i] > 0.0)) continue;
    const double x = std::sqrt(ys[i]);
    if (x > lo && x < hi) out[n++] = x;
  }
  if (n == 2 && out[0] > out[1]) std::swap(out[0], out[1]);
  return n;
}

// The odd quintic minimizing max |1 - p| on [lo, hi] (0 < lo < hi) and that maximum E.
inline bool minimax_quintic(double lo, double hi, Quintic* best, double* E_out) {
  const double pi = 3.14159265358979323846;
  if (hi - lo < 1e-3) {
    *best = Quintic{15.0 / 8.0, -10.0 / 8.0, 3.0 / 8.0};
    double mn = 0.0, mx = 0.0;
    const double cps[2] = {lo, hi};
    mn = std::min(best->eval(cps[0]), best->eval(cps[1]));
    mx = std::max(best->eval(cps[0]), best->eval(cps[1]));
    *E_out = std::max(std::fabs(1.0 - mn), std::fabs(mx - 1.0));
    return true;
  }
  double x[4];
  for (int i = 0; i < 4; ++i) x[i] = 0.5 * (lo + hi) - 0.5 * (hi - lo) * std::cos(pi * i / 3.0);
  Quintic p{0.0, 0.0, 0.0};
  double E = 0.0;
  for (int iter = 0; iter < 200; ++iter) {
    double M[4][4], r[4], z[4];
    for (int i = 0; i < 4; ++i) {
      const double x2 = x[i] * x[i];
      M[i][0] = x[i];
      M[i][1] = x[i] * x2;
      M[i][2] = x[i] * x2 * x2;
      M[i][3] = (i % 2 == 0) ? 1.0 : -1.0;   // p(x_i) + (+-E) = 1  <=>  1 - p(x_i) = +-E
      r[i] = 1.0;
    }
    if (!solve4(M, r, z)) return false;
    p = Quintic{z[0], z[1], z[2]};
    E = z[3];
    double cp[2];
    if (critical_points(p, lo, hi, cp) != 2) break;    // the exchange has converged or cannot proceed
    const double moved = std::max(std::fabs(cp[0] - x[1]), std::fabs(cp[1] - x[2]));
    x[1] = cp[0];
    x[2] = cp[1];
    if (moved <= 1e-15 * hi) break;
  }
  if (!std::isfinite(p.a) || !std::isfinite(p.b) || !std::isfinite(p.c) || !std::isfinite(E)) return false;
  *best = p;
  *E_out = std::fabs(E);
  return true;
}

// Minimum and maximum of p over [lo, hi].
inline void image(const Quintic& p, double lo, double hi, double* mn, double* mx) {
  double vals[4] = {p.eval(lo), p.eval(hi), 0.0, 0.0};
  int n = 2;
  double cp[2];
  const int k = critical_points(p, lo, hi, cp);
  for (int i = 0; i < k; ++i) vals[n++] = p.eval(cp[i]);
  *mn = *std::min_element(vals, vals + n);
  *mx = *std::max_element(vals, vals + n);
}

}  // namespace polar_express
}  // namespace muon
