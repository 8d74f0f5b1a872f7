// Polar Express coefficients for the Newton-Schulz steps of Muon, computed on
// the host in double precision.
//
// "¿Cómo Entrenar Tu Propio ChatGPT por $50?", section "2. Optimizador Muon",
// prints the first two (a, b, c) tuples of a five-step table and elides the
// rest.  The table is the output of the Polar Express construction (Amsel,
// Persson, Musco and Gower, 2025): step t takes the odd quintic
// p(x) = a x + b x^3 + c x^5 that best approximates 1 in max-norm on
// [max(l, cushion * u), u], rescales it so that 1 - p(l) = p(u) - 1, divides
// its argument by a safety factor (p(x) -> p(x / s)), and passes on the image
// interval [p(l), 2 - p(l)].  With l0 = 1e-3, cushion 0.02 and safety 1.02
// the first two tuples agree with the printed ones to their three decimals.
#include "polar_express_table.h"

#include <math.h>

#include <mutex>

namespace gpt {

namespace {

// Solve the 4x4 system m x = rhs by Gaussian elimination with partial pivoting.
bool solve4(double m[4][4], double rhs[4], double x[4]) {
  int piv[4] = {0, 1, 2, 3};
  for (int col = 0; col < 4; ++col) {
    int best = col;
    for (int r = col + 1; r < 4; ++r)
      if (fabs(m[piv[r]][col]) > fabs(m[piv[best]][col])) best = r;
    const int tmp = piv[col];
    piv[col] = piv[best];
    piv[best] = tmp;
    const double p = m[piv[col]][col];
    if (p == 0.0) return false;
    for (int r = col + 1; r < 4; ++r) {
      const double f = m[piv[r]][col] / p;
      for (int cc = col; cc < 4; ++cc) m[piv[r]][cc] -= f * m[piv[col]][cc];
      rhs[piv[r]] -= f * rhs[piv[col]];
    }
  }
  for (int col = 3; col >= 0; --col) {
    double s = rhs[piv[col]];
    for (int cc = col + 1; cc < 4; ++cc) s -= m[piv[col]][cc] * x[cc];
    x[col] = s / m[piv[col]][col];
  }
  return true;
}

// Remez exchange for the equioscillating odd quintic on [lo, hi]:
// p(lo) = 1 - E, p(q) = 1 + E, p(r) = 1 - E, p(hi) = 1 + E at the interior extrema q < r.
void best_quintic(double lo, double hi, double coef[3]) {
  double q = lo + 0.3 * (hi - lo), r = lo + 0.7 * (hi - lo);
  double sol[4] = {0, 0, 0, 0};
  for (int it = 0; it < 200; ++it) {
    const double pts[4] = {lo, q, r, hi};
    const double sgn[4] = {1.0, -1.0, 1.0, -1.0};
    double m[4][4], rhs[4];
    for (int i = 0; i < 4; ++i) {
      const double x = pts[i];
      m[i][0] = x;
      m[i][1] = x * x * x;
      m[i][2] = x * x * x * x * x;
      m[i][3] = sgn[i];
      rhs[i] = 1.0;
    }
    if (!solve4(m, rhs, sol)) break;
    const double a = sol[0], b = sol[1], c = sol[2];
    // p'(x) = a + 3 b x^2 + 5 c x^4 = 0, a quadratic in x^2
    const double disc = 9.0 * b * b - 20.0 * a * c;
    if (disc < 0.0 || c == 0.0) break;
    double y1 = (-3.0 * b - sqrt(disc)) / (10.0 * c);
    double y2 = (-3.0 * b + sqrt(disc)) / (10.0 * c);
    if (y1 <= 0.0 || y2 <= 0.0) break;
    double nq = sqrt(y1), nr = sqrt(y2);
    if (nq > nr) {
      const double t = nq;
      nq = nr;
      nr = t;
    }
    const bool done = fabs(nq - q) < 1e-16 && fabs(nr - r) < 1e-16;
    q = nq;
    r = nr;
    if (done) break;
  }
  coef[0] = sol[0];
  coef[1] = sol[1];
  coef[2] = sol[2];
}

double poly(const double c[3], double x) { return c[0] * x + c[1] * x * x * x + c[2] * x * x * x * x * x; }

double g_table[kPolarSteps][3];

}  // namespace

const double (*polar_coefficients())[3] {
  static std::once_flag once;
  std::call_once(once, [] {
    const double l0 = 1e-3, cushion = 0.02, safety = 1.02;
    double lo = l0, hi = 1.0;
    for (int t = 0; t < kPolarSteps; ++t) {
      double c[3];
      best_quintic(lo > cushion * hi ? lo : cushion * hi, hi, c);
      const double centre = 2.0 / (poly(c, lo) + poly(c, hi));
      for (double& v : c) v *= centre;
      c[0] /= safety;
      c[1] /= safety * safety * safety;
      c[2] /= safety * safety * safety * safety * safety;
      for (int i = 0; i < 3; ++i) g_table[t][i] = c[i];
      lo = poly(c, lo);
      hi = 2.0 - lo;
    }
  });
  return g_table;
}

}  // namespace gpt
