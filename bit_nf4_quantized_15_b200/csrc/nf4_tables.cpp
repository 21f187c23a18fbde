// NF4 codebook and decision thresholds, derived on the host at first use.
//
// nlp-lineage "QLoRA" milestone page, section "The idea", NF4 bullet: 16
// values placed so that each covers an equal share of the normal
// distribution, with an exact zero.  Construction: 8 positive levels at the
// standard-normal quantiles of 8 equally spaced probabilities from
// delta = 1 - (1/32 + 1/30)/2 down towards 1/2, 7 negative levels mirrored
// from 7 equally spaced probabilities over the same range, plus 0, all
// divided by the largest level so that the endpoints are exactly -1 and +1.
//
// The quantile is computed here by Newton's method on Phi(x) = erfc(-x/sqrt2)/2
// in extended precision; the result is rounded to fp32.
#include <atomic>
#include <cmath>
#include <mutex>
#include <utility>

#include "internal.h"

namespace qnf4 {
namespace {

long double phi_cdf(long double x) { return 0.5L * std::erfc(-x / std::sqrt(2.0L)); }
long double phi_pdf(long double x) {
  return std::exp(-0.5L * x * x) / std::sqrt(2.0L * 3.14159265358979323846264338327950288L);
}

long double quantile(long double p) {
  long double x = 0.0L;
  for (int it = 0; it < 200; ++it) {
    const long double step = (phi_cdf(x) - p) / phi_pdf(x);
    x -= step;
    if (std::fabs(step) < 1e-19L * (1.0L + std::fabs(x))) break;
  }
  return x;
}

// Largest float <= v.
float round_down_to_float(double v) {
  float f = (float)v;
  if ((double)f > v) f = std::nextafterf(f, -INFINITY);
  return f;
}

// f(x) evaluated the way the kernel does it: Horner in fp32 with fused
// multiply-adds (poly[0] holds c0 - 1/2).
float eval_poly_f32(const float* p, float x) {
  float f = p[5];
  for (int k = 4; k >= 0; --k) f = std::fmaf(f, x, p[k]);
  return f + 0.5f;
}

// Least-squares fit of f through (t[i], i + 1/2) and the anchors (-1, 0.3),
// (1, 14.7), then a check of the conditions the quantiser relies on.
void fit_code_polynomial(Nf4Tables& t) {
  double xs[17], ys[17];
  for (int i = 0; i < 15; ++i) {
    xs[i] = t.t[i];
    ys[i] = i + 0.5;
  }
  xs[15] = -1.0, ys[15] = 0.3;
  xs[16] = 1.0, ys[16] = 14.7;
  double A[6][7] = {};
  for (int n = 0; n < 17; ++n) {
    double pw[6];
    pw[0] = 1.0;
    for (int k = 1; k < 6; ++k) pw[k] = pw[k - 1] * xs[n];
    for (int r = 0; r < 6; ++r) {
      for (int c = 0; c < 6; ++c) A[r][c] += pw[r] * pw[c];
      A[r][6] += pw[r] * ys[n];
    }
  }
  for (int c = 0; c < 6; ++c) {  // Gauss-Jordan with partial pivoting
    int piv = c;
    for (int r = c + 1; r < 6; ++r)
      if (std::fabs(A[r][c]) > std::fabs(A[piv][c])) piv = r;
    for (int k = 0; k < 7; ++k) std::swap(A[c][k], A[piv][k]);
    for (int r = 0; r < 6; ++r) {
      if (r == c) continue;
      const double m = A[r][c] / A[c][c];
      for (int k = c; k < 7; ++k) A[r][k] -= m * A[c][k];
    }
  }
  for (int k = 0; k < 6; ++k) t.poly[k] = (float)(A[k][6] / A[k][k]);
  t.poly[0] = (float)((double)t.poly[0] - 0.5);
  bool ok = eval_poly_f32(t.poly, -1.0f) >= 0.1f && eval_poly_f32(t.poly, 1.0f) <= 14.9f;
  for (int i = 0; i < 15; ++i) {
    const float f = eval_poly_f32(t.poly, t.t[i]);
    ok = ok && f >= i + 0.1f && f <= i + 0.9f;
  }
  float prev = eval_poly_f32(t.poly, -1.0f);
  for (int n = 1; n <= 1 << 16 && ok; ++n) {  // increasing on a fine grid of [-1, 1]
    const float f = eval_poly_f32(t.poly, -1.0f + 2.0f * (float)n / (float)(1 << 16));
    ok = f > prev;
    prev = f;
  }
  t.poly_ok = ok;
}

Nf4Tables build() {
  const long double delta = 1.0L - 0.5L * (1.0L / 32.0L + 1.0L / 30.0L);
  long double lv[16];
  int n = 0;
  for (int i = 0; i <= 6; ++i) lv[n++] = -quantile(delta + i * (0.5L - delta) / 7.0L);  // negative side
  lv[n++] = 0.0L;
  for (int i = 7; i >= 0; --i) lv[n++] = quantile(delta + i * (0.5L - delta) / 8.0L);   // positive side
  const long double top = lv[15];
  Nf4Tables t{};
  for (int i = 0; i < 16; ++i) t.q[i] = (float)(double)(lv[i] / top);
  t.q[0] = -1.0f;  // lv[0] = -lv[15] exactly by construction
  t.q[7] = 0.0f;
  t.q[15] = 1.0f;
  for (int i = 0; i < 15; ++i) t.t[i] = round_down_to_float(((double)t.q[i] + (double)t.q[i + 1]) * 0.5);
  fit_code_polynomial(t);
  return t;
}

// Levels given as doubles (each the correctly rounded fp64 value of an exact
// rational), rounded once to fp32, with their thresholds.
Nf4Tables from_levels(const double (&lv)[16]) {
  Nf4Tables t{};
  for (int i = 0; i < 16; ++i) t.q[i] = (float)lv[i];
  for (int i = 0; i < 15; ++i) t.t[i] = round_down_to_float(((double)t.q[i] + (double)t.q[i + 1]) * 0.5);
  t.poly_ok = false;
  return t;
}

// "A standard 4-bit float" (section "What it showed", third bullet): OCP
// E2M1 magnitudes 0, 1/2, 1, 3/2, 2, 3, 4, 6 over 6, mirrored, one zero,
// and the pad level -2.
Nf4Tables build_fp4() {
  const double mags[7] = {0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  double lv[16];
  lv[0] = -2.0;
  for (int i = 0; i < 7; ++i) lv[1 + i] = -mags[6 - i] / 6.0;
  lv[8] = 0.0;
  for (int i = 0; i < 7; ++i) lv[9 + i] = mags[i] / 6.0;
  return from_levels(lv);
}

// "4-bit integers" (same bullet): symmetric levels k/7, k = -7 .. 7, and the
// unused two's-complement code -8 as the pad level -8/7.
Nf4Tables build_int4() {
  double lv[16];
  for (int k = -8; k < 8; ++k) lv[k + 8] = (double)k / 7.0;
  return from_levels(lv);
}

}  // namespace

namespace {
std::atomic<uint64_t> g_launches{0};
}

void count_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
uint64_t launches_so_far() { return g_launches.load(std::memory_order_relaxed); }

const Nf4Tables& nf4_tables() {
  static Nf4Tables tables;
  static std::once_flag once;
  std::call_once(once, [] { tables = build(); });
  return tables;
}

const Nf4Tables& code_tables(int format) {
  static Nf4Tables fp4, int4;
  static std::once_flag once;
  std::call_once(once, [] {
    fp4 = build_fp4();
    int4 = build_int4();
  });
  return format == 1 ? fp4 : format == 2 ? int4 : nf4_tables();
}

}  // namespace qnf4
