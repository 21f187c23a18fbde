// Host check of the NF4 quantiser's fast code path (csrc/quant.cu), run by
// tests/test_quant_fastpath_host.py.
//
// For block scales c in [2^-90, 2^100) the kernel does not divide: it takes a
// correctly rounded reciprocal rc = RN32(1/c), forms q0 = RN32(w * rc), one
// fused correction e = fma(q0, -c, w), x = fma(e, rc, q0) (a Markstein
// step), then evaluates the library's code-search polynomial f(x) with fused
// multiply-adds, takes k = round(f(x) - 1/2) through the 1.5 * 2^23 trick and
// finishes with one threshold compare, code = k + (x > t[k]).
//
// This program replays exactly that arithmetic on the host (fmaf is a
// correctly rounded fused multiply-add, -ffp-contract=off keeps the other
// operations separate) for every pair of bf16 values (w, c) with c in that
// range and |w| <= c, and compares the code with the definition: the number
// of thresholds below the IEEE quotient w / c.  Prints the pair count and the
// mismatch count; exits 1 on any mismatch.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "internal.h"

static float bf16_value(uint32_t bits) {
  const uint32_t u = bits << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}
static uint32_t float_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}

int main() {
  const qnf4::Nf4Tables& t = qnf4::nf4_tables();
  if (!t.poly_ok) {
    std::printf("polynomial check failed on the host\n");
    return 1;
  }
  const uint32_t c_lo = 0x1280u, c_hi = 0x7180u;  // bf16 bits of 2^-90 and 2^100
  long long pairs = 0, bad = 0, k_out = 0;
#pragma omp parallel for schedule(dynamic, 16) reduction(+ : pairs, bad, k_out)
  for (int cb = (int)c_lo; cb < (int)c_hi; ++cb) {
    const float c = bf16_value((uint32_t)cb);
    const float rc = 1.0f / c;
    for (uint32_t wb = 0; wb < 0x10000u; ++wb) {
      if ((wb & 0x7F80u) == 0x7F80u) continue;  // Inf / NaN patterns
      const float w = bf16_value(wb);
      if (std::fabs(w) > c) continue;
      const float q0 = w * rc;
      const float e = std::fmaf(q0, -c, w);
      const float x = std::fmaf(e, rc, q0);
      float f = t.poly[5];
      for (int k = 4; k >= 0; --k) f = std::fmaf(f, x, t.poly[k]);
      const float y = f + 12582912.0f;
      const uint32_t k = float_bits(y) - 0x4B400000u;
      uint32_t code = 99;
      if (k <= 14u) code = k + (x > t.t[k] ? 1u : 0u);
      else ++k_out;
      const float ex = w / c;
      uint32_t ref = 0;
      for (int i = 0; i < 15; ++i) ref += ex > t.t[i] ? 1u : 0u;
      ++pairs;
      if (code != ref) ++bad;
    }
  }
  std::printf("pairs=%lld mismatches=%lld k_out_of_range=%lld\n", pairs, bad, k_out);
  return bad != 0 || k_out != 0;
}
