/* Exhaustive checks of the divisions the append kernel takes without an IEEE
 * divide. All inputs are BF16 (or, for the INT8 range, the f32 difference of
 * two BF16 values), so every case the kernel can meet is enumerated.
 *
 * Mode "scale": the row scale. For a constant c and r = RN(1/c),
 *     q = RN(a r), q2 = fma(fma(-q, c, a), r, q)
 * must equal the IEEE quotient RN(a / c) bit for bit:
 *   c = 448 and c = 57344 for every non-negative BF16 a (the E4M3 and E5M2
 *   amax), c = 255 for every a = RN(hi - lo) with BF16 hi >= 0 >= lo (the
 *   INT8 range). The arguments slice the hi patterns.
 *
 * Mode "quot": the code quotient. For a BF16 scale s >= 2^-100 and every BF16
 * x with |x| <= 65536 s (subnormal x included), with r = RN(1/s):
 *     q = RN(x r), e = fma(q, s, -x), q2 = fma(-e, r, q)
 * (e is minus the exact residual; with the sign folded this way a zero x keeps
 * its sign through the correction, -0 giving -0).
 * q2 may differ from RN(x / s) in its last bit, but the E4M3 code (RNE,
 * saturating at 448), the E5M2 code (RNE, saturating at 57344) and the rint
 * integer taken from it must not. Scales below 2^-100 take the IEEE divide in
 * the kernel and are not enumerated. The arguments slice the scale patterns.
 *
 * Usage: scale_division_check scale|quot <first pattern> <end pattern>
 * Prints "checked N differ D mismatches M" and exits 1 on any mismatch.
 * Host-only test program; it shares nothing with the kernels it checks. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float from_bf16(uint32_t h) {
  const uint32_t u = h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static uint32_t f32_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

/* Finite magnitudes of an FP8 format in code order, from its definition. */
static void fp8_table(double* t, int mbits, int bias, int ncodes) {
  for (int c = 0; c < ncodes; ++c) {
    const int e = c >> mbits, m = c & ((1 << mbits) - 1);
    const double frac = (double)m / (double)(1 << mbits);
    t[c] = e ? (1.0 + frac) * ldexp(1.0, e - bias) : frac * ldexp(1.0, 1 - bias);
  }
}

/* Nearest table entry, ties to the even code, saturating, sign bit kept. */
static int encode(const double* t, int n, float x) {
  const double m = fabs((double)x);
  int code;
  if (m >= t[n - 1]) {
    code = n - 1;
  } else {
    int lo = 0, hi = n - 1;
    while (hi - lo > 1) {
      const int mid = (lo + hi) / 2;
      if (t[mid] <= m) lo = mid; else hi = mid;
    }
    const double dl = m - t[lo], dh = t[hi] - m;
    code = (dh < dl || (dh == dl && hi % 2 == 0)) ? hi : lo;
  }
  return signbit(x) ? (code | 0x80) : code;
}

static float div_const(float a, float c, float r) {
  const float q = a * r;
  return fmaf(fmaf(-q, c, a), r, q);
}

int main(int argc, char** argv) {
  if (argc != 4) {
    fprintf(stderr, "usage: %s scale|quot first end\n", argv[0]);
    return 2;
  }
  const int quot = strcmp(argv[1], "quot") == 0;
  const uint32_t first = (uint32_t)strtoul(argv[2], 0, 0), end = (uint32_t)strtoul(argv[3], 0, 0);
  unsigned long long checked = 0, differ = 0, bad = 0;
  if (!quot) {
    if (first == 0) {
      const float cs[2] = {448.0f, 57344.0f};
      for (int k = 0; k < 2; ++k) {
        const float c = cs[k], r = 1.0f / c;
        for (uint32_t h = 0; h < 0x7F80; ++h) {
          const float a = from_bf16(h);
          ++checked;
          if (f32_bits(div_const(a, c, r)) != f32_bits(a / c)) {
            if (bad < 8) printf("mismatch a=%a c=%g\n", a, c);
            ++bad;
          }
        }
      }
    }
    const float c = 255.0f, r = 1.0f / c;
    for (uint32_t hh = first; hh < end && hh < 0x7F80; ++hh) {
      const float hi = from_bf16(hh);
      for (uint32_t hl = 0; hl < 0x7F80; ++hl) {
        const float a = hi - -from_bf16(hl);
        if (isinf(a)) continue;
        ++checked;
        if (f32_bits(div_const(a, c, r)) != f32_bits(a / c)) {
          if (bad < 8) printf("mismatch range=%a\n", a);
          ++bad;
        }
      }
    }
    printf("checked %llu differ %llu mismatches %llu\n", checked, bad, bad);
    return bad ? 1 : 0;
  }
  static double e4m3[127], e5m2[124];
  fp8_table(e4m3, 3, 7, 127);   /* 0x7F is NaN; 0x7E = 448 */
  fp8_table(e5m2, 2, 15, 124);  /* 0x7C.. are inf/NaN; 0x7B = 57344 */
  const float s_fast = ldexpf(1.0f, -100);
  for (uint32_t hs = first; hs < end && hs < 0x7F80; ++hs) {
    const float s = from_bf16(hs);
    if (!(s >= s_fast)) continue;
    const float r = 1.0f / s;
    const float lim = 65536.0f * s;
    for (uint32_t hx = 0; hx < 0x7F80; ++hx) {
      const float xa = from_bf16(hx);
      if (xa > lim) break;
      for (int neg = 0; neg < 2; ++neg) {
        const float x = neg ? -xa : xa;
        const float q = x * r;
        const float e = fmaf(q, s, -x);          /* minus the residual x - q s, exact */
        const float q2 = fmaf(-e, r, q);
        const float ref = x / s;
        ++checked;
        if (f32_bits(q2) == f32_bits(ref)) continue;
        ++differ;
        if (encode(e4m3, 127, q2) != encode(e4m3, 127, ref) ||
            encode(e5m2, 124, q2) != encode(e5m2, 124, ref) || nearbyintf(q2) != nearbyintf(ref)) {
          if (bad < 8) printf("mismatch s=%a x=%a q2=%a ieee=%a\n", s, x, q2, ref);
          ++bad;
        }
      }
    }
  }
  printf("checked %llu differ %llu mismatches %llu\n", checked, differ, bad);
  return bad ? 1 : 0;
}
