/* Exhaustive host check of the fast division the kernels use.
 *
 * The GEMM, dequantisation and merge kernels form the block scale from the
 * second-level constants as q = c2 / c1 with a cached correctly rounded
 * reciprocal rc = RN(1/c1) and one residual correction
 *     y = RN(w rc);  e = fma(-c1, y, w);  q = fma(e, rc, y).
 * The quantiser forms x = w / s the same way for bf16 w and bf16 s.
 * This program checks that q equals the correctly rounded quotient:
 *   int8  : every fp32 significand of c1 in [1, 2) against every integer
 *           numerator in [-127, 127] (the Int8 constants), then c1 at the
 *           exponents -60 and +60 with a stride through the significands;
 *   e4m3  : the same c1 significands against every finite E4M3 value (the FP8
 *           constants);
 *   bf16  : every bf16 s in [1, 2) against every bf16 w with 2^-102 <= |w|
 *           <= s, both signs (the quantiser; smaller quotients map to the
 *           zero code whatever their last bits), also against an exact
 *           128-bit integer division.
 * A zero numerator is the one case where the sequence can differ: -0 gives +0
 * instead of -0.  The block scale is RN(q + mean) with mean >= 0, which is the
 * same for either zero, so zero quotients are compared by value.
 * Numerator and denominator scale by powers of two without changing any
 * rounding, as long as every intermediate stays normal, so these ranges cover
 * c1 in [2^-60, 2^60].  The reference is the host's IEEE single-precision
 * division; build without FMA contraction (-ffp-contract=off) on x86-64 SSE.
 * Usage: division_check int8|e4m3|bf16 ; prints "total N bad M", exits 1 on
 * any mismatch. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float f_of(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }
static uint32_t u_of(float x) { uint32_t v; memcpy(&v, &x, 4); return v; }

static float fast_div(float w, float c, float rc) {
  const float y = w * rc;
  const float e = fmaf(-c, y, w);
  return fmaf(e, rc, y);
}

/* RN(a / b) for positive normal a, b by integer long division */
static float exact_div(float a, float b) {
  int ea, eb;
  const float ma = frexpf(a, &ea), mb = frexpf(b, &eb);
  const uint64_t A = (uint64_t)ldexpf(ma, 24), B = (uint64_t)ldexpf(mb, 24);
  const unsigned __int128 num = (unsigned __int128)A << 40;
  const uint64_t qi = (uint64_t)(num / B);
  const int rem = (num % B) != 0;
  int sh = 0;
  uint64_t t = qi;
  while (t >= (1ull << 25)) { t >>= 1; ++sh; }
  const int sticky = rem || (qi & ((1ull << sh) - 1)) != 0;
  uint64_t q24 = t >> 1;
  const int guard = (int)(t & 1);
  if (guard && (sticky || (q24 & 1))) ++q24;
  return (float)ldexp((double)q24, ea - eb - 40 + sh + 1);
}

static float e4m3_value(int code) {   /* finite codes only */
  const int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
  const double v = e ? (1.0 + m / 8.0) * ldexp(1.0, e - 7) : m * ldexp(1.0, -9);
  return (float)(s ? -v : v);
}

static long check_c1_range(const float* nums, int nnum, uint32_t exp_bits, uint32_t stride, long* bad) {
  long tot = 0;
  for (uint32_t m = 0; m < (1u << 23); m += stride) {
    const float c = f_of(exp_bits | m);
    const float rc = 1.0f / c;
    for (int i = 0; i < nnum; ++i) {
      const float w = nums[i];
      const float q = fast_div(w, c, rc), ref = w / c;
      ++tot;
      if (u_of(q) != u_of(ref) && !(q == 0.0f && ref == 0.0f)) {
        if (*bad < 5) printf("c1=%a w=%a fast=%a ieee=%a\n", c, w, q, ref);
        ++*bad;
      }
    }
  }
  return tot;
}

int main(int argc, char** argv) {
  long tot = 0, bad = 0;
  if (argc < 2) return 2;
  if (!strcmp(argv[1], "int8") || !strcmp(argv[1], "e4m3")) {
    float nums[256];
    int n = 0;
    if (!strcmp(argv[1], "int8")) {
      for (int c = -127; c <= 127; ++c) nums[n++] = (float)c;
    } else {
      for (int code = 0; code < 256; ++code)
        if ((code & 0x7F) != 0x7F) nums[n++] = e4m3_value(code);
    }
    tot += check_c1_range(nums, n, 0x3F800000u, 1, &bad);                 /* c1 in [1, 2) */
    tot += check_c1_range(nums, n, (uint32_t)(127 - 60) << 23, 97, &bad);  /* c1 near 2^-60 */
    tot += check_c1_range(nums, n, (uint32_t)(127 + 60) << 23, 97, &bad);  /* c1 near 2^60 */
  } else if (!strcmp(argv[1], "bf16")) {
    for (uint32_t sb = 0x3F80; sb < 0x4000; ++sb) {
      const float s = f_of(sb << 16);
      const float r = 1.0f / s;
      for (int neg = 0; neg < 2; ++neg)
        for (uint32_t wb = 0x0C80; wb <= sb; ++wb) {   /* 0x0C80 is 2^-102 */
          float w = f_of(wb << 16);
          const float ex = neg ? -exact_div(w, s) : exact_div(w, s);
          if (neg) w = -w;
          const float q = fast_div(w, s, r), ref = w / s;
          ++tot;
          if (u_of(q) != u_of(ex) || u_of(ref) != u_of(ex)) {
            if (bad < 5) printf("s=%a w=%a fast=%a ieee=%a exact=%a\n", s, w, q, ref, ex);
            ++bad;
          }
        }
    }
  } else {
    return 2;
  }
  printf("total %ld bad %ld\n", tot, bad);
  return bad ? 1 : 0;
}
