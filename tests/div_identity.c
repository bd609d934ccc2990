/* Checks the division identity the quantization kernel relies on (Markstein's
 * FMA-corrected quotient, "IA-64 and Elementary Functions", ch. 8): with r = RN(1/d),
 * q = RN(x r), e = x - q d (one FMA), RN(q + e r) with the sign of x equals the IEEE
 * binary32 quotient x / d
 *   - for every positive finite E4M3 divisor and every |x / d| in [2^-4, 2^4), visiting
 *     every `stride`-th binary32 x (stride 1 = exhaustive), both signs, and x = -0;
 *   - for d = 6 and every `stride`-th positive binary32 x whose quotient is normal.
 * And the one the second-level scale relies on: for every `stride`-th non-negative finite
 * binary32 x, fp32(double(x) * RN64(1/2688)) equals the IEEE binary32 quotient x / 2688
 * (the exact quotient's binary fraction repeats with period 6 -- 2688 = 21 * 2^7 -- so it
 * is never within 2^-52 of a binary32 rounding midpoint; subnormal quotients included).
 * And the per-element divisions of the quantizers by an arbitrary binary32 divisor d:
 * fp32(double(x) * c) equals x / d, with c the kernel's double reciprocal (the binary32
 * reciprocal refined by two Newton steps in double FMAs, d < 2^-64 scaled by 2^64), for
 * 4000 pseudo-random divisors in [2^-130, 2^21) and every (stride * 641)-th binary32 x.
 * And the paired-lane form the FP4 quantizer evaluates: with nr = -RN(1/d),
 * q' = RN(x nr), e = RN(x + q' d) (one FMA), RN(e nr + q') (one FMA) is, bit for bit,
 * div_fma(x, d) with its sign bit flipped -- for every positive finite E4M3 divisor, both
 * signs of +-0 and of the 4095 smallest subnormals (whose products underflow), and every
 * (stride * 67)-th binary32 x of the rest of the finite range whose quotient is finite
 * (the encoder then flips the E2M1 sign bits back).
 * Prints the number of mismatches of each part; exit status 0 when all are 0. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static double e4m3_value(int b) {
  const int e = (b >> 3) & 15, m = b & 7;
  return e == 0 ? ldexp(m, -9) : ldexp(1.0 + m / 8.0, e - 7);
}

static double recip_d(float d) {
  const int tiny = d < 5.421010862427522e-20f;
  const float ds = tiny ? d * 18446744073709551616.0f : d;
  const double dd = (double)ds;
  double y = (double)(1.0f / ds);
  y = fma(y, fma(-dd, y, 1.0), y);
  y = fma(y, fma(-dd, y, 1.0), y);
  return tiny ? y * 18446744073709551616.0 : y;
}

static float div_fma(float x, float d, float r) {
  const float q = x * r;
  const float e = fmaf(-q, d, x);
  return copysignf(fmaf(e, r, q), x);
}

/* The quantizer's negated form: no copysign, every step the negation of div_fma's. */
static float div_fma_neg(float x, float d, float nr) {
  const float nq = x * nr;
  const float e = fmaf(nq, d, x);
  return fmaf(e, nr, nq);
}

int main(int argc, char** argv) {
  const uint32_t stride = argc > 1 ? (uint32_t)strtoul(argv[1], NULL, 10) : 1u;
  long bad = 0, n = 0;
  for (int b = 1; b <= 0x7E; ++b) {
    const float d = (float)e4m3_value(b), r = 1.0f / d;
    const uint32_t lo = u_of(d * 0.0625f), hi = u_of(d * 16.0f);
    for (uint32_t u = lo; u < hi; u += stride) {
      for (int sg = 0; sg < 2; ++sg) {
        const float x = sg ? -f_of(u) : f_of(u);
        if (u_of(div_fma(x, d, r)) != u_of(x / d)) ++bad;
        ++n;
      }
    }
    if (u_of(div_fma(-0.0f, d, r)) != u_of(-0.0f / d)) ++bad;
    if (u_of(div_fma(0.0f, d, r)) != u_of(0.0f / d)) ++bad;
    n += 2;
  }
  long bad6 = 0, n6 = 0;
  const float r6 = 1.0f / 6.0f;
  for (uint32_t u = 0x01000000u; u < 0x7F800000u; u += stride) {  /* a / 6 normal */
    const float a = f_of(u);
    if (u_of(div_fma(a, 6.0f, r6)) != u_of(a / 6.0f)) ++bad6;
    ++n6;
  }
  long n2688 = 0, bad2688 = 0;
  const double c2688 = 1.0 / 2688.0;
  for (uint32_t u = 0; u < 0x7F800000u; u += stride) {  /* second-level scale: x / 2688 */
    const float x = f_of(u);
    volatile float ref = x / 2688.0f;
    const float got = (float)((double)x * c2688);
    ++n2688;
    if (u_of(ref) != u_of(got)) ++bad2688;
  }
  long nd = 0, badd = 0;
  uint32_t lcg = 12345u;
  for (int gi = 0; gi < 4000; ++gi) {  /* arbitrary divisors: quantizer x / g and x / s */
    lcg = lcg * 1664525u + 1013904223u;
    const float d = f_of(0x00000001u + (lcg >> 4) % 0x4A000000u);
    const double c = recip_d(d);
    for (uint32_t u = (lcg & 1023u); u < 0x7F800000u; u += stride * 641u) {
      const float x = f_of(u);
      volatile float ref = x / d;
      const float got = (float)((double)x * c);
      ++nd;
      if (u_of(ref) != u_of(got)) ++badd;
    }
  }
  long nneg = 0, badneg = 0;
  for (int b = 1; b <= 0x7E; ++b) {  /* the negated paired-lane form, every E4M3 divisor */
    const float d = (float)e4m3_value(b), r = 1.0f / d, nr = -r;
    /* +-0 and the 4095 smallest subnormals one by one, then every (stride * 67)-th x */
    for (uint32_t u = 0; u < 0x7F800000u; u += (u < 4096u ? 1u : stride * 67u)) {
      for (int sg = 0; sg < 2; ++sg) {
        const float x = sg ? -f_of(u) : f_of(u);
        const float ref = div_fma(x, d, r);
        if (!isfinite(ref)) continue;  /* |x / d| overflows: never in a block, whose scale */
                                       /* is at least its absmax / 6 or saturates at 448 */
        if (u_of(div_fma_neg(x, d, nr)) != (u_of(ref) ^ 0x80000000u)) ++badneg;
        ++nneg;
      }
    }
  }
  printf("e4m3 divisors: %ld checks, %ld mismatches; d = 6: %ld checks, %ld mismatches; "
         "x / 2688 by a double product: %ld checks, %ld mismatches; x / d by a double product: "
         "%ld checks, %ld mismatches; negated paired-lane form: %ld checks, %ld mismatches\n",
         n, bad, n6, bad6, n2688, bad2688, nd, badd, nneg, badneg);
  return (bad == 0 && bad6 == 0 && bad2688 == 0 && badd == 0 && badneg == 0) ? 0 : 1;
}
