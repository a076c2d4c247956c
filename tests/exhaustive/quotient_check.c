/* Exhaustive check of the encoder's quotient: for a divisor s whose
 * significand has at most 11 bits (every fp16 value; also 3, 15 and 255) and any
 * binary32 dividend u, Markstein's correction step
 *     r = RN(1/s), q0 = RN(u r), q1 = RN(q0 + RN(u - q0 s) r)   (FMAs)
 * gives q1 = RN(u / s).  All steps scale exactly with the exponents of u and
 * s, so it suffices to take u and s in [1, 2): 2^10 divisor significands x
 * 2^23 dividend significands.  The reference RN32(RN64(u / s)) is correctly
 * rounded because binary64 has more than 2 * 24 + 2 bits.
 * Prints "mismatches N of M"; exit status 0 iff N == 0.
 * argv[1] (optional): "skip-correction" drops the correction (q1 = q0), a
 * control that must report mismatches. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float from_bits(uint32_t b) {
  float f;
  memcpy(&f, &b, sizeof f);
  return f;
}

int main(int argc, char** argv) {
  const int control = argc > 1 && strcmp(argv[1], "skip-correction") == 0;
  long long bad = 0, total = 0;
#pragma omp parallel for reduction(+ : bad, total) schedule(dynamic)
  for (int m = 0; m < 1024; ++m) {
    const float s = from_bits(0x3F800000u | ((uint32_t)m << 13));
    const float r = (float)(1.0 / (double)s);
    long long local = 0;
    for (uint32_t um = 0; um < (1u << 23); ++um) {
      const float u = from_bits(0x3F800000u | um);
      const float q0 = u * r;
      const float q1 = control ? q0 : fmaf(fmaf(-q0, s, u), r, q0);
      if (q1 != (float)((double)u / (double)s)) ++local;
    }
    bad += local;
    total += 1LL << 23;
  }
  printf("mismatches %lld of %lld\n", bad, total);
  return bad != 0;
}
