/* The NVFP4 block scale divides the block amax by 6 with one FMA correction of m * fp32(1/6)
 * instead of an IEEE division (quant_nvfp4.cu, div6_rn).  This program checks that claim for
 * every FP32 value m in [2^-125, FLT_MAX]: fma(fma(-6, q0, m), fp32(1/6), q0) with
 * q0 = fp32(m * fp32(1/6)) must equal the correctly rounded m / 6.  Prints the number of
 * mismatches and of values checked. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float from_bits(uint32_t b) {
  float x;
  memcpy(&x, &b, sizeof x);
  return x;
}

int main(void) {
  const float sixth = 0.16666667163372039794921875f; /* fp32(1/6) = 0x3E2AAAAB */
  uint64_t bad = 0, n = 0;
  for (uint32_t b = 0x01000000u; b <= 0x7F7FFFFFu; ++b) { /* 2^-125 .. FLT_MAX */
    const float m = from_bits(b);
    const float q0 = m * sixth;
    const float q = fmaf(fmaf(-6.0f, q0, m), sixth, q0);
    bad += (q != m / 6.0f);
    ++n;
  }
  printf("%llu %llu\n", (unsigned long long)bad, (unsigned long long)n);
  return 0;
}
