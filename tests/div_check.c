/* Exhaustive check of the division-by-a-constant method the CUDA kernels use
 * for block scales (Markstein's correction step, P. Markstein, "Computation
 * of elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
 * Dev. 34(1), 1990):  q0 = RN(y * c), r = fma(-q0, d, y), q = fma(r, c, q0)
 * with c = RN(1/d).  Compares q with the IEEE quotient RN(y / d) for every
 * float y with bit pattern in [lo, hi); prints the number of mismatches and
 * the largest mismatching y.  Usage: div_check lo hi [d] (d defaults to 6:
 * the NVFP4 and MXFP4 grid maximum; 7.5 and 28 are the FP6 maxima). */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

int main(int argc, char **argv) {
  uint32_t lo = (uint32_t)strtoul(argv[1], 0, 0), hi = (uint32_t)strtoul(argv[2], 0, 0);
  volatile float six = argc > 3 ? strtof(argv[3], 0) : 6.0f, one = 1.0f;
  const float d = six;
  float c = one / six;
  uint64_t bad = 0;
  float worst = 0.0f;
  for (uint32_t b = lo; b < hi; ++b) {
    float y;
    memcpy(&y, &b, 4);
    float q0 = y * c;
    float r = fmaf(-q0, d, y);
    float q = fmaf(r, c, q0);
    float ref = y / six;
    if (q != ref) { ++bad; if (y > worst) worst = y; }
  }
  printf("%llu %.9g\n", (unsigned long long)bad, worst);
  return 0;
}
