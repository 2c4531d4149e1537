/* Exhaustive check of the division-by-6 method the CUDA kernels use for
 * block scales (Markstein's correction step, P. Markstein, "Computation of
 * elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
 * Dev. 34(1), 1990):  q0 = RN(y * c), r = fma(-q0, 6, y), q = fma(r, c, q0)
 * with c = RN(1/6).  Compares q with the IEEE quotient RN(y / 6) for every
 * float y with bit pattern in [lo, hi); prints the number of mismatches and
 * the largest mismatching y. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

int main(int argc, char **argv) {
  uint32_t lo = (uint32_t)strtoul(argv[1], 0, 0), hi = (uint32_t)strtoul(argv[2], 0, 0);
  volatile float six = 6.0f, one = 1.0f;
  float c = one / six;
  uint64_t bad = 0;
  float worst = 0.0f;
  for (uint32_t b = lo; b < hi; ++b) {
    float y;
    memcpy(&y, &b, 4);
    float q0 = y * c;
    float r = fmaf(-q0, 6.0f, y);
    float q = fmaf(r, c, q0);
    float ref = y / six;
    if (q != ref) { ++bad; if (y > worst) worst = y; }
  }
  printf("%llu %.9g\n", (unsigned long long)bad, worst);
  return 0;
}
