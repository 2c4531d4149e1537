/* Check of the stochastic-rounding method the CUDA kernels use, against the
 * oracle's definition (linked from oracle/fp4q_oracle.c): for |v| in [1, 6]
 * the E2M1 grid coordinate is G * 2^22 = bits(|v|) - 0x3F000000 and the code
 * is (bits - 0x3EC00001 - (u << 6)) >> 22 (one carry decides "u * 64 < frac");
 * below 1 the grid is uniform, C = ceil(|v| * 2^17) is read from
 * RU(|v| * 2^17 + 2^23) and the code is (C + 0xFFFF - u) >> 16.
 * Usage: sr_check <n_random> -- prints the number of mismatches. */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

uint8_t orc_e2m1_sr(float v, uint32_t u16);

static uint32_t bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float flt(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

static uint32_t method(float v, uint32_t u16) {
  uint32_t raw = bits(v), b = raw & 0x7FFFFFFFu;
  uint32_t codeA = (b - 0x3EC00001u - (u16 << 6)) >> 22;
  if (codeA > 7u) codeA = 7u;
  fesetround(FE_UPWARD);
  volatile float a = flt(b);
  float xu = fmaf(a, 131072.0f, 8388608.0f);
  fesetround(FE_TONEAREST);
  uint32_t codeB = (bits(xu) - 0x4AFF0001u - u16) >> 16;
  uint32_t code = b >= 0x3F800000u ? codeA : codeB;
  return code | ((raw >> 28) & 8u);
}

static uint64_t s = 0x9E3779B97F4A7C15ull;
static uint64_t rnd(void) { s ^= s << 13; s ^= s >> 7; s ^= s << 17; return s; }

int main(int argc, char **argv) {
  long n = atol(argv[1]);
  long bad = 0;
  /* every E2M1 boundary region: values near grid points and midpoints,
     with all 2^16 u for each, then random (v, u) pairs */
  const float pts[] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f, 0.25f, 0.75f,
                       1.25f, 1.75f, 2.5f, 3.5f, 5.0f, 8.0f};
  for (unsigned i = 0; i < sizeof pts / sizeof pts[0]; ++i)
    for (int d = -6; d <= 6; ++d) {
      uint32_t b = bits(pts[i]);
      if ((int64_t)b + d < 0) continue;
      float v = flt(b + d);
      for (uint32_t u = 0; u < 65536; ++u) {
        if (method(v, u) != orc_e2m1_sr(v, u)) ++bad;
        if (method(-v, u) != orc_e2m1_sr(-v, u)) ++bad;
      }
    }
  for (long i = 0; i < n; ++i) {
    uint64_t r = rnd();
    /* magnitudes spread over [2^-30, 16) */
    float v = flt((uint32_t)(0x30800000u + (r % (0x41800000u - 0x30800000u))));
    if (r >> 63) v = -v;
    uint32_t u = (uint32_t)(r >> 40) & 0xFFFFu;
    if (method(v, u) != orc_e2m1_sr(v, u)) ++bad;
  }
  printf("%ld\n", bad);
  return 0;
}
