/* Check of the stochastic-rounding methods the CUDA kernels use, against the
 * oracle's definition (linked from oracle/fp4q_oracle.c).
 *
 * Method 0 (codes): for |v| in [1, 6] the E2M1 grid coordinate is
 * G * 2^22 = bits(|v|) - 0x3F000000 and the code is
 * (bits - 0x3EC00001 - (u << 6)) >> 22 (one carry decides "u * 64 < frac");
 * below 1 the grid is uniform, C = ceil(|v| * 2^17) is read from
 * RU(|v| * 2^17 + 2^23) and the code is (C + 0xFFFF - u) >> 16.
 *
 * Method 1 (values): on [1, 8) E2M1 is a float with one mantissa bit, so the
 * stochastically rounded magnitude is (bits(w) + 0x3FFFFF - 64 u) with the
 * low 22 bits cleared; below 1 the spacing 0.5 is that of [1, 2), so
 * w = RU(|v| + 1) is rounded the same way and 1 subtracted again (rounding
 * the sum up keeps "64 u < frac" exact, as frac is compared with an integer).
 * The sign is copied and the value converted by round-to-nearest-even with
 * saturation (the hardware conversion; the oracle's RNE stands in for it
 * here), which also maps 8 to 6.
 *
 * Method 2 (subnormal scaling): multiplying |v| by 2^-126 maps E2M1's grid
 * onto float bit patterns with one rule everywhere: [1, 8) becomes three
 * normal binades whose E2M1 values keep one mantissa bit, and [0, 1) becomes
 * the subnormal range, whose uniform step 2^-149 makes E2M1's spacing 0.5
 * (2^-127) exactly 2^22 steps, the same as in [1, 2).  So the magnitude is
 * rounded by adding 0x3FFFFF - 64 u to bits(w) and clearing the low 22 bits,
 * for every |v|, with no test of the range.  The product is rounded up
 * (towards +inf on the non-negative |v|), which keeps "64 u < frac" exact
 * where the scaling drops low bits of |v| < 1.  The sign is put back, the
 * value multiplied by 2^126 (exact) and converted as for method 1.
 *
 * Method 3 (method 2 with a truncating conversion): the low 22 bits are left
 * as they are and the conversion truncates towards zero onto the E2M1 grid,
 * saturating at 6 (cvt.rs.satfinite.e2m1x4 with zero random bits, which adds
 * nothing below the kept bits).  Everything below the kept mantissa bit is
 * then dropped by the conversion instead of the mask.  Without the mask an
 * infinite |v| would turn into a NaN pattern, so the scaled product saturates
 * at 1 (mul.rp.sat): every |v| >= 2^126 maps to [1, 1.5) * 2^126, which the
 * conversion saturates to 6 like the oracle.

 * Usage: sr_check <n_random> [method] -- prints the number of mismatches. */
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

uint8_t orc_e2m1_rne(float v);

static uint32_t method1(float v, uint32_t u16) {
  uint32_t raw = bits(v);
  float av = fabsf(v);
  float a = av < 1.0f ? 1.0f : 0.0f;
  fesetround(FE_UPWARD);
  volatile float w = av + a;
  fesetround(FE_TONEAREST);
  uint32_t R = (bits(w) + (0x3FFFFFu - (u16 << 6))) & 0xFFC00000u;
  volatile float r = flt(R) - a;
  return orc_e2m1_rne(flt(bits(r) | (raw & 0x80000000u)));
}

static uint32_t method2(float v, uint32_t u16) {
  uint32_t raw = bits(v);
  fesetround(FE_UPWARD);
  volatile float w = fabsf(v) * 0x1p-126f;
  fesetround(FE_TONEAREST);
  uint32_t R = (bits(w) + 0x3FFFFFu - (u16 << 6)) & 0xFFC00000u;
  volatile float r = flt(R | (raw & 0x80000000u)) * 0x1p126f;
  return orc_e2m1_rne(r);
}

/* truncation of x towards zero onto the E2M1 grid, saturating at 6 */
static uint32_t e2m1_trunc(float x) {
  static const float grid[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  float a = fabsf(x);
  uint32_t c = 0;
  for (uint32_t k = 0; k < 8; ++k)
    if (grid[k] <= a) c = k;
  return c | (signbit(x) ? 8u : 0u);
}

static uint32_t method3(float v, uint32_t u16) {
  uint32_t raw = bits(v);
  fesetround(FE_UPWARD);
  volatile float w = fabsf(v) * 0x1p-126f;
  fesetround(FE_TONEAREST);
  float ws = w > 1.0f ? 1.0f : w;            /* .sat */
  uint32_t T = bits(ws) + 0x3FFFFFu - (u16 << 6);
  volatile float r = flt(T | (raw & 0x80000000u)) * 0x1p126f;
  return e2m1_trunc(r);
}

static uint64_t s = 0x9E3779B97F4A7C15ull;
static uint64_t rnd(void) { s ^= s << 13; s ^= s >> 7; s ^= s << 17; return s; }

static int which = 0;
static uint32_t pick(float v, uint32_t u16) {
  return which == 3   ? method3(v, u16)
         : which == 2 ? method2(v, u16)
         : which      ? method1(v, u16)
                      : method(v, u16);
}

int main(int argc, char **argv) {
  long n = atol(argv[1]);
  if (argc > 2) which = atoi(argv[2]);
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
        if (pick(v, u) != orc_e2m1_sr(v, u)) ++bad;
        if (pick(-v, u) != orc_e2m1_sr(-v, u)) ++bad;
      }
    }
  /* the extremes that method 2's scaling reaches: subnormal and tiny v
     (the product drops low bits), the smallest normals, and magnitudes so
     large that the scaled value rounds up to 2^128 */
  const uint32_t edge[] = {0x00000001u, 0x00000003u, 0x00012345u, 0x007FFFFFu, 0x00800000u,
                           0x00800001u, 0x01000000u, 0x0C000001u, 0x33800001u, 0x34000001u,
                           0x7F7FFFFFu, 0x7F3FFFFFu, 0x7F400000u, 0x7E000001u,
                           0x7F800000u, 0x7E800000u, 0x7E7FFFFFu, 0x40FFFFFFu, 0x41000000u};
  if (which >= 2)
    for (unsigned i = 0; i < sizeof edge / sizeof edge[0]; ++i)
      for (uint32_t u = 0; u < 65536; ++u) {
        float v = flt(edge[i]);
        if (pick(v, u) != orc_e2m1_sr(v, u)) ++bad;
        if (pick(-v, u) != orc_e2m1_sr(-v, u)) ++bad;
      }
  for (long i = 0; i < n; ++i) {
    uint64_t r = rnd();
    /* magnitudes spread over [2^-30, 16) */
    float v = flt((uint32_t)(0x30800000u + (r % (0x41800000u - 0x30800000u))));
    if (r >> 63) v = -v;
    uint32_t u = (uint32_t)(r >> 40) & 0xFFFFu;
    if (pick(v, u) != orc_e2m1_sr(v, u)) ++bad;
  }
  printf("%ld\n", bad);
  return 0;
}
