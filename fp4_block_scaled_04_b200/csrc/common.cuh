// common.cuh -- device helpers shared by the fp4q kernels (sm_100a only).
//
// Every floating-point step that decides a code uses an explicitly rounded
// intrinsic (__fmul_rn, __fadd_rn, __fdiv_rn, __fmaf_rn) or a hand-written
// PTX conversion, and the translation units are compiled with -fmad=false
// -ftz=false -prec-div=true, so the result is the same binary32 value the
// library documents in include/fp4q.h.
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fp4q.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "fp4q kernels target sm_100a only"
#endif

namespace fp4q {


// ---------------------------------------------------------------------------
// element loads
// ---------------------------------------------------------------------------

// BF16 pair packed in a 32-bit word: the low half is the lower address.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Load 8 consecutive elements starting at p (16-byte aligned for BF16, 32 for FP32).
template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
  __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&v)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
  }
};
template <> struct Vec8<float> {
  __device__ __forceinline__ static void load(const float *p, float (&v)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};

// ---------------------------------------------------------------------------
// E2M1 encode / decode
// ---------------------------------------------------------------------------

// Round two floats to E2M1 (nearest, ties to even, saturating at +-6, sign
// kept) with the sm_100a conversion instruction; `lo` lands in bits 0..3.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
      "cvt.u16.u8 %0, t;\n\t}"
      : "=h"(r) : "f"(lo), "f"(hi));
  return r;
}

// Eight floats -> eight nibbles in one word, v[0] in bits 0..3.
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
        "f"(v[7]));
  return r;
}

// Four floats -> four nibbles in the low 16 bits, f0 in bits 0..3.
__device__ __forceinline__ uint32_t e2m1x4(float f0, float f1, float f2, float f3) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1;\n\t.reg .b16 h;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "mov.b16 h, {b0, b1};\n\t"
      "cvt.u32.u16 %0, h;\n\t}"
      : "=r"(r) : "f"(f0), "f"(f1), "f"(f2), "f"(f3));
  return r;
}

// The truncating forms of e2m1x8 and e2m1x4: each value goes to the largest
// E2M1 magnitude not above |v| (6 for anything larger, infinity included),
// with its sign.  This is cvt.rs.satfinite with zero random bits: the
// stochastic conversion adds its random bits below the kept ones before
// dropping them, so with none it truncates.  The stochastic-rounding paths
// feed it the dithered values of e2m1_sr_dithered2.  The first operand of
// the x4 conversion lands in the top nibble.
__device__ __forceinline__ uint32_t e2m1x8_rz(const float (&v)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b16 h0, h1;\n\t"
      "cvt.rs.satfinite.e2m1x4.f32 h0, {%4, %3, %2, %1}, %9;\n\t"
      "cvt.rs.satfinite.e2m1x4.f32 h1, {%8, %7, %6, %5}, %9;\n\t"
      "mov.b32 %0, {h0, h1};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
        "f"(v[7]), "r"(0u));
  return r;
}
__device__ __forceinline__ uint32_t e2m1x4_rz(float f0, float f1, float f2, float f3) {
  uint16_t h;
  asm("cvt.rs.satfinite.e2m1x4.f32 %0, {%4, %3, %2, %1}, %5;"
      : "=h"(h) : "f"(f0), "f"(f1), "f"(f2), "f"(f3), "r"(0u));
  return h;
}

// ---------------------------------------------------------------------------
// E4M3 encode / decode (block scales)
// ---------------------------------------------------------------------------

// s >= 0 -> E4M3 code, round to nearest even, saturating at 448 (0x7E).  The
// code is masked to 7 bits, a no-op for s >= 0 that keeps it a valid index
// into a 128-entry factor table even for a NaN (lanes outside the matrix may
// compute on stale values whose results are never stored).
__device__ __forceinline__ uint32_t e4m3_code(float s) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
  return r & 0x7Fu;
}

// Value of a 7-bit E4M3 magnitude code (sign bit ignored).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t e = (code >> 3) & 15u, m = code & 7u;
  if (e == 0) return __fmul_rn(static_cast<float>(m), 0.001953125f);  // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// ---------------------------------------------------------------------------
// NVFP4 tensor and block scales
// ---------------------------------------------------------------------------

struct TensorScale {
  float enc;  // RN(2688 / amax), clamped to FLT_MAX; 1 if amax == 0
  float dec;  // RN(amax / 2688); 1 if amax == 0
};

// Tensor scales for a block grid whose largest magnitude is QMAX: the top
// value is QMAX * 448 (E4M3 max), 2688 for NVFP4 (QMAX 6) and 1792 for the
// four-over-six variant (QMAX 4).
template <int QMAX>
__device__ __forceinline__ TensorScale tensor_scale_q(float amax) {
  constexpr float top = static_cast<float>(QMAX) * 448.0f;
  TensorScale t;
  if (amax == 0.0f) {
    t.enc = 1.0f;
    t.dec = 1.0f;
  } else {
    t.enc = fminf(__fdiv_rn(top, amax), 3.402823466e+38f);
    t.dec = __fdiv_rn(amax, top);
  }
  return t;
}

__device__ __forceinline__ TensorScale tensor_scale(float amax) {
  return tensor_scale_q<6>(amax);
}

// RN(y / 6) in three instructions: Markstein's correction of RN(y * RN(1/6))
// with an exact FMA remainder (P. Markstein, IBM J. Res. Dev. 34(1), 1990).
// Equal to the IEEE quotient for every float y in [2^-125, 4096] (checked
// exhaustively on the host by tests/div_check.c); below that the quotient
// is subnormal, where callers either do not care (E4M3 rounds it to 0) or
// use the IEEE division.
__device__ __forceinline__ float div6(float y) {
  constexpr float kInv6 = 1.0f / 6.0f;   // RN(1/6)
  const float q0 = __fmul_rn(y, kInv6);
  const float r = __fmaf_rn(-q0, 6.0f, y);
  return __fmaf_rn(r, kInv6, q0);
}

// RN(y / d) by the same correction for the FP6 grid maxima d = 7.5 and 28
// (inv_d = RN(1/d)); equal to the IEEE quotient for every float y >= 2^-122
// (tests/div_check.c, exhaustively), the IEEE division below that.
__device__ __forceinline__ float div_qmax(float y, float d, float inv_d) {
  if (!(y >= 0x1p-122f)) return __fdiv_rn(y, d);
  const float q0 = __fmul_rn(y, inv_d);
  const float r = __fmaf_rn(-q0, d, y);
  return __fmaf_rn(r, inv_d, q0);
}

// E4M3 code of the block scale: RN(RN(m * s_enc) / 6).  RN(m * s_enc) is at
// most 2688 (1 + 2^-23); where it is below 2^-125 both quotients lie far
// below the smallest E4M3 subnormal and give code 0.
__device__ __forceinline__ uint32_t nvfp4_scale_code(float block_amax, float s_enc) {
  return e4m3_code(div6(__fmul_rn(block_amax, s_enc)));
}

// The same for a grid maximum QMAX: RN(RN(m * s_enc) / QMAX); dividing by 4
// is the exact product with 0.25.
template <int QMAX>
__device__ __forceinline__ uint32_t scale_code_q(float block_amax, float s_enc) {
  static_assert(QMAX == 6 || QMAX == 4, "grid maximum 6 or 4");
  if (QMAX == 6) return nvfp4_scale_code(block_amax, s_enc);
  return e4m3_code(__fmul_rn(__fmul_rn(block_amax, s_enc), 0.25f));
}

// Per-CTA table of r = RN(s_enc / S) for the 128 non-negative E4M3 codes
// (0 for S == 0, clamped to FLT_MAX like s_enc); one IEEE division per code
// instead of one per block.
__device__ __forceinline__ void fill_factor_table(float *tab, float s_enc) {
  for (int c = threadIdx.x; c < 128; c += blockDim.x) {
    float S = e4m3_value(static_cast<uint32_t>(c));
    tab[c] = (S == 0.0f) ? 0.0f : fminf(__fdiv_rn(s_enc, S), 3.402823466e+38f);
  }
}

// ---------------------------------------------------------------------------
// E8M0 shared exponent (MXFP4)
// ---------------------------------------------------------------------------

// Unbiased exponent e in [-127, 127] of the power-of-two scale of a block
// whose maximum magnitude is m.  Modes as in fp4q_e8m0_mode.
__device__ __forceinline__ int e8m0_exponent(float m, int mode) {
  if (!(m > 0.0f)) return -127;
  int e;
  if (mode == FP4Q_E8M0_OCP_FLOOR) {
    uint32_t b = __float_as_uint(m);
    int E = static_cast<int>(b >> 23) - 127;
    if ((b >> 23) == 0) E = -127 - (__clz(static_cast<int>(b)) - 9);  // subnormal
    e = E - 2;
  } else {
    float t = m >= 2.4e-37f ? div6(m) : __fdiv_rn(m, 6.0f);
    if (!(t > 0.0f)) return -127;
    uint32_t b = __float_as_uint(t);
    int E;
    uint32_t frac;  // fraction bits below the leading one, left-aligned to 23 bits
    if ((b >> 23) != 0) {
      E = static_cast<int>(b >> 23) - 127;
      frac = b & 0x7FFFFFu;
    } else {  // subnormal: b = mant * 2^-149, leading one at bit p
      int p = 31 - __clz(static_cast<int>(b));
      E = p - 149;
      frac = (b << (23 - p)) & 0x7FFFFFu;
    }
    if (mode == FP4Q_E8M0_CEIL) {
      e = (frac != 0) ? E + 1 : E;
    } else {  // nearest power of two; midpoint 1.5 * 2^E -> even biased exponent
      if (frac > 0x400000u) e = E + 1;
      else if (frac < 0x400000u) e = E;
      else e = (((E + 127) & 1) == 0) ? E : E + 1;
    }
  }
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// The exponent for an element format whose largest magnitude is qmax =
// 1.x * 2^emax (MXFP6: 7.5 = 1.875 * 2^2 for E2M3, 28 = 1.75 * 2^4 for E3M2):
// OCP floor(log2 m) - emax, or RN(m / qmax) rounded up (CEIL) or to the
// nearest power of two with ties to the even biased exponent (RNE).
__device__ __forceinline__ int e8m0_exponent_q(float m, int mode, float qmax, float inv_qmax,
                                               int emax) {
  if (!(m > 0.0f)) return -127;
  int e;
  if (mode == FP4Q_E8M0_OCP_FLOOR) {
    uint32_t b = __float_as_uint(m);
    int E = static_cast<int>(b >> 23) - 127;
    if ((b >> 23) == 0) E = -127 - (__clz(static_cast<int>(b)) - 9);  // subnormal
    e = E - emax;
  } else {
    const float t = div_qmax(m, qmax, inv_qmax);
    if (!(t > 0.0f)) return -127;
    uint32_t b = __float_as_uint(t);
    int E;
    uint32_t frac;
    if ((b >> 23) != 0) {
      E = static_cast<int>(b >> 23) - 127;
      frac = b & 0x7FFFFFu;
    } else {
      int p = 31 - __clz(static_cast<int>(b));
      E = p - 149;
      frac = (b << (23 - p)) & 0x7FFFFFu;
    }
    if (mode == FP4Q_E8M0_CEIL) {
      e = (frac != 0) ? E + 1 : E;
    } else {
      if (frac > 0x400000u) e = E + 1;
      else if (frac < 0x400000u) e = E;
      else e = (((E + 127) & 1) == 0) ? E : E + 1;
    }
  }
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// Biased E8M0 exponent (e + 127, clamped to [0, 254]) of a block with
// maximum m, as e8m0_exponent, with the common case -- a normal quotient
// RN(m/6) -- done by carries on the bit pattern: adding 0x3FFFFF plus the
// exponent's parity bit rounds to the nearest power of two with ties to the
// even exponent (RNE mode); adding 0x7FFFFF rounds up (CEIL mode).
__device__ __forceinline__ uint32_t e8m0_biased(float m, int mode) {
  if (mode == FP4Q_E8M0_OCP_FLOOR || !(m >= 7.1e-38f))   // OCP rule, or a subnormal quotient
    return static_cast<uint32_t>(e8m0_exponent(m, mode) + 127);
  const uint32_t b = __float_as_uint(div6(m));
  const uint32_t add = mode == FP4Q_E8M0_CEIL ? 0x7FFFFFu : 0x3FFFFFu + ((b >> 23) & 1u);
  return min((b + add) >> 23, 254u);
}

// 2^-(byte - 127) as a float for a biased E8M0 exponent byte.
__device__ __forceinline__ float e8m0_inverse(uint32_t byte) {
  return byte == 254u ? __uint_as_float(0x00400000u) : __uint_as_float((254u - byte) << 23);
}

// 2^e as a float for a stored E8M0 byte (e = byte - 127, e <= 127).
__device__ __forceinline__ float e8m0_value(uint32_t byte) {
  if (byte == 0) return __uint_as_float(0x00400000u);
  return __uint_as_float(byte << 23);
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., SC'11) and stochastic rounding
// ---------------------------------------------------------------------------

struct U32x4 { uint32_t x, y, z, w; };

// ---------------------------------------------------------------------------
// scale-factor layouts
// ---------------------------------------------------------------------------

// Byte offset of scale (r, c) in an [rows, cols] scale matrix.
__device__ __forceinline__ int64_t scale_offset(int64_t r, int64_t c, int64_t cols,
                                                int layout) {
  if (layout == FP4Q_SCALE_LINEAR) return r * cols + c;
  int64_t tile = (r >> 7) * (cols >> 2) + (c >> 2);
  return tile * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

// ---------------------------------------------------------------------------
// misc
// ---------------------------------------------------------------------------

// ---------------------------------------------------------------------------
// one block of N contiguous BF16 or FP32 values (16-byte aligned) to FP32
// ---------------------------------------------------------------------------

template <int N, typename T>
__device__ __forceinline__ void load_values(const T *p, float (&v)[N]) {
  const uint4 *q = reinterpret_cast<const uint4 *>(p);
  if (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < N / 8; ++i) {
      const uint4 u = __ldg(q + i);
      v[8 * i + 0] = bf16_lo(u.x); v[8 * i + 1] = bf16_hi(u.x);
      v[8 * i + 2] = bf16_lo(u.y); v[8 * i + 3] = bf16_hi(u.y);
      v[8 * i + 4] = bf16_lo(u.z); v[8 * i + 5] = bf16_hi(u.z);
      v[8 * i + 6] = bf16_lo(u.w); v[8 * i + 7] = bf16_hi(u.w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const uint4 u = __ldg(q + i);
      v[4 * i + 0] = __uint_as_float(u.x); v[4 * i + 1] = __uint_as_float(u.y);
      v[4 * i + 2] = __uint_as_float(u.z); v[4 * i + 3] = __uint_as_float(u.w);
    }
  }
}

// ---------------------------------------------------------------------------
// packed arithmetic (sm_100a f32x2 and bf16x2)
// ---------------------------------------------------------------------------

// (a.x * b.x, a.y * b.y), each rounded to nearest even
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;\n\t}"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;\n\t}"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;\n\t}"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
// (fma(a.x, b.x, c.x), fma(a.y, b.y, c.y)), single rounding each
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}

// The E4M3 codes of two block scales at once: the same correctly rounded
// steps as nvfp4_scale_code lane by lane (RN(m * s_enc), then Markstein's
// division by 6) as f32x2 operations, and one conversion for both codes:
// code of a in bits 0..7, of b in bits 8..15.
__device__ __forceinline__ uint32_t nvfp4_scale_code2(float a, float b, float s_enc) {
  constexpr float kInv6 = 1.0f / 6.0f;
  const float2 y = mul2(make_float2(a, b), make_float2(s_enc, s_enc));
  const float2 q0 = mul2(y, make_float2(kInv6, kInv6));
  const float2 r = fma2(q0, make_float2(-6.0f, -6.0f), y);
  const float2 q = fma2(r, make_float2(kInv6, kInv6), q0);
  uint16_t c;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(q.y), "f"(q.x));
  return c;
}

// per 16-bit lane: max(|a|, |b|) of two BF16 pairs (the sign bits of the
// result are meaningless; mask with 0x7FFF7FFF)
__device__ __forceinline__ uint32_t maxabs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// the larger magnitude of the two BF16 lanes of a max.xorsign.abs result,
// as an FP32 value
__device__ __forceinline__ float bf16x2_hmax(uint32_t m) {
  m &= 0x7FFF7FFFu;
  return __uint_as_float(max(m << 16, m & 0xFFFF0000u));
}

// |x| max over 8 BF16 in a uint4 -> FP32
__device__ __forceinline__ float absmax8(uint4 u) {
  return bf16x2_hmax(maxabs_bf16x2(maxabs_bf16x2(u.x, u.y), maxabs_bf16x2(u.z, u.w)));
}

// Stochastic rounding of v onto the E2M1 grid by scaling (the oracle's rule:
// the magnitude goes up iff u < t * 2^16, with u the 16-bit uniform and t the
// position of |v| between its two grid neighbours).  w = |v| * 2^-126 maps
// the whole grid onto float bit patterns that keep the top 2^22 ulps of the
// low bits: [1, 8) onto normal binades with one mantissa bit kept, [0, 1)
// onto the subnormals, whose uniform step makes E2M1's 0.5 spacing 2^22 steps
// too.  Adding 0x3FFFFF - 64 u to the bits of w therefore carries into the
// kept bit exactly when 64 u < frac, with no test of the range; rounding the
// product up keeps that comparison exact where the scaling drops low bits of
// |v| < 1.  The sign of v is put back and the value multiplied by 2^126
// (exact).  The bits below the kept one are not cleared here: the truncating
// conversion (e2m1x8_rz, e2m1x4_rz) drops them, and maps 8 and above to 6.
// The values the kernels pass stay below about 6.5 (the factor is s_enc / S
// for the block's own rounded scale S), but unmasked an infinite |v| would
// become a NaN pattern, so the scaled product saturates at 1 (mul.rp.sat, at
// no cost): any |v| >= 2^126 lands in [1, 1.5) * 2^126, which the conversion
// saturates to 6 as the oracle does.  Checked against the oracle by
// tests/sr_check.c, method 3, infinity included.  x64 = 64 u (sr_x_lo /
// sr_x_hi).
__device__ __forceinline__ uint32_t sr_dither_bits(float v, uint32_t x64) {
  float w;
  asm("mul.rp.sat.f32 %0, %1, %2;" : "=f"(w) : "f"(fabsf(v)), "f"(0x1p-126f));
  return (__float_as_uint(w) + 0x3FFFFFu - x64) | (__float_as_uint(v) & 0x80000000u);
}
// two values at once; the final exact scaling is one f32x2 product
__device__ __forceinline__ float2 e2m1_sr_dithered2(float2 v, uint32_t xa, uint32_t xb) {
  return mul2(make_float2(__uint_as_float(sr_dither_bits(v.x, xa)),
                          __uint_as_float(sr_dither_bits(v.y, xb))),
              make_float2(0x1p126f, 0x1p126f));
}
// 64 u of the low / high 16-bit uniform of a 32-bit word
__device__ __forceinline__ uint32_t sr_x_lo(uint32_t w) { return (w << 6) & 0x3FFFC0u; }
__device__ __forceinline__ uint32_t sr_x_hi(uint32_t w) { return (w >> 10) & 0x3FFFC0u; }

// max(|a|, |b|, |c|) in one three-input maximum (inputs finite)
__device__ __forceinline__ float absmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(fabsf(a)), "f"(fabsf(b)), "f"(fabsf(c)));
  return r;
}
// max over |v[0..N)|, N >= 3 odd or even
template <int N>
__device__ __forceinline__ float absmax_n(const float (&v)[N]) {
  float m = absmax3(v[0], v[1], v[2]);
#pragma unroll
  for (int i = 3; i + 1 < N; i += 2) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(m), "f"(fabsf(v[i])), "f"(fabsf(v[i + 1])));
    m = r;
  }
  if ((N - 3) % 2 == 1) m = fmaxf(m, fabsf(v[N - 1]));
  return m;
}

// Philox4x32-10 with the round keys held by the caller (they depend only on
// the seed).
struct PhiloxKey {
  uint32_t k0[10], k1[10];
  __device__ __forceinline__ explicit PhiloxKey(uint64_t seed) {
    uint32_t a = static_cast<uint32_t>(seed), b = static_cast<uint32_t>(seed >> 32);
#pragma unroll
    for (int i = 0; i < 10; ++i) {
      k0[i] = a;
      k1[i] = b;
      a += 0x9E3779B9u;
      b += 0xBB67AE85u;
    }
  }
};

__device__ __forceinline__ U32x4 philox(const PhiloxKey &K, uint32_t c0, uint32_t c1,
                                        uint32_t c2, uint32_t c3) {
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c0;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c2;
    const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ K.k0[i];
    const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ K.k1[i];
    c1 = static_cast<uint32_t>(p1);
    c3 = static_cast<uint32_t>(p0);
    c0 = n0;
    c2 = n2;
  }
  return U32x4{c0, c1, c2, c3};
}

// ---------------------------------------------------------------------------
// cp.async staging (16-byte global -> shared copies, grouped per thread)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Coordinates (tile row tt, tile column tc) of a linear tile index over a
// grid of tiles_c tile columns, stepped by a fixed number of tiles without
// dividing.  I is the index type: int32_t where the launcher has checked that
// every index fits, int64_t otherwise.
template <typename I>
struct TileCursorT {
  I tile, tt, tc;
  __device__ __forceinline__ void init(I t, I tiles_c) {
    tile = t;
    tt = t / tiles_c;
    tc = t - tt * tiles_c;
  }
  __device__ __forceinline__ void advance(I step, I dtt, I dtc, I tiles_c) {
    tile += step;
    tt += dtt;
    tc += dtc;
    if (tc >= tiles_c) {
      tc -= tiles_c;
      ++tt;
    }
  }
};
using TileCursor = TileCursorT<int64_t>;

// scale_offset in the index type I
template <typename I>
__device__ __forceinline__ I scale_offset_t(I r, I c, I cols, int layout) {
  if (layout == FP4Q_SCALE_LINEAR) return r * cols + c;
  const I tile = (r >> 7) * (cols >> 2) + (c >> 2);
  return tile * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

}  // namespace fp4q
