// if6.cu -- IF6: the IF per-block choice at 6 bits, quantize and dequantize.
//
// "Adaptive Block-Scaled Data Types" explainer, section 2: each 16-value
// block is quantized both to a float grid and to a scaled integer grid, the
// one with the smaller squared error is kept, and the scale's sign bit says
// which; the idea extends to 6 bits (IF6).  Read here with FP6 E2M3 (largest
// 7.5, the finer FP6 grid of "FP6で隣り合う値の間隔を見てみる") against INT6
// (-31..31) rescaled by 7.5/31 (the 6/7 method with 31 and 7.5):
//
//   s_enc = RN(3360 / amax), s_dec = RN(amax / 3360)        (3360 = 7.5 * 448)
//   S = E4M3_rne_sat(RN(RN(m * s_enc) / 7.5)),  r = RN(s_enc / S),  v = RN(x * r)
//   FP6:  g = E2M3(v) (round to nearest even, saturating, sign copied)
//   INT6: k = clamp(rint(RN(v * RN(31/7.5))), -31, 31),  h = RN(k * RN(7.5/31))
//   e = sum over the block, in order, of fma(d, d, e) with d = RN(v - q)
//   INT6 iff e_int < e_fp; scale bit 7 flags INT6.
//
// Codes are 6 bits (the E2M3 code, or k in two's complement), four per three
// bytes (code j of a group in bits 6j..6j+5), so a block is 12 bytes.
// Quantize: one thread per block, 32 or 64 bytes in, three 4-byte code stores
// and a scale byte out; r comes from a per-CTA table over the 128 scale codes.
// Exact shortcuts (as in IF4): rint by adding and subtracting 1.5 * 2^23, whose
// bits also carry the INT6 code, packed by multiply-add; FP6 errors by a
// mixed-precision subtract from the decoded f16 grid values.
// Dequantize: one thread per block, y = RN(RN(q * S) * s_dec) with q the E2M3
// value or h.
#include <cuda_fp16.h>

#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;
constexpr float kTop = 7.5f * 448.0f;             // 3360
constexpr float kUp = 31.0f / 7.5f;               // RN(31/7.5)
constexpr float kDown = 7.5f / 31.0f;             // RN(7.5/31)

__device__ __forceinline__ float2 e2m3x2_value(uint32_t two_codes) {
  uint32_t h;
  const uint16_t w = static_cast<uint16_t>(two_codes);
  asm("cvt.rn.f16x2.e2m3x2 %0, %1;" : "=r"(h) : "h"(w));
  __half2 v;
  memcpy(&v, &h, sizeof(v));
  return __half22float2(v);
}

constexpr float kMagic = 12582912.0f;             // 1.5 * 2^23: RN(t + kMagic) - kMagic = rint(t)
// bits(RN(t + kMagic)) = 0x4B400000 + rint(t); four such words summed with
// weights 64^i, minus this, give sum of (rint(t_i) + 32) 64^i
constexpr uint32_t kGroupBias = (0x4B400000u - 32u) * (1u + 64u + 4096u + 262144u);

// Four values to FP6 E2M3 codes (one per byte, value order) and the
// differences d = RN(g - v) from their grid values g (exact in f16; the
// square equals that of RN(v - g)), subtracted in mixed precision.
__device__ __forceinline__ uint32_t e2m3x4_codes_diffs(const float (&v)[4], float (&d)[4]) {
  uint32_t w;
  asm("{\n\t.reg .b16 p0, p1;\n\t.reg .b32 h0, h1;\n\t.reg .f16 g0, g1, g2, g3;\n\t"
      "cvt.rn.satfinite.e2m3x2.f32 p0, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m3x2.f32 p1, %8, %7;\n\t"
      "and.b16 p0, p0, 0x3F3F;\n\t"
      "and.b16 p1, p1, 0x3F3F;\n\t"
      "mov.b32 %0, {p0, p1};\n\t"
      "cvt.rn.f16x2.e2m3x2 h0, p0;\n\t"
      "cvt.rn.f16x2.e2m3x2 h1, p1;\n\t"
      "mov.b32 {g0, g1}, h0;\n\t"
      "mov.b32 {g2, g3}, h1;\n\t"
      "sub.rn.f32.f16 %1, g0, %5;\n\t"
      "sub.rn.f32.f16 %2, g1, %6;\n\t"
      "sub.rn.f32.f16 %3, g2, %7;\n\t"
      "sub.rn.f32.f16 %4, g3, %8;\n\t}"
      : "=r"(w), "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]));
  return w;
}

template <typename T, typename I>
__global__ void __launch_bounds__(kThreads)
if6_kernel(const T *__restrict__ x, I rows, I cols, I ld, const float *__restrict__ amax,
           float *__restrict__ s_dec_out, uint8_t *__restrict__ q, uint8_t *__restrict__ sf,
           int scale_layout) {
  __shared__ float tab[128];
  const float a = *amax;
  const float s_enc = a == 0.0f ? 1.0f : fminf(__fdiv_rn(kTop, a), 3.402823466e+38f);
  if (blockIdx.x == 0 && threadIdx.x == 0 && s_dec_out)
    *s_dec_out = a == 0.0f ? 1.0f : __fdiv_rn(a, kTop);
  fill_factor_table(tab, s_enc);
  __syncthreads();
  const I bpr = cols / 16, nblk = rows * bpr;
  const I stride = static_cast<I>(gridDim.x) * kThreads;
  for (I b = static_cast<I>(blockIdx.x) * kThreads + threadIdx.x; b < nblk; b += stride) {
    const I r = b / bpr, cb = b - r * bpr;
    float v[16];
    load_values<16, T>(x + r * ld + cb * 16, v);
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < 16; ++k) m = fmaxf(m, fabsf(v[k]));
    const uint32_t code = e4m3_code(div_qmax(__fmul_rn(m, s_enc), 7.5f, 1.0f / 7.5f));
    const float rf = tab[code];
    // |t| <= RN(RN(m * r) * RN(31/7.5)) by monotonicity; only a block reaching
    // 31.25 needs the clamp (which then makes rint land on +-31, as clamping
    // rint(t) to +-31 does)
    const bool clamp = __fmul_rn(__fmul_rn(m, rf), kUp) > 31.25f;
    float e_fp = 0.0f, e_int = 0.0f;
    uint32_t fp_group[4], int_group[4];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {                   // groups of four elements
      float vv[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) vv[h] = __fmul_rn(v[4 * q4 + h], rf);
      float d[4];
      const uint32_t w = e2m3x4_codes_diffs(vv, d);     // codes as bytes; d = RN(g - v)
#pragma unroll
      for (int h = 0; h < 4; ++h) e_fp = __fmaf_rn(d[h], d[h], e_fp);
      fp_group[q4] = (w & 0x3Fu) | ((w >> 2) & 0xFC0u) | ((w >> 4) & 0x3F000u) |
                     ((w >> 6) & 0xFC0000u);
      uint32_t tb[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {                    // element order, as the errors sum
        float t = __fmul_rn(vv[h], kUp);
        if (clamp) t = fminf(fmaxf(t, -31.25f), 31.25f);
        const float tm = __fadd_rn(t, kMagic);         // rint(t) in the low bits
        const float kf = __fsub_rn(tm, kMagic);        // exact
        const float dint = __fsub_rn(vv[h], __fmul_rn(kf, kDown));
        e_int = __fmaf_rn(dint, dint, e_int);
        tb[h] = __float_as_uint(tm);
      }
      const uint32_t acc = ((tb[3] * 64u + tb[2]) * 64u + tb[1]) * 64u + tb[0];
      // sum of (k + 32) 64^i, then bit 5 of each field flipped: k in two's complement
      int_group[q4] = (acc - kGroupBias) ^ 0x820820u;
    }
    const bool use_int = e_int < e_fp;
    uint32_t g[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) g[t] = use_int ? int_group[t] : fp_group[t];
    uint32_t *dst = reinterpret_cast<uint32_t *>(q + b * 12);   // codes are dense, 12 B per block
    dst[0] = g[0] | g[1] << 24;
    dst[1] = g[1] >> 8 | g[2] << 16;
    dst[2] = g[2] >> 16 | g[3] << 8;
    sf[scale_offset(r, cb, bpr, scale_layout)] = static_cast<uint8_t>(code | (use_int ? 0x80u : 0u));
  }
}

template <typename OutT, typename I>
__global__ void __launch_bounds__(kThreads)
if6_dequant_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ sf,
                   int scale_layout, const float *__restrict__ s_dec_ptr, I rows, I cols,
                   OutT *__restrict__ y) {
  const float s_dec = *s_dec_ptr;
  const I bpr = cols / 16, nblk = rows * bpr;
  const I stride = static_cast<I>(gridDim.x) * kThreads;
  for (I b = static_cast<I>(blockIdx.x) * kThreads + threadIdx.x; b < nblk; b += stride) {
    const I r = b / bpr, cb = b - r * bpr;
    const uint32_t *src = reinterpret_cast<const uint32_t *>(q + b * 12);
    const uint32_t w0 = __ldg(src), w1 = __ldg(src + 1), w2 = __ldg(src + 2);
    const uint32_t g[4] = {w0 & 0xFFFFFFu, (w0 >> 24 | w1 << 8) & 0xFFFFFFu,
                           (w1 >> 16 | w2 << 16) & 0xFFFFFFu, w2 >> 8};
    const uint32_t sb = __ldg(sf + scale_offset(r, cb, bpr, scale_layout));
    const float S = e4m3_value(sb & 0x7Fu);
    float out[16];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
#pragma unroll
      for (int h = 0; h < 4; h += 2) {
        const uint32_t c0 = (g[t] >> (6 * h)) & 0x3Fu, c1 = (g[t] >> (6 * h + 6)) & 0x3Fu;
        float q0, q1;
        if (sb & 0x80u) {                               // INT6: k in two's complement
          const int k0 = static_cast<int>(c0) - ((c0 & 0x20u) ? 64 : 0);
          const int k1 = static_cast<int>(c1) - ((c1 & 0x20u) ? 64 : 0);
          q0 = __fmul_rn(static_cast<float>(k0), kDown);
          q1 = __fmul_rn(static_cast<float>(k1), kDown);
        } else {
          const float2 v = e2m3x2_value(c0 | c1 << 8);
          q0 = v.x;
          q1 = v.y;
        }
        out[4 * t + h] = __fmul_rn(__fmul_rn(q0, S), s_dec);
        out[4 * t + h + 1] = __fmul_rn(__fmul_rn(q1, S), s_dec);
      }
    }
    OutT *o = y + b * 16;                               // the output is dense as well
    if (sizeof(OutT) == 2) {
      uint4 *d = reinterpret_cast<uint4 *>(o);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __nv_bfloat162 h2 = __floats2bfloat162_rn(out[8 * i + 2 * k], out[8 * i + 2 * k + 1]);
          memcpy(&w[k], &h2, sizeof(uint32_t));
        }
        d[i] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      float4 *d = reinterpret_cast<float4 *>(o);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        d[i] = make_float4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
    }
  }
}

int grid_for(int64_t nblk, const Launch &L) {
  const int64_t want = (nblk + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(L.num_sms) * 8;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

// 32-bit indices when every element offset, and every block index a
// grid-stride step can reach, stays below 2^31
bool narrow(int64_t rows, int64_t cols, int64_t ld, int grid) {
  return rows * (ld > cols ? ld : cols) + 16 * static_cast<int64_t>(grid) * kThreads <
         (int64_t{1} << 31);
}

template <typename T>
cudaError_t launch_q(const void *x, int64_t rows, int64_t cols, int64_t ld, const float *amax,
                     float *s_dec_out, uint8_t *q, uint8_t *sf, int scale_layout,
                     const Launch &L) {
  const int grid = grid_for(rows * (cols / 16), L);
  const T *p = static_cast<const T *>(x);
  if (narrow(rows, cols, ld, grid))
    if6_kernel<T, uint32_t><<<grid, kThreads, 0, L.stream>>>(
        p, static_cast<uint32_t>(rows), static_cast<uint32_t>(cols), static_cast<uint32_t>(ld),
        amax, s_dec_out, q, sf, scale_layout);
  else
    if6_kernel<T, int64_t><<<grid, kThreads, 0, L.stream>>>(p, rows, cols, ld, amax, s_dec_out, q,
                                                           sf, scale_layout);
  return cudaGetLastError();
}

template <typename OutT>
cudaError_t launch_dq(const uint8_t *q, const uint8_t *sf, int scale_layout, const float *s_dec,
                      int64_t rows, int64_t cols, void *y, const Launch &L) {
  const int grid = grid_for(rows * (cols / 16), L);
  OutT *o = static_cast<OutT *>(y);
  if (narrow(rows, cols, cols, grid))
    if6_dequant_kernel<OutT, uint32_t><<<grid, kThreads, 0, L.stream>>>(
        q, sf, scale_layout, s_dec, static_cast<uint32_t>(rows), static_cast<uint32_t>(cols), o);
  else
    if6_dequant_kernel<OutT, int64_t><<<grid, kThreads, 0, L.stream>>>(q, sf, scale_layout, s_dec,
                                                                      rows, cols, o);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_if6(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                       const float *amax, float *s_dec_out, uint8_t *q, uint8_t *sf,
                       int scale_layout, const Launch &L) {
  if (dtype == FP4Q_BF16)
    return launch_q<__nv_bfloat16>(x, rows, cols, ld, amax, s_dec_out, q, sf, scale_layout, L);
  return launch_q<float>(x, rows, cols, ld, amax, s_dec_out, q, sf, scale_layout, L);
}

cudaError_t launch_if6_dequant(const uint8_t *q, const uint8_t *sf, int scale_layout,
                               const float *s_dec, int64_t rows, int64_t cols, void *y,
                               int y_dtype, const Launch &L) {
  if (y_dtype == FP4Q_BF16)
    return launch_dq<__nv_bfloat16>(q, sf, scale_layout, s_dec, rows, cols, y, L);
  return launch_dq<float>(q, sf, scale_layout, s_dec, rows, cols, y, L);
}

}  // namespace fp4q
