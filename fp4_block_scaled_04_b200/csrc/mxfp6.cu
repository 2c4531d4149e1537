// mxfp6.cu -- MXFP6 (OCP FP6 E2M3 / E3M2 with E8M0 block scales), quantize
// and dequantize.
//
// "FP6から考えるLLM量子化" (blog.ast.moe), "FP6で隣り合う値の間隔を見てみる":
// E3M2 spends its bits on range (largest 28), E2M3 on spacing (largest 7.5);
// 32 values share one power-of-two (E8M0) scale as in MXFP4.  Elements
// v = RN(x * 2^-e) are rounded to nearest even with saturation by the sm_100a
// conversion cvt.rn.satfinite.{e2m3x2,e3m2x2}.f32, which leaves each 6-bit code
// in the low bits of a byte.  Four codes are packed into three bytes, code j
// of a group in bits 6j..6j+5 of the little-endian 24-bit word, so a block of
// 32 values is 24 code bytes.
//
// One thread per block: 32 values in (64 or 128 bytes), one scale byte and
// three 8-byte stores out.  Decoding unpacks the 24-bit groups back into byte
// containers and converts pairs with cvt.rn.f16x2.{e2m3x2,e3m2x2} (every FP6
// value is exact in f16), then multiplies by 2^e.
#include <cuda_fp16.h>

#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;

// two values -> two 6-bit codes in the low bits of bytes 0 and 1 (lo first)
template <int F6>
__device__ __forceinline__ uint32_t fp6x2(float lo, float hi) {
  uint16_t r;
  if (F6 == FP4Q_FP6_E2M3)
    asm("cvt.rn.satfinite.e2m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  else
    asm("cvt.rn.satfinite.e3m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// two byte containers (code 0 in byte 0) -> the two values in f16x2
template <int F6>
__device__ __forceinline__ uint32_t fp6x2_to_f16x2(uint32_t two_bytes) {
  uint32_t h;
  const uint16_t w = static_cast<uint16_t>(two_bytes);
  if (F6 == FP4Q_FP6_E2M3)
    asm("cvt.rn.f16x2.e2m3x2 %0, %1;" : "=r"(h) : "h"(w));
  else
    asm("cvt.rn.f16x2.e3m2x2 %0, %1;" : "=r"(h) : "h"(w));
  return h;
}

__device__ __forceinline__ float2 half2_bits_to_f32x2(uint32_t h) {
  __half2 v;
  memcpy(&v, &h, sizeof(v));
  return __half22float2(v);
}

template <typename T>
__device__ __forceinline__ void load32(const T *p, float (&v)[32]) {
  const uint4 *q = reinterpret_cast<const uint4 *>(p);
  if (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 u = __ldg(q + i);
      v[8 * i + 0] = bf16_lo(u.x); v[8 * i + 1] = bf16_hi(u.x);
      v[8 * i + 2] = bf16_lo(u.y); v[8 * i + 3] = bf16_hi(u.y);
      v[8 * i + 4] = bf16_lo(u.z); v[8 * i + 5] = bf16_hi(u.z);
      v[8 * i + 6] = bf16_lo(u.w); v[8 * i + 7] = bf16_hi(u.w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 u = __ldg(q + i);
      v[4 * i + 0] = __uint_as_float(u.x); v[4 * i + 1] = __uint_as_float(u.y);
      v[4 * i + 2] = __uint_as_float(u.z); v[4 * i + 3] = __uint_as_float(u.w);
    }
  }
}

template <typename T, int F6>
__global__ void __launch_bounds__(kThreads)
mxfp6_kernel(const T *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, int mode,
             uint8_t *__restrict__ q, uint8_t *__restrict__ sf, int scale_layout) {
  const float qmax = F6 == FP4Q_FP6_E2M3 ? 7.5f : 28.0f;
  const int emax = F6 == FP4Q_FP6_E2M3 ? 2 : 4;
  const int64_t bpr = cols / 32, nblk = rows * bpr, rb = cols * 3 / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; b < nblk;
       b += stride) {
    const int64_t r = b / bpr, cb = b - r * bpr;
    float v[32];
    load32<T>(x + r * ld + cb * 32, v);
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < 32; ++k) m = fmaxf(m, fabsf(v[k]));
    const uint32_t byte = static_cast<uint32_t>(e8m0_exponent_q(m, mode, qmax, emax) + 127);
    const float inv = e8m0_inverse(byte);
    uint32_t g[8];                                     // 24-bit groups
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 a = mul2(make_float2(v[4 * j], v[4 * j + 1]), make_float2(inv, inv));
      const float2 c = mul2(make_float2(v[4 * j + 2], v[4 * j + 3]), make_float2(inv, inv));
      const uint32_t p01 = fp6x2<F6>(a.x, a.y), p23 = fp6x2<F6>(c.x, c.y);
      g[j] = (p01 & 0x3Fu) | ((p01 >> 8) & 0x3Fu) << 6 | (p23 & 0x3Fu) << 12 |
             ((p23 >> 8) & 0x3Fu) << 18;
    }
    uint2 *dst = reinterpret_cast<uint2 *>(q + r * rb + cb * 24);
    dst[0] = make_uint2(g[0] | g[1] << 24, g[1] >> 8 | g[2] << 16);
    dst[1] = make_uint2(g[2] >> 16 | g[3] << 8, g[4] | g[5] << 24);
    dst[2] = make_uint2(g[5] >> 8 | g[6] << 16, g[6] >> 16 | g[7] << 8);
    sf[scale_offset(r, cb, bpr, scale_layout)] = static_cast<uint8_t>(byte);
  }
}

template <typename OutT, int F6>
__global__ void __launch_bounds__(kThreads)
mxfp6_dequant_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ sf,
                     int scale_layout, int64_t rows, int64_t cols, OutT *__restrict__ y) {
  const int64_t bpr = cols / 32, nblk = rows * bpr, rb = cols * 3 / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; b < nblk;
       b += stride) {
    const int64_t r = b / bpr, cb = b - r * bpr;
    const uint2 *src = reinterpret_cast<const uint2 *>(q + r * rb + cb * 24);
    const uint2 w0 = __ldg(src), w1 = __ldg(src + 1), w2 = __ldg(src + 2);
    const uint32_t g[8] = {w0.x & 0xFFFFFFu, (w0.x >> 24 | w0.y << 8) & 0xFFFFFFu,
                           (w0.y >> 16 | w1.x << 16) & 0xFFFFFFu, w1.x >> 8,
                           w1.y & 0xFFFFFFu, (w1.y >> 24 | w2.x << 8) & 0xFFFFFFu,
                           (w2.x >> 16 | w2.y << 16) & 0xFFFFFFu, w2.y >> 8};
    const float p = e8m0_value(__ldg(sf + scale_offset(r, cb, bpr, scale_layout)));
    float out[32];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      // codes 0, 1 -> bytes 0, 1 of one container; codes 2, 3 of the other
      const uint32_t c01 = (g[j] & 0x3Fu) | ((g[j] >> 6) & 0x3Fu) << 8;
      const uint32_t c23 = ((g[j] >> 12) & 0x3Fu) | ((g[j] >> 18) & 0x3Fu) << 8;
      const float2 a = mul2(half2_bits_to_f32x2(fp6x2_to_f16x2<F6>(c01)), make_float2(p, p));
      const float2 c = mul2(half2_bits_to_f32x2(fp6x2_to_f16x2<F6>(c23)), make_float2(p, p));
      out[4 * j] = a.x; out[4 * j + 1] = a.y; out[4 * j + 2] = c.x; out[4 * j + 3] = c.y;
    }
    OutT *o = y + r * cols + cb * 32;
    if (sizeof(OutT) == 2) {
      uint4 *d = reinterpret_cast<uint4 *>(o);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __nv_bfloat162 h = __floats2bfloat162_rn(out[8 * i + 2 * k], out[8 * i + 2 * k + 1]);
          w[k] = *reinterpret_cast<uint32_t *>(&h);
        }
        d[i] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      float4 *d = reinterpret_cast<float4 *>(o);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        d[i] = make_float4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
    }
  }
}

int grid_for(int64_t nblk, const Launch &L) {
  const int64_t want = (nblk + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(L.num_sms) * 8;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

template <typename T>
cudaError_t launch_q(const void *x, int64_t rows, int64_t cols, int64_t ld, int fmt, int mode,
                     uint8_t *q, uint8_t *sf, int scale_layout, const Launch &L) {
  const int grid = grid_for(rows * (cols / 32), L);
  const T *p = static_cast<const T *>(x);
  if (fmt == FP4Q_FP6_E2M3)
    mxfp6_kernel<T, FP4Q_FP6_E2M3><<<grid, kThreads, 0, L.stream>>>(p, rows, cols, ld, mode, q,
                                                                      sf, scale_layout);
  else
    mxfp6_kernel<T, FP4Q_FP6_E3M2><<<grid, kThreads, 0, L.stream>>>(p, rows, cols, ld, mode, q,
                                                                      sf, scale_layout);
  return cudaGetLastError();
}

template <typename OutT>
cudaError_t launch_dq(const uint8_t *q, const uint8_t *sf, int scale_layout, int64_t rows,
                      int64_t cols, int fmt, void *y, const Launch &L) {
  const int grid = grid_for(rows * (cols / 32), L);
  OutT *o = static_cast<OutT *>(y);
  if (fmt == FP4Q_FP6_E2M3)
    mxfp6_dequant_kernel<OutT, FP4Q_FP6_E2M3><<<grid, kThreads, 0, L.stream>>>(q, sf, scale_layout,
                                                                               rows, cols, o);
  else
    mxfp6_dequant_kernel<OutT, FP4Q_FP6_E3M2><<<grid, kThreads, 0, L.stream>>>(q, sf, scale_layout,
                                                                               rows, cols, o);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mxfp6(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                         int fp6_format, int e8m0_mode, uint8_t *q, uint8_t *sf,
                         int scale_layout, const Launch &L) {
  if (dtype == FP4Q_BF16)
    return launch_q<__nv_bfloat16>(x, rows, cols, ld, fp6_format, e8m0_mode, q, sf, scale_layout,
                                   L);
  return launch_q<float>(x, rows, cols, ld, fp6_format, e8m0_mode, q, sf, scale_layout, L);
}

cudaError_t launch_mxfp6_dequant(const uint8_t *q, const uint8_t *sf, int scale_layout,
                                 int64_t rows, int64_t cols, int fp6_format, void *y,
                                 int y_dtype, const Launch &L) {
  if (y_dtype == FP4Q_BF16)
    return launch_dq<__nv_bfloat16>(q, sf, scale_layout, rows, cols, fp6_format, y, L);
  return launch_dq<float>(q, sf, scale_layout, rows, cols, fp6_format, y, L);
}

}  // namespace fp4q
