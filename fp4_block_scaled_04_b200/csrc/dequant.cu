// dequant.cu -- block-scaled FP4 back to FP32 / BF16.
//
// Ultralytics glossary "FP4", "FP4の仕組み": the reconstructed value is the
// grid value times its sign times the block scale.  NVFP4 also multiplies by
// the per-tensor decode scale; IF4 INT4 blocks (scale bit 7) decode k * 6/7
// (the 6/7 method of the "Adaptive Block-Scaled Data Types" explainer).
//   NVFP4 / IF4-FP4:  y = RN(RN(g * S) * s_dec)
//   IF4-INT4:         y = RN(RN(RN(k * RN(6/7)) * S) * s_dec)
//   MXFP4:            y = g * 2^(byte - 127)
//
// The codes [rows, cols/2] and the output [rows, cols] are both dense, so the
// kernel walks the flat element range in units of E elements (one 16-byte
// output store: E = 8 for BF16, 4 for FP32), consecutive units on
// consecutive lanes: code loads and output stores are contiguous across the
// warp.  E2M1 pairs decode with cvt.rn.f16x2.e2m1x2; g * S is exact in f16
// (at most 6 significant bits, within [2^-10, 2688]) and is formed as an
// f16x2 product; the multiplication by s_dec is the one FP32 rounding.  INT4
// values are formed arithmetically: k = (2^23 + (nibble ^ 8)) - (2^23 + 8).
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t h2;
  asm("{\n\t.reg .b8 q;\n\t.reg .b16 w;\n\t"
      "cvt.u16.u32 w, %1;\n\t"
      "cvt.u8.u16 q, w;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, q;\n\t}"
      : "=r"(h2) : "r"(byte));
  return h2;
}

__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t h) {
  const __half2 v = *reinterpret_cast<const __half2 *>(&h);
  return __half22float2(v);
}

// the two values of one code byte (element 2i in the low nibble)
template <int FMT>
__device__ __forceinline__ float2 decode_pair(uint32_t byte, uint32_t sbyte, float s_dec,
                                              float c67) {
  if (FMT == FP4Q_FMT_MXFP4) {
    const float p = e8m0_value(sbyte);
    return mul2(f16x2_to_f32x2(e2m1x2_to_f16x2(byte)), make_float2(p, p));
  }
  const float S = e4m3_value(sbyte & 0x7Fu);
  if (FMT == FP4Q_FMT_IF4 && (sbyte & 0x80u)) {
    // k from the two's complement nibble, exactly: (2^23 + (n ^ 8)) - (2^23 + 8)
    const float k0 = __fsub_rn(__uint_as_float(0x4B000000u | ((byte & 0xFu) ^ 8u)), 8388616.0f);
    const float k1 = __fsub_rn(__uint_as_float(0x4B000000u | ((byte >> 4) ^ 8u)), 8388616.0f);
    const float2 h = mul2(make_float2(k0, k1), make_float2(c67, c67));
    return mul2(mul2(h, make_float2(S, S)), make_float2(s_dec, s_dec));
  }
  const __half hs = __float2half_rn(S);                  // exact: S is an E4M3 value
  const uint32_t s2 = static_cast<uint32_t>(__half_as_ushort(hs)) * 0x10001u;
  const uint32_t gs = hmul2_bits(e2m1x2_to_f16x2(byte), s2);
  return mul2(f16x2_to_f32x2(gs), make_float2(s_dec, s_dec));
}

template <int FMT, int BROWS, bool BF16_OUT>
__global__ void __launch_bounds__(kThreads)
dequant_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ sf, int scale_layout,
               const float *__restrict__ s_dec_ptr, int64_t rows, int64_t cols,
               void *__restrict__ y) {
  constexpr int E = BF16_OUT ? 8 : 4;                  // elements per unit
  constexpr int BLK = FMT == FP4Q_FMT_MXFP4 ? 32 : 16;
  const float s_dec = (FMT == FP4Q_FMT_MXFP4) ? 1.0f : *s_dec_ptr;
  const float c67 = __fdiv_rn(6.0f, 7.0f);
  const int64_t upr = cols / E;                        // units per row
  const int64_t total = rows * upr;
  const int64_t bpr = cols / BLK;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  int64_t u = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  if (u >= total) return;
  // (row, column) of the unit, advanced by a fixed stride each step
  int64_t r = u / upr, c = (u - r * upr) * E;
  const int64_t dr = stride / upr, dc = (stride - dr * upr) * E;
  for (; u < total; u += stride) {
    const uint32_t sbyte = (BROWS == 16) ? sf[(r / 16) * bpr + c / 16]
                                         : sf[scale_offset(r, c / BLK, bpr, scale_layout)];
    const int64_t e = r * cols + c;
    float v[E];
    if (E == 8) {
      const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(q + e / 2));
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 p = decode_pair<FMT>((w >> (8 * i)) & 0xFFu, sbyte, s_dec, c67);
        v[2 * i] = p.x;
        v[(2 * i + 1) % E] = p.y;
      }
    } else {
      const uint32_t w = __ldg(reinterpret_cast<const uint16_t *>(q + e / 2));
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 p = decode_pair<FMT>((w >> (8 * i)) & 0xFFu, sbyte, s_dec, c67);
        v[2 * i] = p.x;
        v[2 * i + 1] = p.y;
      }
    }
    if (BF16_OUT) {
      uint32_t p[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h2 = __floats2bfloat162_rn(v[(2 * i) % E], v[(2 * i + 1) % E]);
        p[i] = *reinterpret_cast<uint32_t *>(&h2);
      }
      *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(y) + e) = make_uint4(p[0], p[1], p[2], p[3]);
    } else {
      *reinterpret_cast<float4 *>(static_cast<float *>(y) + e) =
          make_float4(v[0], v[1], v[2 % E], v[3 % E]);
    }
    r += dr;
    c += dc;
    if (c >= cols) {
      c -= cols;
      ++r;
    }
  }
}

template <int FMT, int BROWS>
cudaError_t launch_fmt(const uint8_t *q, const uint8_t *sf, int scale_layout, const float *s_dec,
                       int64_t rows, int64_t cols, void *y, int y_dtype, const Launch &L) {
  const bool bf = y_dtype == FP4Q_BF16;
  const int64_t units = rows * (cols / (bf ? 8 : 4));
  int64_t want = (units + kThreads - 1) / kThreads;
  int64_t cap = static_cast<int64_t>(L.num_sms) * 8;
  int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
  if (bf)
    dequant_kernel<FMT, BROWS, true><<<grid, kThreads, 0, L.stream>>>(q, sf, scale_layout, s_dec,
                                                                     rows, cols, y);
  else
    dequant_kernel<FMT, BROWS, false><<<grid, kThreads, 0, L.stream>>>(q, sf, scale_layout, s_dec,
                                                                      rows, cols, y);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dequant(int format, const uint8_t *q, const uint8_t *sf, int scale_layout,
                           int block_rows, int block_cols, const float *s_dec, int64_t rows,
                           int64_t cols, void *y, int y_dtype, const Launch &L) {
  (void)block_cols;
  if (format == FP4Q_FMT_MXFP4)
    return launch_fmt<FP4Q_FMT_MXFP4, 1>(q, sf, scale_layout, s_dec, rows, cols, y, y_dtype, L);
  if (format == FP4Q_FMT_IF4)
    return launch_fmt<FP4Q_FMT_IF4, 1>(q, sf, scale_layout, s_dec, rows, cols, y, y_dtype, L);
  if (block_rows == 16)
    return launch_fmt<FP4Q_FMT_NVFP4, 16>(q, sf, scale_layout, s_dec, rows, cols, y, y_dtype, L);
  return launch_fmt<FP4Q_FMT_NVFP4, 1>(q, sf, scale_layout, s_dec, rows, cols, y, y_dtype, L);
}

}  // namespace fp4q
