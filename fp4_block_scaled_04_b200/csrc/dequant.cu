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
// Two blocks per thread.  E2M1 pairs decode with cvt.rn.f16x2.e2m1x2; the
// product g * S is exact in f16 (at most 6 significant bits, within
// [2^-10, 2688]), so it is formed as an f16x2 product and widened; the
// multiplication by s_dec is the one FP32 rounding.  INT4 values come from a
// 16-entry table of RN(k * RN(6/7)).
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

// 16 codes (two words) of one block -> 16 FP32 values
template <int FMT>
__device__ __forceinline__ void decode16(uint32_t w0, uint32_t w1, uint32_t sbyte, float s_dec,
                                         const float *itab, float (&y)[16]) {
  const uint32_t w[2] = {w0, w1};
  if (FMT == FP4Q_FMT_MXFP4) {
    const float p = e8m0_value(sbyte);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 g = f16x2_to_f32x2(e2m1x2_to_f16x2((w[i >> 2] >> (8 * (i & 3))) & 0xFFu));
      const float2 v = mul2(g, make_float2(p, p));
      y[2 * i] = v.x;
      y[2 * i + 1] = v.y;
    }
  } else if (FMT == FP4Q_FMT_IF4 && (sbyte & 0x80u)) {
    const float S = e4m3_value(sbyte & 0x7Fu);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t byte = (w[i >> 2] >> (8 * (i & 3))) & 0xFFu;
      const float2 h = make_float2(itab[byte & 0xFu], itab[byte >> 4]);
      const float2 v = mul2(mul2(h, make_float2(S, S)), make_float2(s_dec, s_dec));
      y[2 * i] = v.x;
      y[2 * i + 1] = v.y;
    }
  } else {
    const float S = e4m3_value(sbyte & 0x7Fu);
    const __half hs = __float2half_rn(S);                  // exact: S is an E4M3 value
    const uint32_t s2 = static_cast<uint32_t>(__half_as_ushort(hs)) * 0x10001u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t gs = hmul2_bits(e2m1x2_to_f16x2((w[i >> 2] >> (8 * (i & 3))) & 0xFFu), s2);
      const float2 v = mul2(f16x2_to_f32x2(gs), make_float2(s_dec, s_dec));
      y[2 * i] = v.x;
      y[2 * i + 1] = v.y;
    }
  }
}

template <bool BF16_OUT>
__device__ __forceinline__ void store16(void *y, int64_t off, const float (&v)[16]) {
  if (BF16_OUT) {
    uint32_t p[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      p[i] = *reinterpret_cast<uint32_t *>(&h2);
    }
    uint4 *d = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(y) + off);
    d[0] = make_uint4(p[0], p[1], p[2], p[3]);
    d[1] = make_uint4(p[4], p[5], p[6], p[7]);
  } else {
    float4 *d = reinterpret_cast<float4 *>(static_cast<float *>(y) + off);
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

// One work unit = 16 consecutive codes of a row (one NVFP4/IF4 block or half an
// MXFP4 block) plus the next 16; a thread handles one unit pair per step.
template <int FMT, int BROWS, bool BF16_OUT>
__global__ void __launch_bounds__(kThreads)
dequant_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ sf, int scale_layout,
               const float *__restrict__ s_dec_ptr, int64_t rows, int64_t cols,
               void *__restrict__ y) {
  __shared__ float itab[16];
  if (threadIdx.x < 16) {
    const int k = threadIdx.x >= 8 ? static_cast<int>(threadIdx.x) - 16 : static_cast<int>(threadIdx.x);
    itab[threadIdx.x] = __fmul_rn(static_cast<float>(k), __fdiv_rn(6.0f, 7.0f));
  }
  __syncthreads();
  const float s_dec = (FMT == FP4Q_FMT_MXFP4) ? 1.0f : *s_dec_ptr;
  constexpr int BLK = FMT == FP4Q_FMT_MXFP4 ? 32 : 16;
  const int64_t upr = cols / 32;                 // 32-code unit pairs per row (cols % 32 == 0)
  const int64_t bpr = cols / BLK;
  const int64_t total = rows * upr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; u < total;
       u += stride) {
    const int64_t r = u / upr, c = (u - r * upr) * 32;
    const uint4 cw = __ldg(reinterpret_cast<const uint4 *>(q + r * (cols / 2) + c / 2));
    uint32_t s0, s1;
    if (BROWS == 16) {           // 16x16 tiles: linear [rows/16, cols/16]
      s0 = sf[(r / 16) * bpr + c / 16];
      s1 = sf[(r / 16) * bpr + c / 16 + 1];
    } else if (BLK == 32) {
      s0 = s1 = sf[scale_offset(r, c / 32, bpr, scale_layout)];
    } else {
      s0 = sf[scale_offset(r, c / 16, bpr, scale_layout)];
      s1 = sf[scale_offset(r, c / 16 + 1, bpr, scale_layout)];
    }
    float v0[16], v1[16];
    decode16<FMT>(cw.x, cw.y, s0, s_dec, itab, v0);
    decode16<FMT>(cw.z, cw.w, s1, s_dec, itab, v1);
    store16<BF16_OUT>(y, r * cols + c, v0);
    store16<BF16_OUT>(y, r * cols + c + 16, v1);
  }
}

// Rows whose length is an odd number of 16-code blocks (NVFP4 / IF4 with
// cols % 32 == 16): one block per step.
template <int FMT, int BROWS, bool BF16_OUT>
__global__ void __launch_bounds__(kThreads)
dequant16_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ sf, int scale_layout,
                 const float *__restrict__ s_dec_ptr, int64_t rows, int64_t cols,
                 void *__restrict__ y) {
  __shared__ float itab[16];
  if (threadIdx.x < 16) {
    const int k = threadIdx.x >= 8 ? static_cast<int>(threadIdx.x) - 16 : static_cast<int>(threadIdx.x);
    itab[threadIdx.x] = __fmul_rn(static_cast<float>(k), __fdiv_rn(6.0f, 7.0f));
  }
  __syncthreads();
  const float s_dec = *s_dec_ptr;
  const int64_t bpr = cols / 16, total = rows * bpr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; b < total;
       b += stride) {
    const int64_t r = b / bpr, cb = b - r * bpr;
    const uint2 cw = __ldg(reinterpret_cast<const uint2 *>(q + r * (cols / 2) + cb * 8));
    const uint32_t s = BROWS == 16 ? sf[(r / 16) * bpr + cb] : sf[scale_offset(r, cb, bpr, scale_layout)];
    float v[16];
    decode16<FMT>(cw.x, cw.y, s, s_dec, itab, v);
    store16<BF16_OUT>(y, r * cols + cb * 16, v);
  }
}

template <int FMT, int BROWS>
cudaError_t launch_fmt(const uint8_t *q, const uint8_t *sf, int scale_layout, const float *s_dec,
                       int64_t rows, int64_t cols, void *y, int y_dtype, const Launch &L) {
  const bool pairs = (cols % 32) == 0;
  const int64_t units = pairs ? rows * (cols / 32) : rows * (cols / 16);
  int64_t want = (units + kThreads - 1) / kThreads;
  int64_t cap = static_cast<int64_t>(L.num_sms) * 8;
  int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
  const bool bf = y_dtype == FP4Q_BF16;
  if (pairs) {
    if (bf)
      dequant_kernel<FMT, BROWS, true><<<grid, kThreads, 0, L.stream>>>(q, sf, scale_layout,
                                                                       s_dec, rows, cols, y);
    else
      dequant_kernel<FMT, BROWS, false><<<grid, kThreads, 0, L.stream>>>(q, sf, scale_layout,
                                                                        s_dec, rows, cols, y);
  } else {
    if (bf)
      dequant16_kernel<FMT, BROWS, true><<<grid, kThreads, 0, L.stream>>>(q, sf, scale_layout,
                                                                         s_dec, rows, cols, y);
    else
      dequant16_kernel<FMT, BROWS, false><<<grid, kThreads, 0, L.stream>>>(q, sf, scale_layout,
                                                                          s_dec, rows, cols, y);
  }
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
