// dequant.cu -- block-scaled FP4 back to FP32 / BF16.
//
// Ultralytics glossary "FP4", "FP4の仕組み": the reconstructed value is the
// grid value times its sign times the block scale.  NVFP4 also multiplies by
// the per-tensor decode scale; IF4 INT4 blocks (scale bit 7) decode k * 6/7
// (the 6/7 method of the "Adaptive Block-Scaled Data Types" explainer).
//   NVFP4 / IF4-FP4:  y = RN(RN(g * S) * s_dec)
//   IF4-INT4:         y = RN(RN(RN(k * RN(6/7)) * S) * s_dec)
//   MXFP4:            y = g * 2^(byte - 127)
// One thread per block of 16 (or 32) codes along a row.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;

template <int FMT, int BLK, int BROWS, bool BF16_OUT>
__global__ void __launch_bounds__(kThreads)
dequant_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ sf, int scale_layout,
               const float *__restrict__ s_dec_ptr, int64_t rows, int64_t cols,
               void *__restrict__ y) {
  const float s_dec = (FMT == FP4Q_FMT_MXFP4) ? 1.0f : *s_dec_ptr;
  const float c67 = __fdiv_rn(6.0f, 7.0f);
  const int64_t bpr = cols / BLK, nblk = rows * bpr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; b < nblk;
       b += stride) {
    const int64_t r = b / bpr, cb = b - r * bpr;
    uint32_t words[BLK / 8];
    const uint8_t *qp = q + r * (cols / 2) + cb * (BLK / 2);
    if (BLK == 16) {
      uint2 u = __ldg(reinterpret_cast<const uint2 *>(qp));
      words[0] = u.x; words[1 % (BLK / 8)] = u.y;
    } else {
      uint4 u = __ldg(reinterpret_cast<const uint4 *>(qp));
      words[0] = u.x; words[1] = u.y; words[2 % (BLK / 8)] = u.z; words[3 % (BLK / 8)] = u.w;
    }
    // scale byte of this block: 1 x BLK blocks use the (possibly swizzled)
    // [rows, cols/BLK] matrix; 16 x 16 tiles use the linear [rows/16, cols/16] one
    const uint32_t sbyte = (BROWS == 1) ? sf[scale_offset(r, cb, bpr, scale_layout)]
                                        : sf[(r / 16) * bpr + cb];
    float out[BLK];
    if (FMT == FP4Q_FMT_MXFP4) {
      const float p = e8m0_value(sbyte);
#pragma unroll
      for (int k = 0; k < BLK; ++k)
        out[k] = __fmul_rn(e2m1_value((words[k >> 3] >> (4 * (k & 7))) & 0xFu), p);
    } else {
      const float S = e4m3_value(sbyte & 0x7Fu);
      if (FMT == FP4Q_FMT_IF4 && (sbyte & 0x80u)) {
#pragma unroll
        for (int k = 0; k < BLK; ++k) {
          const int nib = static_cast<int>((words[k >> 3] >> (4 * (k & 7))) & 0xFu);
          const int kk = nib >= 8 ? nib - 16 : nib;
          const float h = __fmul_rn(static_cast<float>(kk), c67);
          out[k] = __fmul_rn(__fmul_rn(h, S), s_dec);
        }
      } else {
#pragma unroll
        for (int k = 0; k < BLK; ++k) {
          const float g = e2m1_value((words[k >> 3] >> (4 * (k & 7))) & 0xFu);
          out[k] = __fmul_rn(__fmul_rn(g, S), s_dec);
        }
      }
    }
    if (BF16_OUT) {
      uint32_t packed[BLK / 2];
#pragma unroll
      for (int k = 0; k < BLK; k += 2) {
        __nv_bfloat162 h2 = __floats2bfloat162_rn(out[k], out[k + 1]);
        packed[k / 2] = *reinterpret_cast<uint32_t *>(&h2);
      }
      uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(y) + r * cols + cb * BLK);
#pragma unroll
      for (int k = 0; k < BLK / 8; ++k)
        dst[k] = make_uint4(packed[4 * k], packed[4 * k + 1], packed[4 * k + 2], packed[4 * k + 3]);
    } else {
      float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(y) + r * cols + cb * BLK);
#pragma unroll
      for (int k = 0; k < BLK / 4; ++k)
        dst[k] = make_float4(out[4 * k], out[4 * k + 1], out[4 * k + 2], out[4 * k + 3]);
    }
  }
}

template <int FMT, int BLK, int BROWS>
cudaError_t launch_fmt(const uint8_t *q, const uint8_t *sf, int scale_layout, const float *s_dec,
                       int64_t rows, int64_t cols, void *y, int y_dtype, const Launch &L) {
  const int64_t nblk = rows * (cols / BLK);
  int64_t want = (nblk + kThreads - 1) / kThreads;
  int64_t cap = static_cast<int64_t>(L.num_sms) * 8;
  int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
  if (y_dtype == FP4Q_BF16)
    dequant_kernel<FMT, BLK, BROWS, true><<<grid, kThreads, 0, L.stream>>>(
        q, sf, scale_layout, s_dec, rows, cols, y);
  else
    dequant_kernel<FMT, BLK, BROWS, false><<<grid, kThreads, 0, L.stream>>>(
        q, sf, scale_layout, s_dec, rows, cols, y);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dequant(int format, const uint8_t *q, const uint8_t *sf, int scale_layout,
                           int block_rows, int block_cols, const float *s_dec, int64_t rows,
                           int64_t cols, void *y, int y_dtype, const Launch &L) {
  if (format == FP4Q_FMT_MXFP4)
    return launch_fmt<FP4Q_FMT_MXFP4, 32, 1>(q, sf, scale_layout, s_dec, rows, cols, y, y_dtype, L);
  if (format == FP4Q_FMT_IF4)
    return launch_fmt<FP4Q_FMT_IF4, 16, 1>(q, sf, scale_layout, s_dec, rows, cols, y, y_dtype, L);
  if (block_rows == 16)
    return launch_fmt<FP4Q_FMT_NVFP4, 16, 16>(q, sf, scale_layout, s_dec, rows, cols, y, y_dtype, L);
  return launch_fmt<FP4Q_FMT_NVFP4, 16, 1>(q, sf, scale_layout, s_dec, rows, cols, y, y_dtype, L);
}

}  // namespace fp4q
