// nvfp4.cu -- NVFP4 1x16 and MXFP4 1x32 quantization, row-wise and/or
// column-wise (the transposed copy the backward pass needs) from one read.
//
// Qiita note on NVFP4 training: "Blockwise" (16 values share one 8-bit
// scale), "誤差逆伝播と転置" (Wgrad / Dgrad consume transposed operands),
// "scaleの導出" (global scale 6*448/amax, local scale = block max / 6 in
// E4M3).  Ultralytics glossary "FP4", "FP4の仕組み" (MXFP4: 32 values per
// power-of-two E8M0 scale).
//
// Two kernels:
//   rowwise_kernel  one thread per block of 16 (NVFP4) or 32 (MXFP4) values
//                   along a row; 128-bit loads, 64/128-bit code stores.
//   tile_kernel     a 64 x 64 tile staged in shared memory; row blocks and
//                   column blocks are quantized from the same staged copy.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;

// Quantize BLK values already scaled into the E2M1 domain (RNE), packed
// nibbles in words (8 values per word).
template <int BLK>
__device__ __forceinline__ void encode_rne(const float *v, uint32_t *words) {
#pragma unroll
  for (int w = 0; w < BLK / 8; ++w) {
    float t[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) t[k] = v[w * 8 + k];
    words[w] = e2m1x8(t);
  }
}

// Stochastic rounding of 16 values whose flat input indices are
// first + k * step (k = 0..15).
__device__ __forceinline__ void encode_sr16(const float *v, uint64_t seed, uint64_t first,
                                            uint64_t step, uint32_t *words) {
  words[0] = words[1] = 0u;
  if (step == 1 && (first % 8) == 0) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      U32x4 bits = sr_bits_group(seed, first / 8 + h);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        words[h] |= e2m1_sr(v[h * 8 + k], half16(bits, k)) << (4 * k);
    }
  } else {
#pragma unroll 1
    for (int k = 0; k < 16; ++k) {
      uint64_t i = first + static_cast<uint64_t>(k) * step;
      U32x4 bits = sr_bits_group(seed, i / 8);
      words[k >> 3] |= e2m1_sr(v[k], half16(bits, static_cast<int>(i % 8))) << (4 * (k & 7));
    }
  }
}

template <typename T>
__device__ __forceinline__ void load_row_block(const T *p, float *v, int blk) {
  for (int c = 0; c < blk; c += 8) Vec8<T>::load(p + c, *reinterpret_cast<float(*)[8]>(v + c));
}

// ----------------------------------------------------------------------------
// row-wise only
// ----------------------------------------------------------------------------
template <typename T, bool MX, bool SR>
__global__ void __launch_bounds__(kThreads)
rowwise_kernel(const T *__restrict__ x, int64_t rows, int64_t cols, int64_t ld,
               const float *__restrict__ amax_ptr, int e8m0_mode, uint64_t seed,
               float *__restrict__ s_dec_out, uint8_t *__restrict__ q,
               uint8_t *__restrict__ sf, int scale_layout) {
  constexpr int BLK = MX ? 32 : 16;
  __shared__ float rtab[128];
  TensorScale ts{1.0f, 1.0f};
  if (!MX) {
    ts = tensor_scale(*amax_ptr);
    fill_factor_table(rtab, ts.enc);
    if (blockIdx.x == 0 && threadIdx.x == 0 && s_dec_out) *s_dec_out = ts.dec;
    __syncthreads();
  }
  const int64_t bpr = cols / BLK, nblk = rows * bpr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; b < nblk;
       b += stride) {
    const int64_t r = b / bpr, cb = b - r * bpr;
    float v[BLK];
    load_row_block(x + r * ld + cb * BLK, v, BLK);
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < BLK; ++k) m = fmaxf(m, fabsf(v[k]));
    uint32_t sbyte;
    float f;
    if (MX) {
      int e = e8m0_exponent(m, e8m0_mode);
      sbyte = static_cast<uint32_t>(e + 127);
      f = exp2_neg(e);
    } else {
      sbyte = nvfp4_scale_code(m, ts.enc);
      f = rtab[sbyte];
    }
#pragma unroll
    for (int k = 0; k < BLK; ++k) v[k] = __fmul_rn(v[k], f);
    uint32_t words[BLK / 8];
    if (SR) encode_sr16(v, seed, static_cast<uint64_t>(r * cols + cb * BLK), 1, words);
    else encode_rne<BLK>(v, words);
    uint8_t *qp = q + r * (cols / 2) + cb * (BLK / 2);
    if (BLK == 16) *reinterpret_cast<uint2 *>(qp) = make_uint2(words[0], words[1]);
    else *reinterpret_cast<uint4 *>(qp) = make_uint4(words[0], words[1], words[2], words[3]);
    sf[scale_offset(r, cb, bpr, scale_layout)] = static_cast<uint8_t>(sbyte);
  }
}

// ----------------------------------------------------------------------------
// row-wise and/or column-wise through a shared-memory tile
// ----------------------------------------------------------------------------
constexpr int kTile = 64;

template <typename T, bool MX, bool SR>
__global__ void __launch_bounds__(kThreads)
tile_kernel(const T *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, unsigned layouts,
            const float *__restrict__ amax_ptr, int e8m0_mode, uint64_t seed,
            float *__restrict__ s_dec_out, uint8_t *__restrict__ q_row,
            uint8_t *__restrict__ sf_row, uint8_t *__restrict__ q_col,
            uint8_t *__restrict__ sf_col, int scale_layout) {
  constexpr int BLK = MX ? 32 : 16;
  constexpr int PAD = 16 / sizeof(T);   // keeps 16-byte row alignment
  __shared__ __align__(16) T tile[kTile][kTile + PAD];
  __shared__ float rtab[128];
  TensorScale ts{1.0f, 1.0f};
  if (!MX) {
    ts = tensor_scale(*amax_ptr);
    fill_factor_table(rtab, ts.enc);
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && s_dec_out)
      *s_dec_out = ts.dec;
  }
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kTile;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTile;
  const int t = threadIdx.x;

  // stage: 64 rows x 8 chunks of 8 elements
  for (int id = t; id < kTile * (kTile / 8); id += kThreads) {
    int rr = id / (kTile / 8), cc = (id % (kTile / 8)) * 8;
    float v[8];
    if (r0 + rr < rows && c0 + cc < cols) {
      Vec8<T>::load(x + (r0 + rr) * ld + c0 + cc, v);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = 0.0f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) tile[rr][cc + k] = static_cast<T>(v[k]);
  }
  __syncthreads();

  auto quantize_block = [&](float *v, uint64_t first, uint64_t step, uint32_t *words) {
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < BLK; ++k) m = fmaxf(m, fabsf(v[k]));
    uint32_t sbyte;
    float f;
    if (MX) {
      int e = e8m0_exponent(m, e8m0_mode);
      sbyte = static_cast<uint32_t>(e + 127);
      f = exp2_neg(e);
    } else {
      sbyte = nvfp4_scale_code(m, ts.enc);
      f = rtab[sbyte];
    }
#pragma unroll
    for (int k = 0; k < BLK; ++k) v[k] = __fmul_rn(v[k], f);
    if (SR) encode_sr16(v, seed, first, step, words);
    else encode_rne<BLK>(v, words);
    return sbyte;
  };

  if (layouts & FP4Q_ROWWISE) {
    constexpr int kBlocks = kTile * (kTile / BLK);
    for (int id = t; id < kBlocks; id += kThreads) {
      int rr = id / (kTile / BLK), cb = id % (kTile / BLK);
      int64_t r = r0 + rr, c = c0 + cb * BLK;
      if (r >= rows || c >= cols) continue;
      float v[BLK];
#pragma unroll
      for (int k = 0; k < BLK; ++k) v[k] = to_f32(tile[rr][cb * BLK + k]);
      uint32_t words[BLK / 8];
      uint32_t sbyte = quantize_block(v, static_cast<uint64_t>(r * cols + c), 1, words);
      uint8_t *qp = q_row + r * (cols / 2) + c / 2;
      if (BLK == 16) *reinterpret_cast<uint2 *>(qp) = make_uint2(words[0], words[1]);
      else *reinterpret_cast<uint4 *>(qp) = make_uint4(words[0], words[1], words[2], words[3]);
      sf_row[scale_offset(r, c / BLK, cols / BLK, scale_layout)] = static_cast<uint8_t>(sbyte);
    }
  }
  if (layouts & FP4Q_COLWISE) {
    constexpr int kBlocks = kTile * (kTile / BLK);
    for (int id = t; id < kBlocks; id += kThreads) {
      int cc = id % kTile, rb = id / kTile;
      int64_t c = c0 + cc, r = r0 + rb * BLK;
      if (c >= cols || r >= rows) continue;
      float v[BLK];
#pragma unroll
      for (int k = 0; k < BLK; ++k) v[k] = to_f32(tile[rb * BLK + k][cc]);
      uint32_t words[BLK / 8];
      uint32_t sbyte =
          quantize_block(v, static_cast<uint64_t>(r * cols + c), static_cast<uint64_t>(cols), words);
      uint8_t *qp = q_col + c * (rows / 2) + r / 2;
      if (BLK == 16) *reinterpret_cast<uint2 *>(qp) = make_uint2(words[0], words[1]);
      else *reinterpret_cast<uint4 *>(qp) = make_uint4(words[0], words[1], words[2], words[3]);
      sf_col[scale_offset(c, r / BLK, rows / BLK, scale_layout)] = static_cast<uint8_t>(sbyte);
    }
  }
}

int rowwise_grid(int64_t nblk, const Launch &L) {
  int64_t want = (nblk + kThreads - 1) / kThreads;
  int64_t cap = static_cast<int64_t>(L.num_sms) * 8;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

template <typename T, bool MX, bool SR>
cudaError_t launch_typed(const T *x, int64_t rows, int64_t cols, int64_t ld, unsigned layouts,
                         const float *amax, int e8m0_mode, uint64_t seed, float *s_dec_out,
                         uint8_t *q_row, uint8_t *sf_row, uint8_t *q_col, uint8_t *sf_col,
                         int scale_layout, const Launch &L) {
  constexpr int BLK = MX ? 32 : 16;
  if (layouts == FP4Q_ROWWISE) {
    rowwise_kernel<T, MX, SR><<<rowwise_grid(rows * (cols / BLK), L), kThreads, 0, L.stream>>>(
        x, rows, cols, ld, amax, e8m0_mode, seed, s_dec_out, q_row, sf_row, scale_layout);
  } else {
    dim3 grid(static_cast<unsigned>((cols + kTile - 1) / kTile),
              static_cast<unsigned>((rows + kTile - 1) / kTile));
    tile_kernel<T, MX, SR><<<grid, kThreads, 0, L.stream>>>(
        x, rows, cols, ld, layouts, amax, e8m0_mode, seed, s_dec_out, q_row, sf_row, q_col,
        sf_col, scale_layout);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_nvfp4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                         unsigned layouts, int round, uint64_t seed, const float *amax,
                         float *s_dec_out, uint8_t *q_row, uint8_t *sf_row, uint8_t *q_col,
                         uint8_t *sf_col, int scale_layout, const Launch &L) {
  const bool sr = round == FP4Q_SR;
  if (dtype == FP4Q_BF16) {
    auto *p = static_cast<const __nv_bfloat16 *>(x);
    return sr ? launch_typed<__nv_bfloat16, false, true>(p, rows, cols, ld, layouts, amax, 0, seed,
                                                         s_dec_out, q_row, sf_row, q_col, sf_col,
                                                         scale_layout, L)
              : launch_typed<__nv_bfloat16, false, false>(p, rows, cols, ld, layouts, amax, 0,
                                                          seed, s_dec_out, q_row, sf_row, q_col,
                                                          sf_col, scale_layout, L);
  }
  auto *p = static_cast<const float *>(x);
  return sr ? launch_typed<float, false, true>(p, rows, cols, ld, layouts, amax, 0, seed, s_dec_out,
                                               q_row, sf_row, q_col, sf_col, scale_layout, L)
            : launch_typed<float, false, false>(p, rows, cols, ld, layouts, amax, 0, seed,
                                                s_dec_out, q_row, sf_row, q_col, sf_col,
                                                scale_layout, L);
}

cudaError_t launch_mxfp4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                         unsigned layouts, int e8m0_mode, uint8_t *q_row, uint8_t *sf_row,
                         uint8_t *q_col, uint8_t *sf_col, int scale_layout, const Launch &L) {
  if (dtype == FP4Q_BF16)
    return launch_typed<__nv_bfloat16, true, false>(static_cast<const __nv_bfloat16 *>(x), rows,
                                                    cols, ld, layouts, nullptr, e8m0_mode, 0,
                                                    nullptr, q_row, sf_row, q_col, sf_col,
                                                    scale_layout, L);
  return launch_typed<float, true, false>(static_cast<const float *>(x), rows, cols, ld, layouts,
                                          nullptr, e8m0_mode, 0, nullptr, q_row, sf_row, q_col,
                                          sf_col, scale_layout, L);
}

}  // namespace fp4q
