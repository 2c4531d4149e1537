// quant2d.cu -- NVFP4 with 16x16 2D block scaling for weights.
//
// Qiita note on NVFP4 training, "2D scaling": with 1x16 blocks q(W) differs
// from q(W^T)^T because the scaling direction changes under transposition;
// square 16x16 tiles give both the same scales, so W and W^T codes come out
// of one pass.  Each 64 x 64 region is staged in shared memory; 16 threads
// share a tile: thread i quantizes row i of the tile (W codes) and column i
// (W^T codes) with the tile's single scale.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;
constexpr int kRegion = 64;

template <typename T>
__global__ void __launch_bounds__(kThreads)
quant2d_kernel(const T *__restrict__ w, int64_t rows, int64_t cols, int64_t ld,
               const float *__restrict__ amax_ptr, float *__restrict__ s_dec_out,
               uint8_t *__restrict__ q_w, uint8_t *__restrict__ q_wt,
               uint8_t *__restrict__ sf_tiles, uint8_t *__restrict__ sf_w_1x16,
               uint8_t *__restrict__ sf_wt_1x16, int scale_layout) {
  // row stride of 68 floats (or 72 BF16) staggers rows across bank groups
  constexpr int PAD = sizeof(T) == 4 ? 4 : 8;
  __shared__ __align__(16) float tile[kRegion][kRegion + PAD];
  __shared__ float rtab[128];
  const TensorScale ts = tensor_scale(*amax_ptr);
  fill_factor_table(rtab, ts.enc);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && s_dec_out) *s_dec_out = ts.dec;

  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kRegion;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kRegion;
  const int t = threadIdx.x;
  for (int id = t; id < kRegion * (kRegion / 8); id += kThreads) {
    int rr = id / (kRegion / 8), cc = (id % (kRegion / 8)) * 8;
    float v[8];
    if (r0 + rr < rows && c0 + cc < cols) {
      Vec8<T>::load(w + (r0 + rr) * ld + c0 + cc, v);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = 0.0f;
    }
    *reinterpret_cast<float4 *>(&tile[rr][cc]) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4 *>(&tile[rr][cc + 4]) = make_float4(v[4], v[5], v[6], v[7]);
  }
  __syncthreads();

  const int tid = t >> 4;            // tile within the region: 4 x 4
  const int i = t & 15;              // row (and column) of the tile this thread owns
  const int tr = tid >> 2, tc = tid & 3;
  const int64_t gr = r0 + tr * 16, gc = c0 + tc * 16;   // tile origin
  const bool valid = gr < rows && gc < cols;

  float rowv[16], colv[16];
#pragma unroll
  for (int k = 0; k < 16; k += 4) {
    float4 a = *reinterpret_cast<const float4 *>(&tile[tr * 16 + i][tc * 16 + k]);
    rowv[k] = a.x; rowv[k + 1] = a.y; rowv[k + 2] = a.z; rowv[k + 3] = a.w;
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) colv[k] = tile[tr * 16 + k][tc * 16 + i];

  float m = 0.0f;
#pragma unroll
  for (int k = 0; k < 16; ++k) m = fmaxf(m, fabsf(rowv[k]));
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (!valid) return;   // (no barrier follows)

  const uint32_t sbyte = nvfp4_scale_code(m, ts.enc);
  const float f = rtab[sbyte];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    rowv[k] = __fmul_rn(rowv[k], f);
    colv[k] = __fmul_rn(colv[k], f);
  }
  uint32_t wr[2], wc[2];
  {
    float a[8], b[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) { a[k] = rowv[k]; b[k] = rowv[k + 8]; }
    wr[0] = e2m1x8(a); wr[1] = e2m1x8(b);
#pragma unroll
    for (int k = 0; k < 8; ++k) { a[k] = colv[k]; b[k] = colv[k + 8]; }
    wc[0] = e2m1x8(a); wc[1] = e2m1x8(b);
  }
  const int64_t r = gr + i, c = gc + i;
  if (q_w) *reinterpret_cast<uint2 *>(q_w + r * (cols / 2) + gc / 2) = make_uint2(wr[0], wr[1]);
  if (q_wt) *reinterpret_cast<uint2 *>(q_wt + c * (rows / 2) + gr / 2) = make_uint2(wc[0], wc[1]);
  if (i == 0) sf_tiles[(gr / 16) * (cols / 16) + gc / 16] = static_cast<uint8_t>(sbyte);
  if (sf_w_1x16) sf_w_1x16[scale_offset(r, gc / 16, cols / 16, scale_layout)] = static_cast<uint8_t>(sbyte);
  if (sf_wt_1x16) sf_wt_1x16[scale_offset(c, gr / 16, rows / 16, scale_layout)] = static_cast<uint8_t>(sbyte);
}

}  // namespace

cudaError_t launch_2d(const void *w, int dtype, int64_t rows, int64_t cols, int64_t ld,
                      const float *amax, float *s_dec_out, uint8_t *q_w, uint8_t *q_wt,
                      uint8_t *sf_tiles, uint8_t *sf_w_1x16, uint8_t *sf_wt_1x16,
                      int scale_layout, const Launch &L) {
  dim3 grid(static_cast<unsigned>((cols + kRegion - 1) / kRegion),
            static_cast<unsigned>((rows + kRegion - 1) / kRegion));
  if (dtype == FP4Q_BF16)
    quant2d_kernel<__nv_bfloat16><<<grid, kThreads, 0, L.stream>>>(
        static_cast<const __nv_bfloat16 *>(w), rows, cols, ld, amax, s_dec_out, q_w, q_wt,
        sf_tiles, sf_w_1x16, sf_wt_1x16, scale_layout);
  else
    quant2d_kernel<float><<<grid, kThreads, 0, L.stream>>>(
        static_cast<const float *>(w), rows, cols, ld, amax, s_dec_out, q_w, q_wt, sf_tiles,
        sf_w_1x16, sf_wt_1x16, scale_layout);
  return cudaGetLastError();
}

}  // namespace fp4q
