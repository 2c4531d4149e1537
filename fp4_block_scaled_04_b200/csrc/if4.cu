// if4.cu -- IF4 adaptive block-scaled quantization, row-wise 1x16.
//
// "Adaptive Block-Scaled Data Types" (gist.science explainer), section 2
// (IF4): every 16-value block is quantized both as FP4 (E2M1) and as INT4,
// the one with the smaller squared error is kept, and the choice goes into
// the otherwise unused sign bit of the block's E4M3 scale.  The 6/7 method
// maps INT4's range 0..7 onto FP4's 0..6: values are multiplied by 7/6
// before rounding to an integer and by 6/7 when decoded.
//
// One thread per block; the block scale S and factor r are the NVFP4 ones.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kThreads)
if4_kernel(const T *__restrict__ x, int64_t rows, int64_t cols, int64_t ld,
           const float *__restrict__ amax_ptr, float *__restrict__ s_dec_out,
           uint8_t *__restrict__ q, uint8_t *__restrict__ sf, int scale_layout) {
  __shared__ float rtab[128];
  const TensorScale ts = tensor_scale(*amax_ptr);
  fill_factor_table(rtab, ts.enc);
  if (blockIdx.x == 0 && threadIdx.x == 0 && s_dec_out) *s_dec_out = ts.dec;
  __syncthreads();
  const float c76 = __fdiv_rn(7.0f, 6.0f);   // RN(7/6)
  const float c67 = __fdiv_rn(6.0f, 7.0f);   // RN(6/7)

  const int64_t bpr = cols / 16, nblk = rows * bpr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; b < nblk;
       b += stride) {
    const int64_t r = b / bpr, cb = b - r * bpr;
    float v[16];
    Vec8<T>::load(x + r * ld + cb * 16, *reinterpret_cast<float(*)[8]>(v));
    Vec8<T>::load(x + r * ld + cb * 16 + 8, *reinterpret_cast<float(*)[8]>(v + 8));
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < 16; ++k) m = fmaxf(m, fabsf(v[k]));
    const uint32_t sbyte = nvfp4_scale_code(m, ts.enc);
    const float f = rtab[sbyte];
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = __fmul_rn(v[k], f);

    // FP4 candidate
    uint32_t wfp[2];
    {
      float a[8], c[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) { a[k] = v[k]; c[k] = v[k + 8]; }
      wfp[0] = e2m1x8(a);
      wfp[1] = e2m1x8(c);
    }
    // INT4 candidate and both squared errors, summed in order k = 0..15
    uint32_t wint[2] = {0u, 0u};
    float e_fp = 0.0f, e_int = 0.0f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float g = e2m1_value((wfp[k >> 3] >> (4 * (k & 7))) & 0xFu);
      float kk = rintf(__fmul_rn(v[k], c76));
      kk = fminf(fmaxf(kk, -7.0f), 7.0f);
      const int ki = static_cast<int>(kk);
      wint[k >> 3] |= (static_cast<uint32_t>(ki) & 0xFu) << (4 * (k & 7));
      const float h = __fmul_rn(static_cast<float>(ki), c67);
      const float dfp = __fsub_rn(v[k], g);
      const float dint = __fsub_rn(v[k], h);
      e_fp = __fmaf_rn(dfp, dfp, e_fp);
      e_int = __fmaf_rn(dint, dint, e_int);
    }
    const bool use_int = e_int < e_fp;
    uint8_t *qp = q + r * (cols / 2) + cb * 8;
    *reinterpret_cast<uint2 *>(qp) =
        use_int ? make_uint2(wint[0], wint[1]) : make_uint2(wfp[0], wfp[1]);
    sf[scale_offset(r, cb, bpr, scale_layout)] =
        static_cast<uint8_t>(sbyte | (use_int ? 0x80u : 0u));
  }
}

}  // namespace

cudaError_t launch_if4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                       const float *amax, float *s_dec_out, uint8_t *q, uint8_t *sf,
                       int scale_layout, const Launch &L) {
  const int64_t nblk = rows * (cols / 16);
  int64_t want = (nblk + kThreads - 1) / kThreads;
  int64_t cap = static_cast<int64_t>(L.num_sms) * 8;
  int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
  if (dtype == FP4Q_BF16)
    if4_kernel<__nv_bfloat16><<<grid, kThreads, 0, L.stream>>>(
        static_cast<const __nv_bfloat16 *>(x), rows, cols, ld, amax, s_dec_out, q, sf,
        scale_layout);
  else
    if4_kernel<float><<<grid, kThreads, 0, L.stream>>>(static_cast<const float *>(x), rows, cols,
                                                       ld, amax, s_dec_out, q, sf, scale_layout);
  return cudaGetLastError();
}

}  // namespace fp4q
