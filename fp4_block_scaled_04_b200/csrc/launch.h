// launch.h -- internal host-side launchers (one per kernel family).  The
// extern "C" entry points in api.cu validate arguments and call these.
#pragma once

#include <cstddef>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

namespace fp4q {

struct Launch {
  cudaStream_t stream;
  int num_sms;
};

// Puts the caller's current device back when an entry point returns: the
// entry points make the device that owns their data current before they
// enqueue work, and the caller's thread state is not theirs to keep.
class DeviceGuard {
 public:
  DeviceGuard() {
    if (cudaGetDevice(&prev_) != cudaSuccess) {
      cudaGetLastError();
      prev_ = -1;
    }
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev_ >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev_) cudaSetDevice(prev_);
  }
  DeviceGuard(const DeviceGuard &) = delete;
  DeviceGuard &operator=(const DeviceGuard &) = delete;

 private:
  int prev_ = -1;
};

// One-time set-up of a kernel on the current device: its dynamic shared
// memory limit and how many of
// its CTAs fit on one SM.  Function attributes belong to a device, so each
// device is set up once; std::call_once makes concurrent first calls from
// several host threads safe.  Devices beyond the first 64 are not cached.
struct KernelSetup {
  std::once_flag once[64];
  cudaError_t err[64] = {};
  int per_sm[64] = {};
};

inline cudaError_t kernel_setup(KernelSetup &ks, const void *kern, int threads, int smem,
                                int *per_sm) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return cudaGetLastError();
  auto run = [&](cudaError_t *err, int *n) {
    *err = cudaSuccess;
    if (smem > 0) {   // the limit counts dynamic shared memory on top of the static
      *err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (*err != cudaSuccess) return;
    }
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(n, kern, threads, smem) != cudaSuccess ||
        *n < 1) {
      cudaGetLastError();
      *n = 1;
    }
  };
  if (dev >= 64) {
    cudaError_t e;
    run(&e, per_sm);
    return e;
  }
  std::call_once(ks.once[dev], [&] { run(&ks.err[dev], &ks.per_sm[dev]); });
  *per_sm = ks.per_sm[dev];
  return ks.err[dev];
}

// The host-side argument checks of fp4q_quantize_nvfp4 that need no device
// (enums, shape, alignment, required pointers); FP4Q_OK or the status that
// call would return.
int check_nvfp4_args(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                     unsigned layouts, int round, const uint8_t *q_row, const uint8_t *sf_row,
                     const uint8_t *q_col, const uint8_t *sf_col, int scale_layout);

cudaError_t launch_amax(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                        float *amax_out, const Launch &L);

cudaError_t launch_nvfp4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                         unsigned layouts, int round, uint64_t seed, const float *amax,
                         float *s_dec_out, uint8_t *q_row, uint8_t *sf_row, uint8_t *q_col,
                         uint8_t *sf_col, int scale_layout, const Launch &L);

// NVFP4 1x16 layout with every block maximum mapped to 4 (round to nearest)
cudaError_t launch_four_over_six(const void *x, int dtype, int64_t rows, int64_t cols,
                                 int64_t ld, unsigned layouts, const float *amax,
                                 float *s_dec_out, uint8_t *q_row, uint8_t *sf_row,
                                 uint8_t *q_col, uint8_t *sf_col, int scale_layout,
                                 const Launch &L);

cudaError_t launch_mxfp4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                         unsigned layouts, int e8m0_mode, uint8_t *q_row, uint8_t *sf_row,
                         uint8_t *q_col, uint8_t *sf_col, int scale_layout, const Launch &L);

cudaError_t launch_2d(const void *w, int dtype, int64_t rows, int64_t cols, int64_t ld,
                      const float *amax, float *s_dec_out, uint8_t *q_w, uint8_t *q_wt,
                      uint8_t *sf_tiles, uint8_t *sf_w_1x16, uint8_t *sf_wt_1x16,
                      int scale_layout, const Launch &L);

cudaError_t launch_rht_amax(const void *dy, int dtype, int64_t tokens, int64_t cols,
                            int64_t ld, int n, uint64_t seed, float *amax_out,
                            const Launch &L);

cudaError_t launch_rht_quant(const void *dy, int dtype, int64_t tokens, int64_t cols,
                             int64_t ld, int n, int round, uint64_t seed, const float *amax,
                             float *s_dec_out, uint8_t *q_t, uint8_t *sf_t, int scale_layout,
                             float *rht_out, const Launch &L);

// One read of dY: row-wise NVFP4 (the Dgrad operand, seed_row, amax_row) and
// the RHT + column-wise NVFP4 of dY^T (the Wgrad operand, seed_col, amax_rht)
cudaError_t launch_rht_backward(const void *dy, int dtype, int64_t tokens, int64_t cols,
                                int64_t ld, int n, int round, uint64_t seed_row,
                                uint64_t seed_col, const float *amax_row, const float *amax_rht,
                                float *s_dec_row, float *s_dec_col, uint8_t *q_row,
                                uint8_t *sf_row, uint8_t *q_t, uint8_t *sf_t, int scale_layout,
                                const Launch &L);

// MXFP6 row-wise (fp6_format FP4Q_FP6_E2M3 / FP4Q_FP6_E3M2), codes packed
// four per three bytes, and its decode
cudaError_t launch_mxfp6(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                         int fp6_format, int e8m0_mode, uint8_t *q, uint8_t *sf,
                         int scale_layout, const Launch &L);
cudaError_t launch_mxfp6_dequant(const uint8_t *q, const uint8_t *sf, int scale_layout,
                                 int64_t rows, int64_t cols, int fp6_format, void *y,
                                 int y_dtype, const Launch &L);

// Options of the tensor-core GEMM: the product is scaled by a = RN(RN(s_a s_b)
// * alpha_mul); with a second accumulator (the IF4 GEMM) that one is scaled by
// RN(a * alpha_int); withhold != 0 (a failure-detection test hook) issues no
// operand loads.
struct GemmOptions {
  float alpha_mul = 1.0f;
  float alpha_int = 1.0f;
  int withhold = 0;
};

// C[M, N] = s_a s_b (A B^T) from NVFP4 operands (codes [rows, K/2], swizzled
// 1x16 scales) on the tensor cores; status (may be NULL) <- 1 if a wait ran out
cudaError_t launch_gemm_nvfp4(const uint8_t *qa, const uint8_t *sfa, const float *s_a,
                              const uint8_t *qb, const uint8_t *sfb, const float *s_b, int64_t M,
                              int64_t N, int64_t K, void *c, int c_dtype, int64_t ldc,
                              int *status, GemmOptions opt, const Launch &L);

// C[M, N] = A B^T from MXFP4 operands (codes [rows, K/2], E8M0 scales per 32
// values in the 128x4 tile layout, no tensor scale) on the tensor cores
cudaError_t launch_gemm_mxfp4(const uint8_t *qa, const uint8_t *sfa, const uint8_t *qb,
                              const uint8_t *sfb, int64_t M, int64_t N, int64_t K, void *c,
                              int c_dtype, int64_t ldc, int *status, const Launch &L);

// IF4 x NVFP4 in one pass over the split operands: C = RN(RN(acc_fp * a) +
// RN(acc_int * RN(a * RN(6/7)))), acc_int accumulating both INT4 parts; FP32
// output, N % 128 == 0
cudaError_t launch_gemm_if4_split(const uint8_t *q_fp, const uint8_t *q_k1, const uint8_t *q_k2,
                                  const uint8_t *sfa, const float *s_a, const uint8_t *qb,
                                  const uint8_t *sfb, const float *s_b, int64_t M, int64_t N,
                                  int64_t K, float *c, int64_t ldc, int *status,
                                  const Launch &L);

// Split IF4 codes [rows, K/2] with flagged scales into three NVFP4 code
// matrices sharing the unflagged scales: FP4 blocks (INT4 blocks zero) and the
// two E2M1 parts g1 + g2 = k of the INT4 blocks (FP4 blocks zero)
cudaError_t launch_if4_split(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t K,
                             int scale_layout, uint8_t *q_fp, uint8_t *q_k1, uint8_t *q_k2,
                             uint8_t *sf_plain, const Launch &L);

// IF6: per 16-value block FP6 E2M3 or INT6 (rescaled by 7.5/31), codes four
// per three bytes; and its decode
cudaError_t launch_if6(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                       const float *amax, float *s_dec_out, uint8_t *q, uint8_t *sf,
                       int scale_layout, const Launch &L);
cudaError_t launch_if6_dequant(const uint8_t *q, const uint8_t *sf, int scale_layout,
                               const float *s_dec, int64_t rows, int64_t cols, void *y,
                               int y_dtype, const Launch &L);

// IF3: per 16-value block FP3 E2M0 or INT3 (rescaled by 4/3), codes eight
// per three bytes; and its decode
cudaError_t launch_if3(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                       const float *amax, float *s_dec_out, uint8_t *q, uint8_t *sf,
                       int scale_layout, const Launch &L);
cudaError_t launch_if3_dequant(const uint8_t *q, const uint8_t *sf, int scale_layout,
                               const float *s_dec, int64_t rows, int64_t cols, void *y,
                               int y_dtype, const Launch &L);

// int4_mode 1: IF4 (per-block choice); 2: NVINT4 (the INT4 candidate everywhere)
cudaError_t launch_if4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                       const float *amax, float *s_dec_out, uint8_t *q, uint8_t *sf,
                       int scale_layout, int int4_mode, const Launch &L);

cudaError_t launch_dequant(int format, const uint8_t *q, const uint8_t *sf, int scale_layout,
                           int block_rows, int block_cols, const float *s_dec, int64_t rows,
                           int64_t cols, void *y, int y_dtype, const Launch &L);

}  // namespace fp4q
