// amax.cu -- tensor amax = max |x| (Qiita note on NVFP4, "scaleの導出": the
// global scale is 6*448 / max|x|).  The maximum is taken on the bit patterns
// of |x| (sign cleared), which orders non-negative floats exactly; a NaN
// input yields a NaN amax.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void block_max_to_global(uint32_t m, unsigned *out) {
  __shared__ uint32_t warp_m[kThreads / 32];
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  if ((threadIdx.x & 31) == 0) warp_m[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t v = threadIdx.x < kThreads / 32 ? warp_m[threadIdx.x] : 0u;
    v = __reduce_max_sync(0xFFFFFFFFu, v);
    if (threadIdx.x == 0) atomicMax(out, v);
  }
}

// BF16: 8 elements per 16-byte chunk; the max of the 16-bit |x| patterns,
// shifted into FP32 position, is the FP32 bit pattern of the amax.
__global__ void __launch_bounds__(kThreads)
amax_bf16_kernel(const uint16_t *__restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                 unsigned *__restrict__ out) {
  const int64_t cpr = cols / 8, total = rows * cpr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  uint32_t acc = 0;  // two 16-bit lanes
  int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  for (; i + stride < total; i += 2 * stride) {
    int64_t r0 = i / cpr, r1 = (i + stride) / cpr;
    uint4 a = __ldg(reinterpret_cast<const uint4 *>(x + r0 * ld + (i - r0 * cpr) * 8));
    uint4 b = __ldg(reinterpret_cast<const uint4 *>(x + r1 * ld + (i + stride - r1 * cpr) * 8));
    acc = __vmaxu2(acc, a.x & 0x7FFF7FFFu); acc = __vmaxu2(acc, a.y & 0x7FFF7FFFu);
    acc = __vmaxu2(acc, a.z & 0x7FFF7FFFu); acc = __vmaxu2(acc, a.w & 0x7FFF7FFFu);
    acc = __vmaxu2(acc, b.x & 0x7FFF7FFFu); acc = __vmaxu2(acc, b.y & 0x7FFF7FFFu);
    acc = __vmaxu2(acc, b.z & 0x7FFF7FFFu); acc = __vmaxu2(acc, b.w & 0x7FFF7FFFu);
  }
  if (i < total) {
    int64_t r0 = i / cpr;
    uint4 a = __ldg(reinterpret_cast<const uint4 *>(x + r0 * ld + (i - r0 * cpr) * 8));
    acc = __vmaxu2(acc, a.x & 0x7FFF7FFFu); acc = __vmaxu2(acc, a.y & 0x7FFF7FFFu);
    acc = __vmaxu2(acc, a.z & 0x7FFF7FFFu); acc = __vmaxu2(acc, a.w & 0x7FFF7FFFu);
  }
  uint32_t m = max(acc & 0xFFFFu, acc >> 16) << 16;
  block_max_to_global(m, out);
}

__global__ void __launch_bounds__(kThreads)
amax_f32_kernel(const uint32_t *__restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                unsigned *__restrict__ out) {
  const int64_t cpr = cols / 4, total = rows * cpr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  uint32_t m = 0;
  int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  for (; i + stride < total; i += 2 * stride) {
    int64_t r0 = i / cpr, r1 = (i + stride) / cpr;
    uint4 a = __ldg(reinterpret_cast<const uint4 *>(x + r0 * ld + (i - r0 * cpr) * 4));
    uint4 b = __ldg(reinterpret_cast<const uint4 *>(x + r1 * ld + (i + stride - r1 * cpr) * 4));
    m = max(m, max(max(a.x & 0x7FFFFFFFu, a.y & 0x7FFFFFFFu), max(a.z & 0x7FFFFFFFu, a.w & 0x7FFFFFFFu)));
    m = max(m, max(max(b.x & 0x7FFFFFFFu, b.y & 0x7FFFFFFFu), max(b.z & 0x7FFFFFFFu, b.w & 0x7FFFFFFFu)));
  }
  if (i < total) {
    int64_t r0 = i / cpr;
    uint4 a = __ldg(reinterpret_cast<const uint4 *>(x + r0 * ld + (i - r0 * cpr) * 4));
    m = max(m, max(max(a.x & 0x7FFFFFFFu, a.y & 0x7FFFFFFFu), max(a.z & 0x7FFFFFFFu, a.w & 0x7FFFFFFFu)));
  }
  block_max_to_global(m, out);
}

}  // namespace

cudaError_t launch_amax(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                        float *amax_out, const Launch &L) {
  cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), L.stream);
  if (e != cudaSuccess) return e;
  const int64_t chunks = rows * cols / (dtype == FP4Q_BF16 ? 8 : 4);
  int64_t want = (chunks + 2 * kThreads - 1) / (2 * kThreads);
  int64_t cap = static_cast<int64_t>(L.num_sms) * 8;
  int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
  if (dtype == FP4Q_BF16)
    amax_bf16_kernel<<<grid, kThreads, 0, L.stream>>>(static_cast<const uint16_t *>(x), rows,
                                                      cols, ld,
                                                      reinterpret_cast<unsigned *>(amax_out));
  else
    amax_f32_kernel<<<grid, kThreads, 0, L.stream>>>(static_cast<const uint32_t *>(x), rows,
                                                     cols, ld,
                                                     reinterpret_cast<unsigned *>(amax_out));
  return cudaGetLastError();
}

}  // namespace fp4q
