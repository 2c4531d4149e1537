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

// The 16-byte chunk idx of a [rows, cols] matrix with row stride ld: a flat
// offset when the rows are contiguous (FLAT, no division), else row idx / cpr.
template <int PER, bool FLAT, typename I>
__device__ __forceinline__ const uint4 *chunk_ptr(const void *x, I idx, I cpr, I ld) {
  const I off = FLAT ? idx * PER : (idx / cpr) * ld + (idx % cpr) * PER;
  return reinterpret_cast<const uint4 *>(static_cast<const char *>(x) +
                                         static_cast<int64_t>(off) * (16 / PER));
}

constexpr int kUnroll = 4;                         // 16-byte loads in flight per thread

// BF16 (PER = 8 elements per chunk): the max of the 16-bit |x| patterns in
// two lanes, shifted into FP32 position, is the FP32 bit pattern of the amax.
// FP32 (PER = 4): the max of the 32-bit |x| patterns.
template <int PER, bool FLAT, typename I>
__global__ void __launch_bounds__(kThreads)
amax_kernel(const void *__restrict__ x, I rows, I cols, I ld, unsigned *__restrict__ out) {
  const I cpr = cols / PER, total = rows * cpr;
  const I stride = static_cast<I>(gridDim.x) * kThreads;
  uint32_t acc = 0;
  for (I i = static_cast<I>(blockIdx.x) * kThreads + threadIdx.x; i < total;
       i += kUnroll * stride) {
    uint4 v[kUnroll];
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      const I idx = i + j * stride;
      v[j] = idx < total ? __ldg(chunk_ptr<PER, FLAT, I>(x, idx, cpr, ld)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      if (PER == 8) {
        acc = __vmaxu2(acc, v[j].x & 0x7FFF7FFFu); acc = __vmaxu2(acc, v[j].y & 0x7FFF7FFFu);
        acc = __vmaxu2(acc, v[j].z & 0x7FFF7FFFu); acc = __vmaxu2(acc, v[j].w & 0x7FFF7FFFu);
      } else {
        acc = max(acc, max(max(v[j].x & 0x7FFFFFFFu, v[j].y & 0x7FFFFFFFu),
                           max(v[j].z & 0x7FFFFFFFu, v[j].w & 0x7FFFFFFFu)));
      }
    }
  }
  const uint32_t m = PER == 8 ? max(acc & 0xFFFFu, acc >> 16) << 16 : acc;
  block_max_to_global(m, out);
}

template <int PER, bool FLAT>
void launch_k(const void *x, int64_t rows, int64_t cols, int64_t ld, unsigned *out, int grid,
              const Launch &L) {
  // 32-bit indices when every chunk index and offset a step can reach fits
  const int64_t reach = rows * (ld > cols ? ld : cols) + int64_t{kUnroll} * grid * kThreads * PER;
  if (reach < (int64_t{1} << 31))
    amax_kernel<PER, FLAT, uint32_t><<<grid, kThreads, 0, L.stream>>>(
        x, static_cast<uint32_t>(rows), static_cast<uint32_t>(cols), static_cast<uint32_t>(ld),
        out);
  else
    amax_kernel<PER, FLAT, int64_t><<<grid, kThreads, 0, L.stream>>>(x, rows, cols, ld, out);
}

}  // namespace

cudaError_t launch_amax(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                        float *amax_out, const Launch &L) {
  cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), L.stream);
  if (e != cudaSuccess) return e;
  const int per = dtype == FP4Q_BF16 ? 8 : 4;
  const int64_t chunks = rows * cols / per;
  const int64_t want = (chunks + kUnroll * kThreads - 1) / (kUnroll * kThreads);
  const int64_t cap = static_cast<int64_t>(L.num_sms) * 8;
  const int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
  unsigned *out = reinterpret_cast<unsigned *>(amax_out);
  const bool flat = ld == cols || rows == 1;
  if (dtype == FP4Q_BF16) {
    if (flat) launch_k<8, true>(x, rows, cols, ld, out, grid, L);
    else launch_k<8, false>(x, rows, cols, ld, out, grid, L);
  } else {
    if (flat) launch_k<4, true>(x, rows, cols, ld, out, grid, L);
    else launch_k<4, false>(x, rows, cols, ld, out, grid, L);
  }
  return cudaGetLastError();
}

}  // namespace fp4q
