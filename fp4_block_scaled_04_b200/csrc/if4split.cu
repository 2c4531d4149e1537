// if4split.cu -- IF4 operands for the block-scaled tensor-core GEMM.
//
// "Adaptive Block-Scaled Data Types" explainer, section 2: an IF4 block is
// either FP4 (E2M1 codes times the E4M3 scale S) or INT4 (k in -7..7, value
// k * RN(6/7) * S), flagged by the scale's sign bit.  The tensor core's
// block-scaled MMA multiplies E2M1 codes by E4M3 block scales only, and
// RN(6/7) * S is not an E4M3 value, so an INT4 block cannot be fed as it is.
// Every k in -7..7 is the sum of at most two E2M1 values (5 = 4 + 1 and
// 7 = 6 + 1, the others are E2M1 values themselves), so an IF4 operand A is
// split into three NVFP4 operands that share the unflagged scales:
//   A_fp: the FP4 blocks (INT4 blocks zero),
//   A_1, A_2: the two E2M1 parts of each INT4 block (FP4 blocks zero),
// and A B^T = A_fp B^T + RN(6/7) (A_1 B^T + A_2 B^T) up to rounding (one GEMM
// pass with two accumulators, in gemm.cu).  One
// thread per 16-value block: 8 code bytes and a scale byte in, three times 8
// code bytes and a scale byte out.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;

// nibble n (k in two's complement) -> E2M1 code of the first / second part of
// k: 0 1 2 3 4 5=4+1 6 7=6+1, and the negatives (-8, never written, is -6-2)
constexpr uint64_t kPart1 = 0xACDEEFFF77665420ull;
constexpr uint64_t kPart2 = 0x0000A0AC20200000ull;

__device__ __forceinline__ uint32_t split_word(uint32_t w, uint64_t table) {
  uint32_t o = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t n = (w >> (4 * i)) & 0xFu;
    o |= static_cast<uint32_t>((table >> (4 * n)) & 0xFu) << (4 * i);
  }
  return o;
}

__global__ void __launch_bounds__(kThreads)
if4_split_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ sf, int64_t rows,
                 int64_t bpr, int scale_layout, uint8_t *__restrict__ q_fp,
                 uint8_t *__restrict__ q_k1, uint8_t *__restrict__ q_k2,
                 uint8_t *__restrict__ sf_plain) {
  const int64_t nblk = rows * bpr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; b < nblk;
       b += stride) {
    const int64_t r = b / bpr, cb = b - r * bpr;
    const int64_t so = scale_offset(r, cb, bpr, scale_layout);
    const uint32_t s = __ldg(sf + so);
    const uint2 w = __ldg(reinterpret_cast<const uint2 *>(q + b * 8));   // dense codes
    const uint2 zero = make_uint2(0u, 0u);
    uint2 fp = w, k1 = zero, k2 = zero;
    if (s & 0x80u) {                                    // INT4 block
      fp = zero;
      k1 = make_uint2(split_word(w.x, kPart1), split_word(w.y, kPart1));
      k2 = make_uint2(split_word(w.x, kPart2), split_word(w.y, kPart2));
    }
    reinterpret_cast<uint2 *>(q_fp)[b] = fp;
    reinterpret_cast<uint2 *>(q_k1)[b] = k1;
    reinterpret_cast<uint2 *>(q_k2)[b] = k2;
    sf_plain[so] = static_cast<uint8_t>(s & 0x7Fu);
  }
}

}  // namespace

cudaError_t launch_if4_split(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t K,
                             int scale_layout, uint8_t *q_fp, uint8_t *q_k1, uint8_t *q_k2,
                             uint8_t *sf_plain, const Launch &L) {
  const int64_t nblk = rows * (K / 16);
  const int64_t want = (nblk + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(L.num_sms) * 8;
  const int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
  if4_split_kernel<<<grid, kThreads, 0, L.stream>>>(q, sf, rows, K / 16, scale_layout, q_fp,
                                                      q_k1, q_k2, sf_plain);
  return cudaGetLastError();
}

}  // namespace fp4q
