// mxfp6.cu -- MXFP6 (OCP FP6 E2M3 / E3M2 with E8M0 block scales), quantize
// and dequantize.
//
// "FP6から考えるLLM量子化" (blog.ast.moe), "FP6で隣り合う値の間隔を見てみる":
// E3M2 spends its bits on range (largest 28), E2M3 on spacing (largest 7.5);
// 32 values share one power-of-two (E8M0) scale as in MXFP4.  Elements
// v = RN(x * 2^-e) are rounded to nearest even with saturation by the sm_100a
// conversion cvt.rn.satfinite.{e2m3x2,e3m2x2}.f32, which leaves each 6-bit code
// in the low bits of a byte.  Four codes are packed into three bytes, code j
// of a group in bits 6j..6j+5 of the little-endian 24-bit word, so a block of
// 32 values is 24 code bytes.
//
// Decoding unpacks the 24-bit groups back into byte containers, converts
// pairs with cvt.rn.f16x2.{e2m3x2,e3m2x2} (every FP6 value is exact in f16)
// and multiplies by 2^e.
#include <cuda_fp16.h>

#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;

// two values -> two 6-bit codes in the low bits of bytes 0 and 1 (lo first)
template <int F6>
__device__ __forceinline__ uint32_t fp6x2(float lo, float hi) {
  uint16_t r;
  if (F6 == FP4Q_FP6_E2M3)
    asm("cvt.rn.satfinite.e2m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  else
    asm("cvt.rn.satfinite.e3m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// two byte containers (code 0 in byte 0) -> the two values in f16x2
template <int F6>
__device__ __forceinline__ uint32_t fp6x2_to_f16x2(uint32_t two_bytes) {
  uint32_t h;
  const uint16_t w = static_cast<uint16_t>(two_bytes);
  if (F6 == FP4Q_FP6_E2M3)
    asm("cvt.rn.f16x2.e2m3x2 %0, %1;" : "=r"(h) : "h"(w));
  else
    asm("cvt.rn.f16x2.e3m2x2 %0, %1;" : "=r"(h) : "h"(w));
  return h;
}

__device__ __forceinline__ float2 half2_bits_to_f32x2(uint32_t h) {
  __half2 v;
  memcpy(&v, &h, sizeof(v));
  return __half22float2(v);
}

// Quantize: one thread per 32-value block (64 or 128 bytes in, 24 code
// bytes and a scale byte out).  Four lanes per block with a shuffled block
// maximum moved the same bytes more slowly on B200: the shuffles and the
// per-lane exponent cost more issue slots than the wider per-thread loads
// lose.  I is the index type (32-bit when the tensor allows).
template <typename T, int F6, typename I>
__global__ void __launch_bounds__(kThreads)
mxfp6_kernel(const T *__restrict__ x, I rows, I cols, I ld, int mode, uint8_t *__restrict__ q,
             uint8_t *__restrict__ sf, int scale_layout) {
  const float qmax = F6 == FP4Q_FP6_E2M3 ? 7.5f : 28.0f;
  const float inv_qmax = F6 == FP4Q_FP6_E2M3 ? 1.0f / 7.5f : 1.0f / 28.0f;
  const int emax = F6 == FP4Q_FP6_E2M3 ? 2 : 4;
  const I bpr = cols / 32, nblk = rows * bpr;
  const I stride = static_cast<I>(gridDim.x) * kThreads;
  for (I b = static_cast<I>(blockIdx.x) * kThreads + threadIdx.x; b < nblk; b += stride) {
    const I r = b / bpr, cb = b - r * bpr;
    float v[32];
    load_values<32, T>(x + r * ld + cb * 32, v);
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < 32; ++k) m = fmaxf(m, fabsf(v[k]));
    const uint32_t byte =
        static_cast<uint32_t>(e8m0_exponent_q(m, mode, qmax, inv_qmax, emax) + 127);
    const float inv = e8m0_inverse(byte);
    uint32_t g[8];                                     // 24-bit groups
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 a = mul2(make_float2(v[4 * j], v[4 * j + 1]), make_float2(inv, inv));
      const float2 c = mul2(make_float2(v[4 * j + 2], v[4 * j + 3]), make_float2(inv, inv));
      const uint32_t p01 = fp6x2<F6>(a.x, a.y), p23 = fp6x2<F6>(c.x, c.y);
      g[j] = (p01 & 0x3Fu) | ((p01 >> 8) & 0x3Fu) << 6 | (p23 & 0x3Fu) << 12 |
             ((p23 >> 8) & 0x3Fu) << 18;
    }
    uint2 *dst = reinterpret_cast<uint2 *>(q + b * 24);   // codes are dense: row r starts at r * rb
    dst[0] = make_uint2(g[0] | g[1] << 24, g[1] >> 8 | g[2] << 16);
    dst[1] = make_uint2(g[2] >> 16 | g[3] << 8, g[4] | g[5] << 24);
    dst[2] = make_uint2(g[5] >> 8 | g[6] << 16, g[6] >> 16 | g[7] << 8);
    sf[scale_offset(r, cb, bpr, scale_layout)] = static_cast<uint8_t>(byte);
  }
}

// Dequantize: the codes and the output are dense, so the walk is flat in
// units of 8 values (6 code bytes, one 16- or 32-byte store), consecutive
// units on consecutive lanes, NU units per lane per step.  A warp's step
// reads 32 * NU * 6 = 768 contiguous code bytes; they are fetched as 16-byte
// pieces (one step ahead, so the loads overlap the decoding of the step
// before), staged in shared memory, and each lane picks out its 6 bytes.
constexpr int NU = 4;
constexpr int kStepBytes = 32 * NU * 6;                 // 768
constexpr int kPieces = kStepBytes / 16;                // 48

// the warp's code bytes for the step starting at unit wb (vb valid bytes, a
// multiple of 24): lane's pieces lane and lane + 32
__device__ __forceinline__ void fetch_step(const uint8_t *src, int64_t vb, int lane,
                                           uint4 (&c)[2]) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int k = lane + 32 * i;
    c[i] = make_uint4(0, 0, 0, 0);
    if (k < kPieces) {
      if (k * 16 + 16 <= vb) {
        c[i] = __ldg(reinterpret_cast<const uint4 *>(src + k * 16));
      } else if (k * 16 + 8 <= vb) {
        const uint2 h = __ldg(reinterpret_cast<const uint2 *>(src + k * 16));
        c[i] = make_uint4(h.x, h.y, 0, 0);
      }
    }
  }
}

template <typename OutT, int F6, typename I>
__global__ void __launch_bounds__(kThreads)
mxfp6_dequant_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ sf,
                     int scale_layout, I rows, I cols, OutT *__restrict__ y) {
  __shared__ __align__(16) uint8_t stage[kThreads / 32][kStepBytes];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const I nunits = rows * (cols / 8), bpr = cols / 32;
  const I warp = (static_cast<I>(blockIdx.x) * kThreads + threadIdx.x) / 32;
  const I step = static_cast<I>(gridDim.x) * (kThreads / 32) * (32 * NU);
  const auto valid_bytes = [&](I wb) -> int64_t {
    if (wb >= nunits) return 0;
    const I left = nunits - wb;
    return static_cast<int64_t>(left < 32 * NU ? left : 32 * NU) * 6;
  };
  I wb = warp * (32 * NU);
  uint4 cur[2];
  fetch_step(q + static_cast<int64_t>(wb) * 6, valid_bytes(wb), lane, cur);
  for (; wb < nunits; wb += step) {
    uint4 nxt[2];
    fetch_step(q + static_cast<int64_t>(wb + step) * 6, valid_bytes(wb + step), lane, nxt);
#pragma unroll
    for (int i = 0; i < 2; ++i)
      if (lane + 32 * i < kPieces)
        *reinterpret_cast<uint4 *>(&stage[wid][(lane + 32 * i) * 16]) = cur[i];
    __syncwarp();
    uint32_t g[NU][2], sb[NU];
#pragma unroll
    for (int j = 0; j < NU; ++j) {
      const uint8_t *src = &stage[wid][(32 * j + lane) * 6];
      if ((lane & 1) == 0) {                           // 6 * unit is a multiple of 4
        const uint32_t a = *reinterpret_cast<const uint32_t *>(src);
        const uint32_t h = *reinterpret_cast<const uint16_t *>(src + 4);
        g[j][0] = a & 0xFFFFFFu;
        g[j][1] = a >> 24 | h << 8;
      } else {
        const uint32_t h = *reinterpret_cast<const uint16_t *>(src);
        const uint32_t a = *reinterpret_cast<const uint32_t *>(src + 2);
        g[j][0] = h | (a & 0xFFu) << 16;
        g[j][1] = a >> 8;
      }
      const I u = wb + 32 * j + lane;
      sb[j] = 127;
      if (u < nunits) {
        const I blk = u / 4, r = blk / bpr;
        sb[j] = __ldg(sf + scale_offset(r, blk - r * bpr, bpr, scale_layout));
      }
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 2; ++i) cur[i] = nxt[i];
#pragma unroll
    for (int j = 0; j < NU; ++j) {
      const I u = wb + 32 * j + lane;
      if (u >= nunits) continue;
      const float p = e8m0_value(sb[j]);
      float out[8];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // codes 0, 1 -> bytes 0, 1 of one container; codes 2, 3 of the other
        const uint32_t c01 = (g[j][h] & 0x3Fu) | ((g[j][h] >> 6) & 0x3Fu) << 8;
        const uint32_t c23 = ((g[j][h] >> 12) & 0x3Fu) | ((g[j][h] >> 18) & 0x3Fu) << 8;
        const float2 a = mul2(half2_bits_to_f32x2(fp6x2_to_f16x2<F6>(c01)), make_float2(p, p));
        const float2 b = mul2(half2_bits_to_f32x2(fp6x2_to_f16x2<F6>(c23)), make_float2(p, p));
        out[4 * h] = a.x; out[4 * h + 1] = a.y; out[4 * h + 2] = b.x; out[4 * h + 3] = b.y;
      }
      OutT *o = y + static_cast<int64_t>(u) * 8;
      if (sizeof(OutT) == 2) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __nv_bfloat162 h2 = __floats2bfloat162_rn(out[2 * k], out[2 * k + 1]);
          memcpy(&w[k], &h2, sizeof(uint32_t));
        }
        *reinterpret_cast<uint4 *>(o) = make_uint4(w[0], w[1], w[2], w[3]);
      } else {
        float4 *d = reinterpret_cast<float4 *>(o);
        d[0] = make_float4(out[0], out[1], out[2], out[3]);
        d[1] = make_float4(out[4], out[5], out[6], out[7]);
      }
    }
  }
}

// Grids are capped at 16 CTAs per SM (a grid-stride loop covers the rest);
// the measured quantize time fell from 8 to 16 and was flat beyond.
int grid_for(int64_t work, int64_t per_cta, const Launch &L) {
  const int64_t want = (work + per_cta - 1) / per_cta;
  const int64_t cap = static_cast<int64_t>(L.num_sms) * 16;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

// 32-bit indices when every element offset, and every index a grid-stride
// step can reach, stays below 2^31
bool narrow(int64_t rows, int64_t cols, int64_t ld, int64_t step) {
  return rows * (ld > cols ? ld : cols) + 8 * step < (int64_t{1} << 31);
}

template <typename T, typename I>
void launch_q_i(const void *x, int64_t rows, int64_t cols, int64_t ld, int fmt, int mode,
                uint8_t *q, uint8_t *sf, int scale_layout, int grid, const Launch &L) {
  const T *p = static_cast<const T *>(x);
  if (fmt == FP4Q_FP6_E2M3)
    mxfp6_kernel<T, FP4Q_FP6_E2M3, I><<<grid, kThreads, 0, L.stream>>>(
        p, static_cast<I>(rows), static_cast<I>(cols), static_cast<I>(ld), mode, q, sf,
        scale_layout);
  else
    mxfp6_kernel<T, FP4Q_FP6_E3M2, I><<<grid, kThreads, 0, L.stream>>>(
        p, static_cast<I>(rows), static_cast<I>(cols), static_cast<I>(ld), mode, q, sf,
        scale_layout);
}

template <typename T>
cudaError_t launch_q(const void *x, int64_t rows, int64_t cols, int64_t ld, int fmt, int mode,
                     uint8_t *q, uint8_t *sf, int scale_layout, const Launch &L) {
  const int grid = grid_for(rows * (cols / 32), kThreads, L);
  if (narrow(rows, cols, ld, int64_t{grid} * kThreads * 32))
    launch_q_i<T, uint32_t>(x, rows, cols, ld, fmt, mode, q, sf, scale_layout, grid, L);
  else
    launch_q_i<T, int64_t>(x, rows, cols, ld, fmt, mode, q, sf, scale_layout, grid, L);
  return cudaGetLastError();
}

template <typename OutT, typename I>
void launch_dq_i(const uint8_t *q, const uint8_t *sf, int scale_layout, int64_t rows,
                 int64_t cols, int fmt, void *y, int grid, const Launch &L) {
  OutT *o = static_cast<OutT *>(y);
  if (fmt == FP4Q_FP6_E2M3)
    mxfp6_dequant_kernel<OutT, FP4Q_FP6_E2M3, I><<<grid, kThreads, 0, L.stream>>>(
        q, sf, scale_layout, static_cast<I>(rows), static_cast<I>(cols), o);
  else
    mxfp6_dequant_kernel<OutT, FP4Q_FP6_E3M2, I><<<grid, kThreads, 0, L.stream>>>(
        q, sf, scale_layout, static_cast<I>(rows), static_cast<I>(cols), o);
}

template <typename OutT>
cudaError_t launch_dq(const uint8_t *q, const uint8_t *sf, int scale_layout, int64_t rows,
                      int64_t cols, int fmt, void *y, const Launch &L) {
  const int grid = grid_for(rows * (cols / 8), kThreads * NU, L);
  if (narrow(rows, cols, cols, int64_t{grid} * kThreads * NU * 8))
    launch_dq_i<OutT, uint32_t>(q, sf, scale_layout, rows, cols, fmt, y, grid, L);
  else
    launch_dq_i<OutT, int64_t>(q, sf, scale_layout, rows, cols, fmt, y, grid, L);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mxfp6(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                         int fp6_format, int e8m0_mode, uint8_t *q, uint8_t *sf,
                         int scale_layout, const Launch &L) {
  if (dtype == FP4Q_BF16)
    return launch_q<__nv_bfloat16>(x, rows, cols, ld, fp6_format, e8m0_mode, q, sf, scale_layout,
                                   L);
  return launch_q<float>(x, rows, cols, ld, fp6_format, e8m0_mode, q, sf, scale_layout, L);
}

cudaError_t launch_mxfp6_dequant(const uint8_t *q, const uint8_t *sf, int scale_layout,
                                 int64_t rows, int64_t cols, int fp6_format, void *y,
                                 int y_dtype, const Launch &L) {
  if (y_dtype == FP4Q_BF16)
    return launch_dq<__nv_bfloat16>(q, sf, scale_layout, rows, cols, fp6_format, y, L);
  return launch_dq<float>(q, sf, scale_layout, rows, cols, fp6_format, y, L);
}

}  // namespace fp4q
