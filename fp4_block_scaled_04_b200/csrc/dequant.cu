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
// The codes [rows, cols/2] and the output [rows, cols] are both dense, so the
// kernel walks the flat element range in units of 8 elements (4 code bytes,
// one 16-byte BF16 store), consecutive units on consecutive lanes, four
// units per lane per step, and loads the next step's codes and scale bytes
// before it decodes this step's, so that eight loads are in flight.  With a linear
// 1x16 or 1x32 scale matrix the scale index is the flat element index / 16
// (or / 32), so the walk needs no row and column; the swizzled and
// 16x16-tile layouts carry (row, column) along with a fixed stride.
//
// Arithmetic: E2M1 pairs decode with cvt.rn.f16x2.e2m1x2 and E4M3 scales
// with cvt.rn.f16x2.e4m3x2.  g * S is exact in f16 (at most 6 significant
// bits, within [2^-10, 2688]).  IF4 blocks are decoded without branching on
// the per-block flag (neighbouring threads hold blocks of either kind): the
// f16 pair is the E2M1 pair or the INT4 pair k = (1024 + (n ^ 8)) - 1032 (exact
// in f16), then RN(pair * m) with m = 1 (FP4) or RN(6/7) (INT4), RN(* S),
// RN(* s_dec), all in FP32 -- for FP4 blocks the first two products are exact
// and the result equals RN(RN(g * S) * s_dec).
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;

// (S, S) in f16 from a 7-bit E4M3 code
__device__ __forceinline__ uint32_t e4m3_to_f16x2_dup(uint32_t code7) {
  uint32_t h2;
  const uint16_t w = static_cast<uint16_t>(code7 * 0x0101u);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(w));
  return h2;
}

__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t hsub2_bits(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t h) {
  const __half2 v = *reinterpret_cast<const __half2 *>(&h);
  return __half22float2(v);
}

struct Store {
  __device__ __forceinline__ static void put(float *y, const float2 (&v)[4]) {
    float4 *p = reinterpret_cast<float4 *>(y);
    p[0] = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
    p[1] = make_float4(v[2].x, v[2].y, v[3].x, v[3].y);
  }
  __device__ __forceinline__ static void put(__nv_bfloat16 *y, const float2 (&v)[4]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[i].x, v[i].y);
      w[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(y) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// The four E2M1 pairs of a code word as f16x2 (byte i -> element pair i).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t codes, uint32_t (&h)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(codes));
}

// The four INT4 pairs of a code word as f16x2 k values: for byte i the
// permute puts its low nibble in bits 0..3 and (from codes >> 4) its high
// nibble in bits 16..19; then 1024 + (n ^ 8) - 1032 = k exactly in f16.
__device__ __forceinline__ void int4x8_to_f16x2(uint32_t codes, uint32_t (&h)[4]) {
  const uint32_t hi = codes >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t t = (__byte_perm(codes, hi, 0x0400u | (0x0101u * i)) & 0x000F000Fu) ^ 0x64086408u;
    h[i] = hsub2_bits(t, 0x64086408u);
  }
}

// 8 values of one unit: 4 code bytes (element 2i in the low nibble)
template <int FMT>
__device__ __forceinline__ void decode8(uint32_t codes, uint32_t sbyte, float s_dec, float c67,
                                        float2 (&v)[4]) {
  const float2 sd = make_float2(s_dec, s_dec);
  uint32_t g[4];
  e2m1x8_to_f16x2(codes, g);
  if (FMT == FP4Q_FMT_MXFP4) {
    const float p = e8m0_value(sbyte);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = mul2(f16x2_to_f32x2(g[i]), make_float2(p, p));
  } else if (FMT == FP4Q_FMT_NVFP4) {
    const uint32_t s2 = e4m3_to_f16x2_dup(sbyte & 0x7Fu);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = mul2(f16x2_to_f32x2(hmul2_bits(g[i], s2)), sd);
  } else {  // IF4
    const bool int4 = (sbyte & 0x80u) != 0;
    const uint32_t s2 = e4m3_to_f16x2_dup(sbyte & 0x7Fu);
    const float S = __half2float(__ushort_as_half(static_cast<unsigned short>(s2 & 0xFFFFu)));
    const float m = int4 ? c67 : 1.0f;
    const uint32_t pick = int4 ? 0xFFFFFFFFu : 0u;   // select, not branch, per pair
    uint32_t k[4];
    int4x8_to_f16x2(codes, k);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t h = (k[i] & pick) | (g[i] & ~pick);
      v[i] = mul2(mul2(mul2(f16x2_to_f32x2(h), make_float2(m, m)), make_float2(S, S)), sd);
    }
  }
}

// Byte offset of the scale of the 8-element unit starting at (r, c) (SWZ:
// the 128x4 tile layout; BROWS == 16: the linear [rows/16, cols/16] tile
// matrix).  I is the index type: 32-bit when every index fits.
template <int BLK, int BROWS, bool SWZ, typename I>
__device__ __forceinline__ I unit_scale(I r, I c, I cols) {
  const I sc = BLK == 32 ? (c >> 5) : (c >> 4);   // c, cols >= 0
  const I scols = BLK == 32 ? (cols >> 5) : (cols >> 4);
  if (BROWS == 16) return (r >> 4) * scols + sc;
  if (!SWZ) return r * scols + sc;
  const I tile = (r >> 7) * (scols >> 2) + (sc >> 2);
  return tile * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (sc & 3);
}

// A warp takes NU x 32 consecutive 8-element units per step, lane l the units
// l, l + 32, ...: every code load and output store of the warp is then one
// contiguous stretch, and a thread has NU independent loads in flight.
// ROWAL: cols % (NU * 32 * 8) == 0, so every row holds whole steps of a
// warp: the NU * 32 units of a warp's step lie in one row, lane l's at
// columns c + 256 j, all inside the matrix or all outside it, and the scale
// byte of unit j sits DS j bytes after that of unit 0.  One cursor step, one
// scale offset and one bound test per step then serve all NU units.
template <int FMT, int BROWS, bool SWZ, typename I, bool ROWAL, typename OutT>
__global__ void __launch_bounds__(kThreads)
dequant_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ sf,
               const float *__restrict__ s_dec_ptr, I rows, I cols, OutT *__restrict__ y) {
  constexpr int NU = 4;
  constexpr int BLK = FMT == FP4Q_FMT_MXFP4 ? 32 : 16;
  constexpr bool FLAT = !SWZ && BROWS == 1;          // scale index from the unit index
  const float s_dec = (FMT == FP4Q_FMT_MXFP4) ? 1.0f : *s_dec_ptr;
  const float c67 = __fdiv_rn(6.0f, 7.0f);
  const I total = rows * (cols / 8);                 // units
  const I lane = threadIdx.x & 31;
  const I warp0 = (static_cast<I>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const I wstride = static_cast<I>(gridDim.x) * (kThreads / 32);
  const uint32_t *qw = reinterpret_cast<const uint32_t *>(q);
  if (ROWAL) {
    constexpr I DS = SWZ ? (BLK == 32 ? 1024 : 2048) : (BLK == 32 ? 8 : 16);
    I rr = 0, cc = 0, dr1 = 0, dc1 = 0;               // row and column of unit 0
    if (!FLAT) {
      const I estride = wstride * NU * 32 * 8;
      dr1 = estride / cols;
      dc1 = estride - dr1 * cols;
      const I e = (warp0 * NU * 32 + lane) * 8;
      rr = e / cols;
      cc = e - rr * cols;
    }
    auto load1 = [&](I b, uint32_t (&w)[NU], uint32_t (&s8)[NU]) {
      const I si0 = FLAT ? (BLK == 32 ? (b >> 2) : (b >> 1))
                         : unit_scale<BLK, BROWS, SWZ, I>(rr, cc, cols);
#pragma unroll
      for (int j = 0; j < NU; ++j) {
        w[j] = __ldg(qw + b + 32 * j);
        s8[j] = __ldg(sf + si0 + DS * j);
      }
      if (!FLAT) {
        rr += dr1;
        cc += dc1;
        if (cc >= cols) {
          cc -= cols;
          ++rr;
        }
      }
    };
    const I step = wstride * NU * 32;
    uint32_t cw[NU], sb[NU];
    I base = warp0 * NU * 32 + lane;
    if (base < total) load1(base, cw, sb);
    for (; base < total; base += step) {
      uint32_t cn[NU], sn[NU];
      if (base + step < total) load1(base + step, cn, sn);
#pragma unroll
      for (int j = 0; j < NU; ++j) {
        float2 v[4];
        decode8<FMT>(cw[j], sb[j], s_dec, c67, v);
        Store::put(y + static_cast<size_t>(base + 32 * j) * 8, v);
      }
#pragma unroll
      for (int j = 0; j < NU; ++j) {
        cw[j] = cn[j];
        sb[j] = sn[j];
      }
    }
    return;
  }
  // (row, column) of each of the lane's NU units, advanced by a fixed stride
  I r[NU], c[NU];
  I dr = 0, dc = 0;
  if (!FLAT) {
    const I estride = wstride * NU * 32 * 8;         // elements per step
    dr = estride / cols;
    dc = estride - dr * cols;
#pragma unroll
    for (int j = 0; j < NU; ++j) {
      const I e = (warp0 * NU * 32 + 32 * j + lane) * 8;
      r[j] = e / cols;
      c[j] = e - r[j] * cols;
    }
  }
  // the codes and scale bytes of the lane's NU units of one step; the next
  // step's are loaded before this step decodes, so the loads overlap the
  // arithmetic (r, c: the units of the next step to load)
  uint32_t cw[NU], sb[NU];
  auto load = [&](I b, uint32_t (&w)[NU], uint32_t (&s8)[NU]) {
#pragma unroll
    for (int j = 0; j < NU; ++j) {
      const I u = b + 32 * j;
      if (u < total) {
        const I si = FLAT ? (BLK == 32 ? (u >> 2) : (u >> 1))
                          : unit_scale<BLK, BROWS, SWZ, I>(r[j], c[j], cols);
        w[j] = __ldg(qw + u);
        s8[j] = __ldg(sf + si);
      }
      if (!FLAT) {
        r[j] += dr;
        c[j] += dc;
        if (c[j] >= cols) {
          c[j] -= cols;
          ++r[j];
        }
      }
    }
  };
  const I step = wstride * NU * 32;
  I base = warp0 * NU * 32 + lane;
  if (base < total) load(base, cw, sb);
  for (; base < total; base += step) {
    uint32_t cn[NU], sn[NU];
    if (base + step < total) load(base + step, cn, sn);
#pragma unroll
    for (int j = 0; j < NU; ++j) {
      const I u = base + 32 * j;
      if (u < total) {
        float2 v[4];
        decode8<FMT>(cw[j], sb[j], s_dec, c67, v);
        Store::put(y + static_cast<size_t>(u) * 8, v);
      }
    }
#pragma unroll
    for (int j = 0; j < NU; ++j) {
      cw[j] = cn[j];
      sb[j] = sn[j];
    }
  }
}

template <int FMT, int BROWS, bool SWZ>
cudaError_t launch_fmt(const uint8_t *q, const uint8_t *sf, const float *s_dec, int64_t rows,
                       int64_t cols, void *y, int y_dtype, const Launch &L) {
  const int64_t units = rows * (cols / 8);
  const int64_t want = (units + 4 * kThreads - 1) / (4 * kThreads);
  const int64_t cap = static_cast<int64_t>(L.num_sms) * 8;
  const int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
  // 32-bit indices when the unit index, stepped once past the end, the
  // element index of a row start and the scale offsets all stay below 2^31
  const bool narrow = units + static_cast<int64_t>(grid) * 4 * kThreads < (int64_t(1) << 31) &&
                      rows * cols < (int64_t(1) << 31);
  const bool rowal = cols % (4 * 32 * 8) == 0;        // whole warp steps per row
  const uint32_t r32 = static_cast<uint32_t>(rows), c32 = static_cast<uint32_t>(cols);
  if (y_dtype == FP4Q_BF16) {
    auto *yp = static_cast<__nv_bfloat16 *>(y);
    if (narrow && rowal)
      dequant_kernel<FMT, BROWS, SWZ, uint32_t, true><<<grid, kThreads, 0, L.stream>>>(
          q, sf, s_dec, r32, c32, yp);
    else if (narrow)
      dequant_kernel<FMT, BROWS, SWZ, uint32_t, false><<<grid, kThreads, 0, L.stream>>>(
          q, sf, s_dec, r32, c32, yp);
    else
      dequant_kernel<FMT, BROWS, SWZ, int64_t, false><<<grid, kThreads, 0, L.stream>>>(
          q, sf, s_dec, rows, cols, yp);
  } else {
    auto *yp = static_cast<float *>(y);
    if (narrow && rowal)
      dequant_kernel<FMT, BROWS, SWZ, uint32_t, true><<<grid, kThreads, 0, L.stream>>>(
          q, sf, s_dec, r32, c32, yp);
    else if (narrow)
      dequant_kernel<FMT, BROWS, SWZ, uint32_t, false><<<grid, kThreads, 0, L.stream>>>(
          q, sf, s_dec, r32, c32, yp);
    else
      dequant_kernel<FMT, BROWS, SWZ, int64_t, false><<<grid, kThreads, 0, L.stream>>>(
          q, sf, s_dec, rows, cols, yp);
  }
  return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_layout(const uint8_t *q, const uint8_t *sf, int scale_layout,
                          const float *s_dec, int64_t rows, int64_t cols, void *y, int y_dtype,
                          const Launch &L) {
  if (scale_layout == FP4Q_SCALE_SWIZZLED_128x4)
    return launch_fmt<FMT, 1, true>(q, sf, s_dec, rows, cols, y, y_dtype, L);
  return launch_fmt<FMT, 1, false>(q, sf, s_dec, rows, cols, y, y_dtype, L);
}

}  // namespace

cudaError_t launch_dequant(int format, const uint8_t *q, const uint8_t *sf, int scale_layout,
                           int block_rows, int block_cols, const float *s_dec, int64_t rows,
                           int64_t cols, void *y, int y_dtype, const Launch &L) {
  (void)block_cols;
  if (format == FP4Q_FMT_MXFP4)
    return launch_layout<FP4Q_FMT_MXFP4>(q, sf, scale_layout, s_dec, rows, cols, y, y_dtype, L);
  if (format == FP4Q_FMT_IF4)
    return launch_layout<FP4Q_FMT_IF4>(q, sf, scale_layout, s_dec, rows, cols, y, y_dtype, L);
  if (block_rows == 16)
    return launch_fmt<FP4Q_FMT_NVFP4, 16, false>(q, sf, s_dec, rows, cols, y, y_dtype, L);
  return launch_layout<FP4Q_FMT_NVFP4>(q, sf, scale_layout, s_dec, rows, cols, y, y_dtype, L);
}

}  // namespace fp4q
