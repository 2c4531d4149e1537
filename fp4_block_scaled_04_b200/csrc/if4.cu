// if4.cu -- IF4 adaptive block-scaled quantization, row-wise 1x16.
//
// "Adaptive Block-Scaled Data Types" (gist.science explainer), section 2
// (IF4): every 16-value block is quantized both as FP4 (E2M1) and as INT4,
// the one with the smaller squared error is kept, and the choice goes into
// the otherwise unused sign bit of the block's E4M3 scale.  The 6/7 method
// maps INT4's range 0..7 onto FP4's 0..6: values are multiplied by 7/6
// before rounding to an integer and by 6/7 when decoded.
//
// A thread quantizes two adjacent blocks at once: every elementwise step is
// one f32x2 instruction whose lanes are (block A element k, block B element
// k), so each lane still sums its own block's squared errors in order
// k = 0..15, as the definition requires.
//   FP4:  codes by cvt.rn.satfinite.e2m1x2, values back by cvt.f16x2.e2m1x2
//   INT4: k = rint(t), t = RN(v * RN(7/6)), as RN(t + 1.5 * 2^23) - 1.5 * 2^23
//         (exact round-half-even for |t| < 2^22; the sum's low bits hold k in
//         two's complement); the clamp to [-7, 7] only matters when the
//         block's largest |t| reaches 7.5, which is tested once per block.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23

// E2M1 values of the two nibbles of a byte, via the sm_100a conversion to f16x2
__device__ __forceinline__ float2 e2m1_byte_values(uint32_t byte) {
  uint32_t h2;
  asm("{\n\t.reg .b8 q;\n\t.reg .b16 w;\n\t"
      "cvt.u16.u32 w, %1;\n\t"
      "cvt.u8.u16 q, w;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, q;\n\t}"
      : "=r"(h2) : "r"(byte));
  const __half2 h = *reinterpret_cast<const __half2 *>(&h2);
  return __half22float2(h);
}

template <typename T, bool CLAMP>
__device__ __forceinline__ void if4_pair(const float (&xa)[16], const float (&xb)[16], float fa,
                                         float fb, float c76, float c67, uint32_t (&wa)[2],
                                         uint32_t (&wb)[2], bool &int_a, bool &int_b) {
  float2 v[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = mul2(make_float2(xa[k], xb[k]), make_float2(fa, fb));
  // FP4 candidate codes (row order within each block)
  uint32_t fpa[2], fpb[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float ta[8], tb[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) { ta[k] = v[8 * h + k].x; tb[k] = v[8 * h + k].y; }
    fpa[h] = e2m1x8(ta);
    fpb[h] = e2m1x8(tb);
  }
  float2 efp = make_float2(0.0f, 0.0f), eint = make_float2(0.0f, 0.0f);
  uint32_t ia[2] = {0u, 0u}, ib[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 16; k += 2) {
    const int h = k >> 3, sh = 4 * (k & 7);
    const float2 ga = e2m1_byte_values((fpa[h] >> sh) & 0xFFu);   // block A, k and k+1
    const float2 gb = e2m1_byte_values((fpb[h] >> sh) & 0xFFu);
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const float2 vk = v[k + s];
      const float2 g = s == 0 ? make_float2(ga.x, gb.x) : make_float2(ga.y, gb.y);
      // No product below feeds a packed add or subtract: ptxas may contract a
      // mul.f32x2 -> add.f32x2 pair into one fused operation even with .rn,
      // which rounds once instead of twice.  Products that are added to are
      // scalar __fmul_rn / __fadd_rn / __fsub_rn, which are never fused.
      // t = RN(v * RN(7/6)) and RN(t + 1.5 * 2^23) = rint(t) + 1.5 * 2^23 are
      // scalar __fmul_rn / __fadd_rn, which are never merged into an FMA
      float tx = __fmul_rn(vk.x, c76), ty = __fmul_rn(vk.y, c76);
      if (CLAMP) {
        tx = fminf(fmaxf(tx, -7.25f), 7.25f);
        ty = fminf(fmaxf(ty, -7.25f), 7.25f);
      }
      const float2 tm = make_float2(__fadd_rn(tx, kMagic), __fadd_rn(ty, kMagic));
      const float2 kf = sub2(tm, make_float2(kMagic, kMagic));    // rint(t), exact
      const float2 hv = mul2(kf, make_float2(c67, c67));
      const float2 dfp = make_float2(__fsub_rn(vk.x, g.x), __fsub_rn(vk.y, g.y));
      const float2 dint = make_float2(__fsub_rn(vk.x, hv.x), __fsub_rn(vk.y, hv.y));
      efp = fma2(dfp, dfp, efp);
      eint = fma2(dint, dint, eint);
      ia[h] |= (__float_as_uint(tm.x) & 0xFu) << (sh + 4 * s);
      ib[h] |= (__float_as_uint(tm.y) & 0xFu) << (sh + 4 * s);
    }
  }
  int_a = eint.x < efp.x;
  int_b = eint.y < efp.y;
  wa[0] = int_a ? ia[0] : fpa[0];
  wa[1] = int_a ? ia[1] : fpa[1];
  wb[0] = int_b ? ib[0] : fpb[0];
  wb[1] = int_b ? ib[1] : fpb[1];
}

template <typename T>
__device__ __forceinline__ void load_pair(const T *p, float (&xa)[16], float (&xb)[16],
                                          float &ma, float &mb) {
  if (sizeof(T) == 2) {
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
    const uint4 u0 = __ldg(q), u1 = __ldg(q + 1), u2 = __ldg(q + 2), u3 = __ldg(q + 3);
    ma = bf16x2_hmax(maxabs_bf16x2(maxabs_bf16x2(maxabs_bf16x2(u0.x, u0.y), maxabs_bf16x2(u0.z, u0.w)),
                                   maxabs_bf16x2(maxabs_bf16x2(u1.x, u1.y), maxabs_bf16x2(u1.z, u1.w))));
    mb = bf16x2_hmax(maxabs_bf16x2(maxabs_bf16x2(maxabs_bf16x2(u2.x, u2.y), maxabs_bf16x2(u2.z, u2.w)),
                                   maxabs_bf16x2(maxabs_bf16x2(u3.x, u3.y), maxabs_bf16x2(u3.z, u3.w))));
    const uint32_t wa[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    const uint32_t wb[8] = {u2.x, u2.y, u2.z, u2.w, u3.x, u3.y, u3.z, u3.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      xa[2 * i] = bf16_lo(wa[i]); xa[2 * i + 1] = bf16_hi(wa[i]);
      xb[2 * i] = bf16_lo(wb[i]); xb[2 * i + 1] = bf16_hi(wb[i]);
    }
  } else {
    const float4 *q = reinterpret_cast<const float4 *>(p);
    ma = mb = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 a = __ldg(q + i), b = __ldg(q + 4 + i);
      xa[4 * i] = a.x; xa[4 * i + 1] = a.y; xa[4 * i + 2] = a.z; xa[4 * i + 3] = a.w;
      xb[4 * i] = b.x; xb[4 * i + 1] = b.y; xb[4 * i + 2] = b.z; xb[4 * i + 3] = b.w;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      ma = fmaxf(ma, fabsf(xa[k]));
      mb = fmaxf(mb, fabsf(xb[k]));
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 2)
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

  // work unit: a pair of adjacent blocks (b, b+1) of one row; an odd last
  // block of a row pairs with itself
  const int64_t bpr = cols / 16, ppr = (bpr + 1) / 2, npairs = rows * ppr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t p = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; p < npairs;
       p += stride) {
    const int64_t r = p / ppr, cb = 2 * (p - r * ppr);
    const bool has_b = cb + 1 < bpr;
    float xa[16], xb[16], ma, mb;
    if (has_b) {
      load_pair<T>(x + r * ld + cb * 16, xa, xb, ma, mb);
    } else {
      // a single trailing block: load it into both lanes (the copy is discarded)
      if (sizeof(T) == 2) {
        const uint4 *qq = reinterpret_cast<const uint4 *>(x + r * ld + cb * 16);
        const uint4 u0 = __ldg(qq), u1 = __ldg(qq + 1);
        ma = bf16x2_hmax(maxabs_bf16x2(maxabs_bf16x2(maxabs_bf16x2(u0.x, u0.y), maxabs_bf16x2(u0.z, u0.w)),
                                       maxabs_bf16x2(maxabs_bf16x2(u1.x, u1.y), maxabs_bf16x2(u1.z, u1.w))));
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) { xa[2 * i] = bf16_lo(w[i]); xa[2 * i + 1] = bf16_hi(w[i]); }
      } else {
        const float4 *qq = reinterpret_cast<const float4 *>(x + r * ld + cb * 16);
        ma = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 a = __ldg(qq + i);
          xa[4 * i] = a.x; xa[4 * i + 1] = a.y; xa[4 * i + 2] = a.z; xa[4 * i + 3] = a.w;
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) ma = fmaxf(ma, fabsf(xa[k]));
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) xb[k] = xa[k];
      mb = ma;
    }
    const uint32_t sa = nvfp4_scale_code(ma, ts.enc), sb = nvfp4_scale_code(mb, ts.enc);
    const float fa = rtab[sa], fb = rtab[sb];
    // |t| of the block maximum: the clamp can only bind when it reaches 7.5
    const float ta = __fmul_rn(__fmul_rn(ma, fa), c76), tb = __fmul_rn(__fmul_rn(mb, fb), c76);
    uint32_t wa[2], wb[2];
    bool ia, ib;
    if (ta < 7.5f && tb < 7.5f)
      if4_pair<T, false>(xa, xb, fa, fb, c76, c67, wa, wb, ia, ib);
    else
      if4_pair<T, true>(xa, xb, fa, fb, c76, c67, wa, wb, ia, ib);
    uint8_t *qp = q + r * (cols / 2) + cb * 8;
    if (has_b) {
      if ((cols & 31) == 0) {
        *reinterpret_cast<uint4 *>(qp) = make_uint4(wa[0], wa[1], wb[0], wb[1]);
      } else {  // rows of codes are only 8-byte aligned
        *reinterpret_cast<uint2 *>(qp) = make_uint2(wa[0], wa[1]);
        *reinterpret_cast<uint2 *>(qp + 8) = make_uint2(wb[0], wb[1]);
      }
      sf[scale_offset(r, cb + 1, bpr, scale_layout)] = static_cast<uint8_t>(sb | (ib ? 0x80u : 0u));
    } else {
      *reinterpret_cast<uint2 *>(qp) = make_uint2(wa[0], wa[1]);
    }
    sf[scale_offset(r, cb, bpr, scale_layout)] = static_cast<uint8_t>(sa | (ia ? 0x80u : 0u));
  }
}

}  // namespace

cudaError_t launch_if4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                       const float *amax, float *s_dec_out, uint8_t *q, uint8_t *sf,
                       int scale_layout, const Launch &L) {
  const int64_t npairs = rows * ((cols / 16 + 1) / 2);
  int64_t want = (npairs + kThreads - 1) / kThreads;
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
