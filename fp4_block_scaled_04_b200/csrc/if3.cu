// if3.cu -- IF3: the IF per-block choice at 3 bits, quantize and dequantize.
//
// "Adaptive Block-Scaled Data Types" explainer, section 2: each 16-value
// block is quantized both to a float grid and to a scaled integer grid, the
// one with the smaller squared error is kept, and the scale's sign bit says
// which; the idea extends to 3 bits (IF3).  A 3-bit code is a sign and two
// magnitude bits.  The float split E1M1 would give the uniform magnitudes
// 0, 0.5, 1, 1.5 (INT3 times 0.5, nothing to choose between), so the float
// grid is E2M0, magnitudes 0, 1, 2, 4, against INT3 (-3..3) rescaled by 4/3
// (the 6/7 method with 3 and 4):
//
//   s_enc = RN(1792 / amax), s_dec = RN(amax / 1792)          (1792 = 4 * 448)
//   S = E4M3_rne_sat(RN(m * s_enc) / 4),  r = RN(s_enc / S),  v = RN(x * r)
//   FP3:  g = nearest of 0, 1, 2, 4 to |v| (ties to the even code, so 0.5 ->
//         0, 1.5 -> 2, 3 -> 2; saturating at 4), sign copied
//   INT3: k = clamp(rint(RN(v * 0.75)), -3, 3),  h = RN(k * RN(4/3))
//   e = sum over the block, in order, of fma(d, d, e) with d = RN(v - q)
//   INT3 iff e_int < e_fp; scale bit 7 flags INT3.
//
// Codes are 3 bits (sign in bit 2 and the magnitude's index, or k in two's
// complement), eight per three bytes (code j of a group in bits 3j..3j+2),
// so a block is 6 bytes.
// Quantize: one thread per pair of blocks, whose elements go through the
// arithmetic as the two lanes of f32x2 instructions; 64 or 128 bytes in,
// three 4-byte code stores and two scale bytes out; r comes from a per-CTA
// table over the 128 scale codes.  The FP3 rounding is three comparisons: with s1 = [|v| > 0.5],
// s2 = [|v| >= 1.5], s3 = [|v| > 3] the magnitude's index is s1 + s2 + s3 and
// its value s1 + s2 + 2 s3.  As in IF4, rint adds and subtracts 1.5 * 2^23;
// the low bits of that sum (and of the index plus 1.5 * 2^23) are packed by
// multiply-adds with the weights 8^j, and one subtraction takes the words'
// common high bits back out.
// Dequantize: one thread per block, y = RN(RN(q * S) * s_dec) with q the E2M0
// value or h.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;
constexpr float kDown = 4.0f / 3.0f;              // RN(4/3)
constexpr float kMagic = 12582912.0f;             // 1.5 * 2^23: RN(t + kMagic) - kMagic = rint(t)
// sum over j < 8 of 8^j, and the bias that eight words 0x4B400000 + n_j
// summed with weights 8^j carry beyond the sum of n_j 8^j (mod 2^32)
constexpr uint32_t kOctets = 0x249249u;
constexpr uint32_t kBiasFp = 0x4B400000u * kOctets;
constexpr uint32_t kBiasInt = (0x4B400000u - 4u) * kOctets;   // fields k + 4
constexpr uint32_t kSignBits = 0x924924u;                     // bit 2 of each field

__device__ __forceinline__ float set_gt(float a, float b) {
  float r;
  asm("set.gt.f32.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ float set_ge(float a, float b) {
  float r;
  asm("set.ge.f32.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// Both candidates of blocks A and B (lanes .x / .y): the packed codes of each
// (two 24-bit groups) and whether INT3 wins.  Each lane sums its own block's
// errors in element order.  No packed add or subtract consumes a product
// (ptxas may contract a mul.f32x2 -> add.f32x2 pair even with .rn); the
// additions that follow a product are scalar __fadd_rn / __fsub_rn.
template <bool CLAMP>
__device__ __forceinline__ void if3_pair(const float (&va)[16], const float (&vb)[16], float2 rf,
                                         uint32_t (&ga)[2], uint32_t (&gb)[2], bool &int_a,
                                         bool &int_b) {
  float2 e_fp = make_float2(0.0f, 0.0f), e_int = make_float2(0.0f, 0.0f);
  uint32_t fa[2] = {0u, 0u}, fb[2] = {0u, 0u}, ia[2] = {0u, 0u}, ib[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 16; ++k) {                       // element order, as the errors sum
    const int h = k >> 3;
    const uint32_t w8 = 1u << (3 * (k & 7));           // code k's weight in its group
    const float2 vv = mul2(make_float2(va[k], vb[k]), rf);
    const float ax = fabsf(vv.x), ay = fabsf(vv.y);
    const float2 s1 = make_float2(set_gt(ax, 0.5f), set_gt(ay, 0.5f));
    const float2 s2 = make_float2(set_ge(ax, 1.5f), set_ge(ay, 1.5f));
    const float2 s3 = make_float2(set_gt(ax, 3.0f), set_gt(ay, 3.0f));
    const float2 s12 = add2(s1, s2);
    const float2 g = fma2(s3, make_float2(2.0f, 2.0f), s12);   // 0, 1, 2 or 4 (exact)
    const float2 dfp = make_float2(__fsub_rn(ax, g.x), __fsub_rn(ay, g.y));
    e_fp = fma2(dfp, dfp, e_fp);
    const float2 idx = add2(add2(s12, make_float2(kMagic, kMagic)), s3);
    const uint32_t bx = __float_as_uint(vv.x), by = __float_as_uint(vv.y);
    fa[h] += (__float_as_uint(idx.x) + ((bx >> 31) << 2)) * w8;
    fb[h] += (__float_as_uint(idx.y) + ((by >> 31) << 2)) * w8;
    float2 t = mul2(vv, make_float2(0.75f, 0.75f));
    if (CLAMP) {
      t.x = fminf(fmaxf(t.x, -3.25f), 3.25f);
      t.y = fminf(fmaxf(t.y, -3.25f), 3.25f);
    }
    const float2 tm = make_float2(__fadd_rn(t.x, kMagic), __fadd_rn(t.y, kMagic));
    const float2 kf = sub2(tm, make_float2(kMagic, kMagic));   // rint(t), exact
    const float2 hv = mul2(kf, make_float2(kDown, kDown));
    const float2 dint = make_float2(__fsub_rn(vv.x, hv.x), __fsub_rn(vv.y, hv.y));
    e_int = fma2(dint, dint, e_int);
    ia[h] += __float_as_uint(tm.x) * w8;
    ib[h] += __float_as_uint(tm.y) * w8;
  }
  int_a = e_int.x < e_fp.x;
  int_b = e_int.y < e_fp.y;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    ga[h] = int_a ? (ia[h] - kBiasInt) ^ kSignBits : fa[h] - kBiasFp;
    gb[h] = int_b ? (ib[h] - kBiasInt) ^ kSignBits : fb[h] - kBiasFp;
  }
}

// Scale code, factor and clamp flag of one block.
struct BlockScale3 {
  uint32_t code;
  float rf;
  bool clamp;
};

__device__ __forceinline__ BlockScale3 block_scale3(const float (&v)[16], float s_enc,
                                                    const float *tab) {
  float m = 0.0f;
#pragma unroll
  for (int k = 0; k < 16; ++k) m = fmaxf(m, fabsf(v[k]));
  BlockScale3 b;
  b.code = scale_code_q<4>(m, s_enc);
  b.rf = tab[b.code];
  // |t| <= RN(RN(m * r) * 0.75) by monotonicity; only a block reaching 3.25
  // needs the clamp (which then makes rint land on +-3, as clamping rint(t)
  // to +-3 does).  A block whose scale is an E4M3 subnormal can get there.
  b.clamp = __fmul_rn(__fmul_rn(m, b.rf), 0.75f) > 3.25f;
  return b;
}

// One thread per pair of consecutive blocks (2p, 2p + 1) in row-major block
// order; the pair's 12 code bytes are contiguous.  With an odd block count
// the last thread's second block is a copy of its first and is not stored.
template <typename T, typename I>
__global__ void __launch_bounds__(kThreads, sizeof(I) == 4 ? 4 : 2)   // 64 registers with 32-bit indices
if3_kernel(const T *__restrict__ x, I rows, I cols, I ld, const float *__restrict__ amax,
           float *__restrict__ s_dec_out, uint8_t *__restrict__ q, uint8_t *__restrict__ sf,
           int scale_layout) {
  __shared__ float tab[128];
  const TensorScale ts = tensor_scale_q<4>(*amax);
  if (blockIdx.x == 0 && threadIdx.x == 0 && s_dec_out) *s_dec_out = ts.dec;
  fill_factor_table(tab, ts.enc);
  __syncthreads();
  const I bpr = cols / 16, nblk = rows * bpr, npairs = (nblk + 1) / 2;
  const I stride = static_cast<I>(gridDim.x) * kThreads;
  for (I p = static_cast<I>(blockIdx.x) * kThreads + threadIdx.x; p < npairs; p += stride) {
    const I b0 = 2 * p;
    const bool has_b = b0 + 1 < nblk;
    const I r0 = b0 / bpr, c0 = b0 - r0 * bpr;
    const I r1 = (c0 + 1 == bpr) ? r0 + 1 : r0, c1 = (c0 + 1 == bpr) ? 0 : c0 + 1;
    float va[16], vb[16];
    load_values<16, T>(x + r0 * ld + c0 * 16, va);
    if (has_b) {
      load_values<16, T>(x + r1 * ld + c1 * 16, vb);
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) vb[k] = va[k];
    }
    const BlockScale3 sa = block_scale3(va, ts.enc, tab), sb = block_scale3(vb, ts.enc, tab);
    uint32_t ga[2], gb[2];
    bool int_a, int_b;
    if (sa.clamp || sb.clamp)
      if3_pair<true>(va, vb, make_float2(sa.rf, sb.rf), ga, gb, int_a, int_b);
    else
      if3_pair<false>(va, vb, make_float2(sa.rf, sb.rf), ga, gb, int_a, int_b);
    sf[scale_offset(r0, c0, bpr, scale_layout)] = static_cast<uint8_t>(sa.code | (int_a ? 0x80u : 0u));
    if (has_b) {
      uint32_t *dst = reinterpret_cast<uint32_t *>(q + b0 * 6);   // 12 B, 4-byte aligned
      dst[0] = ga[0] | ga[1] << 24;
      dst[1] = ga[1] >> 8 | gb[0] << 16;
      dst[2] = gb[0] >> 16 | gb[1] << 8;
      sf[scale_offset(r1, c1, bpr, scale_layout)] = static_cast<uint8_t>(sb.code | (int_b ? 0x80u : 0u));
    } else {
      uint16_t *dst = reinterpret_cast<uint16_t *>(q + b0 * 6);
      dst[0] = static_cast<uint16_t>(ga[0]);
      dst[1] = static_cast<uint16_t>((ga[0] >> 16) | (ga[1] << 8));
      dst[2] = static_cast<uint16_t>(ga[1] >> 8);
    }
  }
}

template <typename OutT, typename I>
__global__ void __launch_bounds__(kThreads)
if3_dequant_kernel(const uint8_t *__restrict__ q, const uint8_t *__restrict__ sf,
                   int scale_layout, const float *__restrict__ s_dec_ptr, I rows, I cols,
                   OutT *__restrict__ y) {
  const float s_dec = *s_dec_ptr;
  const I bpr = cols / 16, nblk = rows * bpr;
  const I stride = static_cast<I>(gridDim.x) * kThreads;
  for (I b = static_cast<I>(blockIdx.x) * kThreads + threadIdx.x; b < nblk; b += stride) {
    const I r = b / bpr, cb = b - r * bpr;
    const uint16_t *src = reinterpret_cast<const uint16_t *>(q + b * 6);
    const uint32_t h0 = __ldg(src), h1 = __ldg(src + 1), h2 = __ldg(src + 2);
    const uint32_t g[2] = {(h0 | h1 << 16) & 0xFFFFFFu, (h1 >> 8) | (h2 << 8)};
    const uint32_t sb = __ldg(sf + scale_offset(r, cb, bpr, scale_layout));
    const float S = e4m3_value(sb & 0x7Fu);
    float out[16];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t c = (g[t] >> (3 * j)) & 7u;
        float qv;
        if (sb & 0x80u) {                               // INT3: k in two's complement
          const int k = static_cast<int>(c) - ((c & 4u) ? 8 : 0);
          qv = __fmul_rn(static_cast<float>(k), kDown);
        } else {                                        // E2M0: 0, 1, 2, 4
          const uint32_t mi = c & 3u;
          const float mag = static_cast<float>(mi + (mi == 3u ? 1u : 0u));
          qv = (c & 4u) ? -mag : mag;
        }
        out[8 * t + j] = __fmul_rn(__fmul_rn(qv, S), s_dec);
      }
    }
    OutT *o = y + b * 16;                               // the output is dense as well
    if (sizeof(OutT) == 2) {
      uint4 *d = reinterpret_cast<uint4 *>(o);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __nv_bfloat162 h2v = __floats2bfloat162_rn(out[8 * i + 2 * k], out[8 * i + 2 * k + 1]);
          memcpy(&w[k], &h2v, sizeof(uint32_t));
        }
        d[i] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      float4 *d = reinterpret_cast<float4 *>(o);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        d[i] = make_float4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
    }
  }
}

int grid_for(int64_t nblk, const Launch &L) {
  const int64_t want = (nblk + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(L.num_sms) * 8;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

// 32-bit indices when every element offset, and every block index a
// grid-stride step can reach, stays below 2^31
bool narrow(int64_t rows, int64_t cols, int64_t ld, int grid) {
  return rows * (ld > cols ? ld : cols) + 16 * static_cast<int64_t>(grid) * kThreads <
         (int64_t{1} << 31);
}

template <typename T>
cudaError_t launch_q(const void *x, int64_t rows, int64_t cols, int64_t ld, const float *amax,
                     float *s_dec_out, uint8_t *q, uint8_t *sf, int scale_layout,
                     const Launch &L) {
  const int grid = grid_for((rows * (cols / 16) + 1) / 2, L);      // one thread per block pair
  const T *p = static_cast<const T *>(x);
  if (narrow(rows, cols, ld, 2 * grid))           // a pair step spans two blocks
    if3_kernel<T, uint32_t><<<grid, kThreads, 0, L.stream>>>(
        p, static_cast<uint32_t>(rows), static_cast<uint32_t>(cols), static_cast<uint32_t>(ld),
        amax, s_dec_out, q, sf, scale_layout);
  else
    if3_kernel<T, int64_t><<<grid, kThreads, 0, L.stream>>>(p, rows, cols, ld, amax, s_dec_out, q,
                                                           sf, scale_layout);
  return cudaGetLastError();
}

template <typename OutT>
cudaError_t launch_dq(const uint8_t *q, const uint8_t *sf, int scale_layout, const float *s_dec,
                      int64_t rows, int64_t cols, void *y, const Launch &L) {
  const int grid = grid_for(rows * (cols / 16), L);
  OutT *o = static_cast<OutT *>(y);
  if (narrow(rows, cols, cols, grid))
    if3_dequant_kernel<OutT, uint32_t><<<grid, kThreads, 0, L.stream>>>(
        q, sf, scale_layout, s_dec, static_cast<uint32_t>(rows), static_cast<uint32_t>(cols), o);
  else
    if3_dequant_kernel<OutT, int64_t><<<grid, kThreads, 0, L.stream>>>(q, sf, scale_layout, s_dec,
                                                                      rows, cols, o);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_if3(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                       const float *amax, float *s_dec_out, uint8_t *q, uint8_t *sf,
                       int scale_layout, const Launch &L) {
  if (dtype == FP4Q_BF16)
    return launch_q<__nv_bfloat16>(x, rows, cols, ld, amax, s_dec_out, q, sf, scale_layout, L);
  return launch_q<float>(x, rows, cols, ld, amax, s_dec_out, q, sf, scale_layout, L);
}

cudaError_t launch_if3_dequant(const uint8_t *q, const uint8_t *sf, int scale_layout,
                               const float *s_dec, int64_t rows, int64_t cols, void *y,
                               int y_dtype, const Launch &L) {
  if (y_dtype == FP4Q_BF16)
    return launch_dq<__nv_bfloat16>(q, sf, scale_layout, s_dec, rows, cols, y, L);
  return launch_dq<float>(q, sf, scale_layout, s_dec, rows, cols, y, L);
}

}  // namespace fp4q
