// if4.cu -- IF4 adaptive block-scaled quantization, row-wise 1x16.
//
// "Adaptive Block-Scaled Data Types" (gist.science explainer), section 2
// (IF4): every 16-value block is quantized both as FP4 (E2M1) and as INT4,
// the one with the smaller squared error is kept, and the choice goes into
// the otherwise unused sign bit of the block's E4M3 scale.  The 6/7 method
// maps INT4's range 0..7 onto FP4's 0..6: values are multiplied by 7/6
// before rounding to an integer and by 6/7 when decoded.
//
// A lane quantizes two adjacent blocks at once: every elementwise step is one
// f32x2 instruction whose lanes are (block A element k, block B element k),
// so each lane still sums its own block's squared errors in order k = 0..15,
// as the definition requires.  Products that feed an add or subtract are
// f32x2 fused multiply-adds with a -0 addend known only at run time, which
// keeps them from being contracted into the add (see if4_pair).
//   FP4:  codes by cvt.rn.satfinite.e2m1x2, values back by cvt.f16x2.e2m1x2,
//         errors RN(g - v) by the mixed-precision sub.f32.f16 (g is exact in
//         f16; the sign of the difference does not change its square)
//   INT4: k = rint(t), t = RN(v * RN(7/6)), as RN(t + 1.5 * 2^23) - 1.5 * 2^23
//         (exact round-half-even for |t| < 2^22; the sum's low bits hold k in
//         two's complement); the clamp to [-7, 7] only matters when the
//         block's largest |t| reaches 7.5, which is tested once per block.
//         IF4 packs four nibbles at a time as an exact float sum: the sum of
//         k_i * 16^i (|sum| < 2^15, by f32x2 fused multiply-adds on the
//         integers k_i) plus 8 * 4369 + 2^23 leaves k_i + 8 in nibble i of
//         the low 16 bits; two such halves make a word, and XOR 0x88888888
//         turns every k_i + 8 into k_i mod 16.  NVINT4, which has no k as a
//         float, packs the same way in integers: the sum of
//         bits(t + 1.5 * 2^23) * 16^i minus a constant.
//
// Memory: each warp streams tiles of 32 block pairs through a three-stage
// cp.async buffer in shared memory (each lane copies and later reads only
// its own pair, so no barrier is needed), so two tiles are in flight while
// one computes.  The lane's 16-byte pieces are XOR-swizzled so that both the
// copies and the reads of eight consecutive lanes hit distinct bank groups.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 3;
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
// sum over i < 8 of (bits(1.5 * 2^23) - 8) * 16^i, modulo 2^32
constexpr uint32_t kPackBias = 0x4B3FFFF8u * 0x11111111u;

// FP4 candidate of eight values: the packed codes (v[0] in bits 0..3) and
// the eight rounding differences d[k] = RN(g_k - v_k).
__device__ __forceinline__ uint32_t fp4_codes_diffs(const float (&v)[8], float (&d)[8]) {
  uint32_t w;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t.reg .b32 h0, h1, h2, h3;\n\t"
      ".reg .f16 g0, g1, g2, g3, g4, g5, g6, g7;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %10, %9;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %12, %11;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %14, %13;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %16, %15;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t"
      "cvt.rn.f16x2.e2m1x2 h0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 h1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 h2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 h3, b3;\n\t"
      "mov.b32 {g0, g1}, h0;\n\t"
      "mov.b32 {g2, g3}, h1;\n\t"
      "mov.b32 {g4, g5}, h2;\n\t"
      "mov.b32 {g6, g7}, h3;\n\t"
      "sub.rn.f32.f16 %1, g0, %9;\n\t"
      "sub.rn.f32.f16 %2, g1, %10;\n\t"
      "sub.rn.f32.f16 %3, g2, %11;\n\t"
      "sub.rn.f32.f16 %4, g3, %12;\n\t"
      "sub.rn.f32.f16 %5, g4, %13;\n\t"
      "sub.rn.f32.f16 %6, g5, %14;\n\t"
      "sub.rn.f32.f16 %7, g6, %15;\n\t"
      "sub.rn.f32.f16 %8, g7, %16;\n\t}"
      : "=r"(w), "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3]), "=f"(d[4]), "=f"(d[5]),
        "=f"(d[6]), "=f"(d[7])
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
        "f"(v[7]));
  return w;
}

// Both candidates of blocks A and B (lanes .x / .y of the pairs); picks the
// smaller error per block (MODE 1, IF4) or keeps INT4 (MODE 2, NVINT4, which
// needs neither the FP4 candidate nor the errors).
// nz is -0.0 passed in at run time: fma(a, b, -0) is exactly RN(a * b), signed
// zeros included, and because the compiler cannot see that the addend is
// zero it keeps the product a separate fused multiply-add, which it never
// contracts with the add or subtract that consumes it.  (A plain f32x2
// multiply followed by an f32x2 add has been seen contracted into one fused
// operation despite .rn, which rounds once instead of twice.)
template <bool CLAMP, int MODE>
__device__ __forceinline__ void if4_pair(const float2 (&v)[16], float c76, float c67, float nz,
                                         uint32_t (&wa)[2], uint32_t (&wb)[2], bool &int_a,
                                         bool &int_b) {
  // FP4 candidates and their differences, in element order
  // (each candidate's squared errors are summed as soon as they exist, in
  // element order, so no difference outlives its half-block)
  uint32_t fpa[2] = {0u, 0u}, fpb[2] = {0u, 0u};
  float2 efp = make_float2(0.0f, 0.0f), eint = make_float2(0.0f, 0.0f);
  if (MODE == 1) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float ta[8], tb[8], ea[8], eb[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) { ta[k] = v[8 * h + k].x; tb[k] = v[8 * h + k].y; }
      fpa[h] = fp4_codes_diffs(ta, ea);
      fpb[h] = fp4_codes_diffs(tb, eb);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        efp = fma2(make_float2(ea[k], eb[k]), make_float2(ea[k], eb[k]), efp);
    }
  }
  uint32_t ia[2] = {0u, 0u}, ib[2] = {0u, 0u};
  // IF4: k packed as exact float sums of k_i * 16^i over four elements
  float2 pk[2][2];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int h = k >> 3, i = k & 7;
    const float2 vk = v[k];
    // t = RN(v * RN(7/6)) and h = RN(k * RN(6/7)) are products that feed an
    // add or subtract: each is fma(a, b, -0) with the run-time zero nz
    float2 t2 = fma2(vk, make_float2(c76, c76), make_float2(nz, nz));
    if (CLAMP) {
      t2.x = fminf(fmaxf(t2.x, -7.25f), 7.25f);
      t2.y = fminf(fmaxf(t2.y, -7.25f), 7.25f);
    }
    const float2 tm = add2(t2, make_float2(kMagic, kMagic));
    if (MODE == 1) {
      const float2 kf = sub2(tm, make_float2(kMagic, kMagic));    // rint(t), exact
      const float2 hv = fma2(kf, make_float2(c67, c67), make_float2(nz, nz));
      const float2 dint = sub2(vk, hv);
      eint = fma2(dint, dint, eint);
      const int q = i >> 2, j = i & 3;
      const float w16 = j == 0 ? 1.0f : j == 1 ? 16.0f : j == 2 ? 256.0f : 4096.0f;
      pk[h][q] = j == 0 ? kf : fma2(kf, make_float2(w16, w16), pk[h][q]);
    } else {
      ia[h] += __float_as_uint(tm.x) << (4 * i);
      ib[h] += __float_as_uint(tm.y) << (4 * i);
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (MODE == 1) {
      // sum + 8 * 4369 + 2^23 is exact and leaves k_i + 8 in nibble i of the
      // low 16 bits
      const float2 lo = add2(pk[h][0], make_float2(8423560.0f, 8423560.0f));
      const float2 hi = add2(pk[h][1], make_float2(8423560.0f, 8423560.0f));
      ia[h] = __byte_perm(__float_as_uint(lo.x), __float_as_uint(hi.x), 0x5410) ^ 0x88888888u;
      ib[h] = __byte_perm(__float_as_uint(lo.y), __float_as_uint(hi.y), 0x5410) ^ 0x88888888u;
    } else {
      ia[h] = (ia[h] - kPackBias) ^ 0x88888888u;
      ib[h] = (ib[h] - kPackBias) ^ 0x88888888u;
    }
  }
  int_a = MODE == 2 || eint.x < efp.x;
  int_b = MODE == 2 || eint.y < efp.y;
  wa[0] = int_a ? ia[0] : fpa[0];
  wa[1] = int_a ? ia[1] : fpa[1];
  wb[0] = int_b ? ib[0] : fpb[0];
  wb[1] = int_b ? ib[1] : fpb[1];
}


// Position of a lane's pair: row r and first block cb = 2 * pc, advanced by
// a fixed stride of pairs.  I is int32_t where every element and input offset
// fits (the launcher checks), int64_t otherwise.
template <typename I>
struct Cursor {
  I p, r, pc;
  __device__ __forceinline__ void init(I p0, I ppr) {
    p = p0;
    r = p0 / ppr;
    pc = p0 - r * ppr;
  }
  // FIXED: the stride is a multiple of the pairs per row, so the lane's
  // pair column never changes (dpc == 0) and only the row moves
  template <bool FIXED>
  __device__ __forceinline__ void advance(I stride, I dr, I dpc, I ppr) {
    p += stride;
    r += dr;
    if (!FIXED) {
      pc += dpc;
      if (pc >= ppr) {
        pc -= ppr;
        ++r;
      }
    }
  }
};

// EVEN: cols % 32 == 0 and an even scale address, so every block has a
// partner, code rows are 16-byte aligned and both scale bytes of a pair go
// out as one 2-byte store (the runtime tests of those cases drop out).
template <typename T, bool SWZ, int MODE, typename I, bool FIXED, bool EVEN>
__global__ void __launch_bounds__(kThreads, 5)
if4_kernel(const T *__restrict__ x, int64_t rows_, int64_t cols_, int64_t ld_,
           const float *__restrict__ amax_ptr, float *__restrict__ s_dec_out,
           uint8_t *__restrict__ q, uint8_t *__restrict__ sf, float nz) {
  const I rows = static_cast<I>(rows_), cols = static_cast<I>(cols_), ld = static_cast<I>(ld_);
  const bool sf_even = (reinterpret_cast<uintptr_t>(sf) & 1u) == 0;
  constexpr int LB = 32 * sizeof(T);          // bytes of a lane's pair
  constexpr int PPL = LB / 16;                // 16-byte pieces per lane
  constexpr int PPB = PPL / 2;                // pieces per block
  constexpr int STAGE = 32 * LB;              // bytes of a warp's stage
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ float rtab[128];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // piece i of this lane sits in slot i ^ swz: eight consecutive lanes then
  // cover eight distinct 16-byte bank groups
  const int swz = PPL == 4 ? ((lane >> 1) & 3) : (lane & 7);
  const uint32_t my_s = static_cast<uint32_t>(__cvta_generic_to_shared(smem)) +
                        static_cast<uint32_t>(warp * kStages * STAGE + lane * LB);
  const uint8_t *my_g = smem + warp * kStages * STAGE + lane * LB;

  // work unit: a pair of adjacent blocks (cb, cb + 1) of one row; an odd
  // last block of a row pairs with itself
  const I bpr = cols / 16, ppr = (bpr + 1) / 2, npairs = rows * ppr;
  const I stride = static_cast<I>(gridDim.x) * kThreads;
  const I p0 = static_cast<I>(blockIdx.x) * kThreads + static_cast<I>(threadIdx.x);
  const I dr = stride / ppr, dpc = stride - dr * ppr;

  auto issue = [&](const Cursor<I> &c, int st) {
    if (c.p >= npairs) return;
    const I cb = 2 * c.pc;
    const uint8_t *src = reinterpret_cast<const uint8_t *>(x + c.r * ld + cb * 16);
    const int n = (EVEN || cb + 1 < bpr) ? PPL : PPB;
    const uint32_t dst = my_s + static_cast<uint32_t>(st * STAGE);
#pragma unroll
    for (int i = 0; i < PPL; ++i)
      if (EVEN || i < n) cp_async16(dst + static_cast<uint32_t>((i ^ swz) * 16), src + 16 * i);
  };

  Cursor<I> ci, cc;
  ci.init(p0, ppr);
  cc = ci;
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    issue(ci, s);
    cp_async_commit();
    ci.template advance<FIXED>(stride, dr, dpc, ppr);
  }
  // the tensor scale and the factor table are set up while the first tiles
  // are already in flight
  const TensorScale ts = tensor_scale(*amax_ptr);
  fill_factor_table(rtab, ts.enc);
  if (blockIdx.x == 0 && threadIdx.x == 0 && s_dec_out) *s_dec_out = ts.dec;
  __syncthreads();
  const float c76 = __fdiv_rn(7.0f, 6.0f);   // RN(7/6)
  const float c67 = __fdiv_rn(6.0f, 7.0f);   // RN(6/7)
  for (int st = 0; cc.p < npairs; st = (st + 1 == kStages ? 0 : st + 1)) {
    issue(ci, st == 0 ? kStages - 1 : st - 1);
    cp_async_commit();
    ci.template advance<FIXED>(stride, dr, dpc, ppr);
    cp_async_wait<kStages - 1>();

    const I r = cc.r, cb = 2 * cc.pc;
    const bool has_b = EVEN || cb + 1 < bpr;
    const uint8_t *buf = my_g + st * STAGE;
    float2 v[16];
    float ma, mb;
    if (sizeof(T) == 2) {
      uint4 u[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) u[i] = *reinterpret_cast<const uint4 *>(buf + 16 * (i ^ swz));
      if (!has_b) { u[2] = u[0]; u[3] = u[1]; }   // a single trailing block: its copy is discarded
      ma = bf16x2_hmax(maxabs_bf16x2(maxabs_bf16x2(maxabs_bf16x2(u[0].x, u[0].y), maxabs_bf16x2(u[0].z, u[0].w)),
                                     maxabs_bf16x2(maxabs_bf16x2(u[1].x, u[1].y), maxabs_bf16x2(u[1].z, u[1].w))));
      mb = bf16x2_hmax(maxabs_bf16x2(maxabs_bf16x2(maxabs_bf16x2(u[2].x, u[2].y), maxabs_bf16x2(u[2].z, u[2].w)),
                                     maxabs_bf16x2(maxabs_bf16x2(u[3].x, u[3].y), maxabs_bf16x2(u[3].z, u[3].w))));
      const uint32_t wa[8] = {u[0].x, u[0].y, u[0].z, u[0].w, u[1].x, u[1].y, u[1].z, u[1].w};
      const uint32_t wb[8] = {u[2].x, u[2].y, u[2].z, u[2].w, u[3].x, u[3].y, u[3].z, u[3].w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[2 * i] = make_float2(bf16_lo(wa[i]), bf16_lo(wb[i]));
        v[2 * i + 1] = make_float2(bf16_hi(wa[i]), bf16_hi(wb[i]));
      }
    } else {
      float4 a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = *reinterpret_cast<const float4 *>(buf + 16 * (i ^ swz));
        b[i] = *reinterpret_cast<const float4 *>(buf + 16 * ((i + 4) ^ swz));
      }
      if (!has_b) {
#pragma unroll
        for (int i = 0; i < 4; ++i) b[i] = a[i];
      }
      ma = mb = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[4 * i] = make_float2(a[i].x, b[i].x);
        v[4 * i + 1] = make_float2(a[i].y, b[i].y);
        v[4 * i + 2] = make_float2(a[i].z, b[i].z);
        v[4 * i + 3] = make_float2(a[i].w, b[i].w);
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        ma = fmaxf(ma, fabsf(v[k].x));
        mb = fmaxf(mb, fabsf(v[k].y));
      }
    }
    const uint32_t sab = nvfp4_scale_code2(ma, mb, ts.enc);
    const uint32_t sa = sab & 0xFFu, sb = sab >> 8;
    const float fa = rtab[sa], fb = rtab[sb];
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = mul2(v[k], make_float2(fa, fb));
    // |t| of the block maximum: the clamp can only bind when it reaches 7.5
    const float ta = __fmul_rn(__fmul_rn(ma, fa), c76), tb = __fmul_rn(__fmul_rn(mb, fb), c76);
    uint32_t wa[2], wb[2];
    bool ia, ib;
    if (ta < 7.5f && tb < 7.5f)
      if4_pair<false, MODE>(v, c76, c67, nz, wa, wb, ia, ib);
    else
      if4_pair<true, MODE>(v, c76, c67, nz, wa, wb, ia, ib);
    uint8_t *qp = q + r * (cols / 2) + cb * 8;
    const uint32_t ba = sa | (ia ? 0x80u : 0u), bb = sb | (ib ? 0x80u : 0u);
    if (has_b) {
      if (EVEN || (cols & 31) == 0) {
        *reinterpret_cast<uint4 *>(qp) = make_uint4(wa[0], wa[1], wb[0], wb[1]);
      } else {  // rows of codes are only 8-byte aligned
        *reinterpret_cast<uint2 *>(qp) = make_uint2(wa[0], wa[1]);
        *reinterpret_cast<uint2 *>(qp + 8) = make_uint2(wb[0], wb[1]);
      }
    } else {
      *reinterpret_cast<uint2 *>(qp) = make_uint2(wa[0], wa[1]);
    }
    if (SWZ) {
      // (cb, cb + 1) are adjacent bytes of one 4-column group (cb even, and
      // bpr % 4 == 0 gives every block a partner): one 2-byte store when the
      // scale matrix starts on an even address (the offset o is even)
      const I tile = (r >> 7) * (bpr >> 2) + (cb >> 2);
      const I o = tile * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (cb & 3);
      if (EVEN || sf_even) {
        *reinterpret_cast<uint16_t *>(sf + o) = static_cast<uint16_t>(ba | (bb << 8));
      } else {
        sf[o] = static_cast<uint8_t>(ba);
        sf[o + 1] = static_cast<uint8_t>(bb);
      }
    } else if (EVEN) {   // r * bpr + cb is even
      *reinterpret_cast<uint16_t *>(sf + r * bpr + cb) = static_cast<uint16_t>(ba | (bb << 8));
    } else {
      sf[r * bpr + cb] = static_cast<uint8_t>(ba);
      if (has_b) sf[r * bpr + cb + 1] = static_cast<uint8_t>(bb);
    }
    cc.template advance<FIXED>(stride, dr, dpc, ppr);
  }
  cp_async_wait<0>();
}

template <typename T, bool SWZ, int MODE, typename I>
cudaError_t launch_i(const T *x, int64_t rows, int64_t cols, int64_t ld, const float *amax,
                     float *s_dec_out, uint8_t *q, uint8_t *sf, const Launch &L) {
  constexpr int SMEM = kWarps * kStages * 32 * 32 * static_cast<int>(sizeof(T));
  // the three forms have the same shared memory and nearly the same
  // registers (the fixed and even forms only drop work); the grid is sized
  // by the smallest occupancy of the forms it may launch
  const void *kern = reinterpret_cast<const void *>(if4_kernel<T, SWZ, MODE, I, false, false>);
  const void *kern_f = reinterpret_cast<const void *>(if4_kernel<T, SWZ, MODE, I, true, false>);
  const void *kern_e = reinterpret_cast<const void *>(if4_kernel<T, SWZ, MODE, I, true, true>);
  static KernelSetup setup, setup_f, setup_e;
  int per_sm = 0, per_sm_f = 0, per_sm_e = 0;
  cudaError_t e = kernel_setup(setup, kern, kThreads, SMEM, &per_sm);
  if (e != cudaSuccess) return e;
  e = kernel_setup(setup_f, kern_f, kThreads, SMEM, &per_sm_f);
  if (e != cudaSuccess) return e;
  e = kernel_setup(setup_e, kern_e, kThreads, SMEM, &per_sm_e);
  if (e != cudaSuccess) return e;
  if (per_sm_e < per_sm_f) per_sm_f = per_sm_e;
  const int64_t ppr = (cols / 16 + 1) / 2, npairs = rows * ppr;
  const int64_t want = (npairs + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(per_sm < per_sm_f ? per_sm : per_sm_f) * L.num_sms;
  int64_t grid = want < 1 ? 1 : (want > cap ? cap : want);
  // a full grid a little smaller than the cap whose stride is a multiple of
  // the pairs per row keeps every lane on one pair column
  bool fixed = (grid * kThreads) % ppr == 0;
  for (int64_t g = grid; !fixed && grid == cap && g > cap - cap / 8; --g)
    if ((g * kThreads) % ppr == 0) {
      grid = g;
      fixed = true;
    }
  const bool even = cols % 32 == 0 && (reinterpret_cast<uintptr_t>(sf) & 1u) == 0;
  // -0.0 as a run-time value (see if4_pair)
  if (fixed && even)
    if4_kernel<T, SWZ, MODE, I, true, true><<<static_cast<int>(grid), kThreads, SMEM, L.stream>>>(
        x, rows, cols, ld, amax, s_dec_out, q, sf, -0.0f);
  else if (fixed)
    if4_kernel<T, SWZ, MODE, I, true, false><<<static_cast<int>(grid), kThreads, SMEM, L.stream>>>(
        x, rows, cols, ld, amax, s_dec_out, q, sf, -0.0f);
  else
    if4_kernel<T, SWZ, MODE, I, false, false><<<static_cast<int>(grid), kThreads, SMEM, L.stream>>>(
        x, rows, cols, ld, amax, s_dec_out, q, sf, -0.0f);
  return cudaGetLastError();
}

// 32-bit index arithmetic where every element offset and input offset fits
template <typename T, bool SWZ, int MODE>
cudaError_t launch_t(const T *x, int64_t rows, int64_t cols, int64_t ld, const float *amax,
                     float *s_dec_out, uint8_t *q, uint8_t *sf, const Launch &L) {
  constexpr int64_t kLim = (int64_t{1} << 31) - (int64_t{1} << 24);
  if (rows * ld < kLim && rows * cols < kLim)
    return launch_i<T, SWZ, MODE, int32_t>(x, rows, cols, ld, amax, s_dec_out, q, sf, L);
  return launch_i<T, SWZ, MODE, int64_t>(x, rows, cols, ld, amax, s_dec_out, q, sf, L);
}

template <typename T, int MODE>
cudaError_t launch_layout(const void *x, int64_t rows, int64_t cols, int64_t ld,
                          const float *amax, float *s_dec_out, uint8_t *q, uint8_t *sf,
                          int scale_layout, const Launch &L) {
  const T *p = static_cast<const T *>(x);
  if (scale_layout == FP4Q_SCALE_SWIZZLED_128x4)
    return launch_t<T, true, MODE>(p, rows, cols, ld, amax, s_dec_out, q, sf, L);
  return launch_t<T, false, MODE>(p, rows, cols, ld, amax, s_dec_out, q, sf, L);
}

template <typename T>
cudaError_t launch_mode(const void *x, int64_t rows, int64_t cols, int64_t ld,
                        const float *amax, float *s_dec_out, uint8_t *q, uint8_t *sf,
                        int scale_layout, int int4_mode, const Launch &L) {
  if (int4_mode == 2)
    return launch_layout<T, 2>(x, rows, cols, ld, amax, s_dec_out, q, sf, scale_layout, L);
  return launch_layout<T, 1>(x, rows, cols, ld, amax, s_dec_out, q, sf, scale_layout, L);
}

}  // namespace

cudaError_t launch_if4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                       const float *amax, float *s_dec_out, uint8_t *q, uint8_t *sf,
                       int scale_layout, int int4_mode, const Launch &L) {
  if (dtype == FP4Q_BF16)
    return launch_mode<__nv_bfloat16>(x, rows, cols, ld, amax, s_dec_out, q, sf, scale_layout,
                                      int4_mode, L);
  return launch_mode<float>(x, rows, cols, ld, amax, s_dec_out, q, sf, scale_layout, int4_mode,
                            L);
}

}  // namespace fp4q
