// rht.cu -- random Hadamard transform of a gradient along tokens, fused with
// column-wise NVFP4 1x16 quantization (stochastic rounding or RNE) of the
// transformed values, written as the Wgrad operand dY^T.
//
// Qiita note on NVFP4 training, "ランダムアダマール変換": Wgrad' =
// q(dY H) q(H^T x) with H H^T = I, the random version multiplying H by a
// diagonal of random signs; it helps Wgrad only.  "確率的丸め": stochastic
// rounding helps gradient quantization.
//
// Register tiles: a thread owns 4 columns x 16 consecutive tokens (one
// 16-token group of the transform and one quantization block per column); a
// warp owns 128 tokens x 16 columns (lane = group + 8 * column quad).
//   * sign flip and the butterfly stages h = 1, 2, 4, 8 run in registers on
//     f32x2 pairs of columns;
//   * for n = 128 the stages h = 16, 32, 64 combine the eight groups: the warp
//     swaps values through an 8 KB shared buffer (XOR-swizzled so that both
//     the write and the transposed read hit every bank once per wavefront),
//     runs the three stages, and swaps back;
//   * block maxima are in-thread; stochastic rounding needs one Philox call
//     per token per 8 columns, which two lanes share (each computes half of
//     the tokens and passes the other lane its 64 bits by shuffle);
//   * dY^T codes leave as 8 lanes x 8 bytes = 64 contiguous bytes per column.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 128;       // 4 warps
constexpr int kWarps = kThreads / 32;

template <typename T>
__device__ __forceinline__ void load4(const T *p, float (&v)[4]);
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[4]) {
  const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
}
template <>
__device__ __forceinline__ void load4<float>(const float *p, float (&v)[4]) {
  const float4 u = __ldg(reinterpret_cast<const float4 *>(p));
  v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
}

__device__ __forceinline__ float flip(float x, uint32_t bit) {
  return __uint_as_float(__float_as_uint(x) ^ (bit << 31));
}

// one butterfly stage over 16 tokens of 4 columns held as two column pairs
template <int H>
__device__ __forceinline__ void stage(float2 (&lo)[16], float2 (&hi)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if ((i & H) == 0) {
      const float2 a = lo[i], b = lo[i + H];
      lo[i] = add2(a, b);
      lo[i + H] = sub2(a, b);
      const float2 c = hi[i], d = hi[i + H];
      hi[i] = add2(c, d);
      hi[i + H] = sub2(c, d);
    }
}

// cross-group stage on 8 groups x 2 offsets: values u[g][o]
template <int H>
__device__ __forceinline__ void xstage(float2 (&lo)[16], float2 (&hi)[16]) {
  // index = 2 * group + offset; stage pairs groups g and g + H
#pragma unroll
  for (int g = 0; g < 8; ++g)
    if ((g & H) == 0)
#pragma unroll
      for (int o = 0; o < 2; ++o) {
        const int i = 2 * g + o, j = 2 * (g + H) + o;
        const float2 a = lo[i], b = lo[j];
        lo[i] = add2(a, b);
        lo[j] = sub2(a, b);
        const float2 c = hi[i], d = hi[j];
        hi[i] = add2(c, d);
        hi[j] = sub2(c, d);
      }
}

// 16-byte chunk (token t, column quad q) of a warp's 128 x 16 FP32 buffer,
// XOR-swizzled within each 128-byte line
__device__ __forceinline__ int chunk(int t, int q) {
  const int sw = ((t >> 4) ^ (t >> 1)) & 7;
  return (t * 4 + q) ^ sw;
}

template <typename T, int N, bool SR, bool AMAX_ONLY>
__global__ void __launch_bounds__(kThreads, 3)
rht_kernel(const T *__restrict__ dy, int64_t tokens, int64_t cols, int64_t ld, uint64_t seed,
           const float *__restrict__ amax_ptr, float *__restrict__ s_dec_out,
           unsigned *__restrict__ amax_out, uint8_t *__restrict__ q_t,
           uint8_t *__restrict__ sf_t, int scale_layout, float *__restrict__ rht_out) {
  __shared__ float rtab[128];
  __shared__ __align__(16) float4 xbuf[N == 128 ? kWarps * 128 * 4 : 1];
  TensorScale ts{1.0f, 1.0f};
  if (!AMAX_ONLY) {
    ts = tensor_scale(*amax_ptr);
    fill_factor_table(rtab, ts.enc);
    if (blockIdx.x == 0 && threadIdx.x == 0 && s_dec_out) *s_dec_out = ts.dec;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, g = lane & 7, cq = lane >> 3;
  float4 *buf = xbuf + (N == 128 ? (threadIdx.x >> 5) * 512 : 0);

  // the random diagonal: bit k of Philox(counter (0,0,1,0), key seed)
  const U32x4 sw = philox4x32_10(U32x4{0u, 0u, 1u, 0u}, static_cast<uint32_t>(seed),
                                 static_cast<uint32_t>(seed >> 32));
  uint32_t signs;   // bit k: sign of token 16 g + k of a 128-token group (bit k of a 16-group)
  if (N == 16) {
    signs = sw.x & 0xFFFFu;
  } else {
    const uint32_t word = (g >> 1) == 0 ? sw.x : (g >> 1) == 1 ? sw.y : (g >> 1) == 2 ? sw.z : sw.w;
    signs = (word >> ((g & 1) * 16)) & 0xFFFFu;
  }
  const float cn = N == 16 ? 0.25f : __frsqrt_rn(128.0f);

  const int64_t tiles_c = (cols + 15) / 16;
  const int64_t ntiles = tiles_c * ((tokens + 127) / 128);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  uint32_t amax_bits = 0u;
  for (int64_t tile = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
       tile < ntiles; tile += nwarps) {
    const int64_t tt = tile / tiles_c, tc = tile - tt * tiles_c;
    const int64_t t0 = tt * 128 + 16 * g, c0 = tc * 16 + 4 * cq;
    // a column quad is all-in or all-out (cols % 8 == 0); a 16-token group
    // likewise (tokens % 16 == 0); for n = 128 all groups of a tile are in
    const bool valid = c0 < cols && t0 < tokens;

    // ---- load, sign flip, stages h = 1..8 -----------------------------------
    float2 lo[16], hi[16];     // columns (c0, c0+1) and (c0+2, c0+3) per token
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      if (valid) load4<T>(dy + (t0 + k) * ld + c0, v);
      const uint32_t bit = (signs >> k) & 1u;
      lo[k] = make_float2(flip(v[0], bit), flip(v[1], bit));
      hi[k] = make_float2(flip(v[2], bit), flip(v[3], bit));
    }
    stage<1>(lo, hi);
    stage<2>(lo, hi);
    stage<4>(lo, hi);
    stage<8>(lo, hi);

    if (N == 128) {
      // ---- stages h = 16, 32, 64 across the eight groups ----------------------
#pragma unroll
      for (int k = 0; k < 16; ++k)
        buf[chunk(16 * g + k, cq)] = make_float4(lo[k].x, lo[k].y, hi[k].x, hi[k].y);
      __syncwarp();
      // now this lane takes in-group offsets 2g, 2g+1 of all eight groups
#pragma unroll
      for (int gg = 0; gg < 8; ++gg)
#pragma unroll
        for (int o = 0; o < 2; ++o) {
          const float4 c = buf[chunk(16 * gg + 2 * g + o, cq)];
          lo[2 * gg + o] = make_float2(c.x, c.y);
          hi[2 * gg + o] = make_float2(c.z, c.w);
        }
      xstage<1>(lo, hi);   // h = 16
      xstage<2>(lo, hi);   // h = 32
      xstage<4>(lo, hi);   // h = 64
#pragma unroll
      for (int gg = 0; gg < 8; ++gg)
#pragma unroll
        for (int o = 0; o < 2; ++o) {
          const int i = 2 * gg + o;
          buf[chunk(16 * gg + 2 * g + o, cq)] = make_float4(lo[i].x, lo[i].y, hi[i].x, hi[i].y);
        }
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float4 c = buf[chunk(16 * g + k, cq)];
        lo[k] = make_float2(c.x, c.y);
        hi[k] = make_float2(c.z, c.w);
      }
      __syncwarp();
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      lo[k] = mul2(lo[k], make_float2(cn, cn));
      hi[k] = mul2(hi[k], make_float2(cn, cn));
    }

    // ---- block maxima (16 tokens of each column) ------------------------------
    float m[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      m[0] = fmaxf(m[0], fabsf(lo[k].x));
      m[1] = fmaxf(m[1], fabsf(lo[k].y));
      m[2] = fmaxf(m[2], fabsf(hi[k].x));
      m[3] = fmaxf(m[3], fabsf(hi[k].y));
    }
    if (AMAX_ONLY) {
      if (valid)
        amax_bits = max(amax_bits, __float_as_uint(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]))));
      continue;
    }
    if (rht_out && valid) {
#pragma unroll
      for (int k = 0; k < 16; ++k)
        *reinterpret_cast<float4 *>(rht_out + (t0 + k) * cols + c0) =
            make_float4(lo[k].x, lo[k].y, hi[k].x, hi[k].y);
    }
    uint32_t sbyte[4];
    float f[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      sbyte[j] = nvfp4_scale_code(m[j], ts.enc);
      f[j] = rtab[sbyte[j]];
    }

    // ---- encode -----------------------------------------------------------------
    uint32_t w[4][2];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      lo[k] = mul2(lo[k], make_float2(f[0], f[1]));
      hi[k] = mul2(hi[k], make_float2(f[2], f[3]));
    }
    if (SR) {
      // element (t, c) draws from the Philox call (t * cols + c) / 8, which
      // covers 8 columns = this lane's quad and its neighbour's (lane ^ 8):
      // the even quad computes tokens 0..7, the odd one tokens 8..15, and each
      // sends the other the two words of its half
      const int half = cq & 1;
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j][0] = w[j][1] = 0u;
      uint32_t chain = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int k = i + 8 * half;
        // `chain` is zero, but opaque to the compiler: it makes each Philox call
        // wait for the previous iteration, so only one call's state is live
        uint32_t dep;
        asm volatile("and.b32 %0, %1, 0;" : "=r"(dep) : "r"(chain));
        const uint64_t gidx =
            (static_cast<uint64_t>(t0 + k) * static_cast<uint64_t>(cols) +
             static_cast<uint64_t>(c0 - 4 * half)) / 8 + dep;
        // the key is re-read through an opaque move so that the ten round keys
        // are formed per call instead of being held in twenty registers
        uint32_t key0, key1;
        asm volatile("mov.b32 %0, %1;" : "=r"(key0) : "r"(static_cast<uint32_t>(seed)));
        asm volatile("mov.b32 %0, %1;" : "=r"(key1) : "r"(static_cast<uint32_t>(seed >> 32)));
        const U32x4 b = philox4x32_10(U32x4{static_cast<uint32_t>(gidx),
                                            static_cast<uint32_t>(gidx >> 32), 0u, 0u},
                                      key0, key1);
        // words 0,1 serve the even quad (columns 0-3), words 2,3 the odd quad
        const uint32_t keep0 = half ? b.z : b.x, keep1 = half ? b.w : b.y;
        const uint32_t send0 = half ? b.x : b.z, send1 = half ? b.y : b.w;
        const uint32_t got0 = __shfl_xor_sync(0xFFFFFFFFu, send0, 8);
        const uint32_t got1 = __shfl_xor_sync(0xFFFFFFFFu, send1, 8);
        // this lane computed token i + 8 half, the partner token i + 8 (1 - half):
        // the words of token i and of token i + 8
        const uint32_t ti0 = half ? got0 : keep0, ti1 = half ? got1 : keep1;
        const uint32_t tj0 = half ? keep0 : got0, tj1 = half ? keep1 : got1;
        const float vi[4] = {lo[i].x, lo[i].y, hi[i].x, hi[i].y};
        const float vj[4] = {lo[i + 8].x, lo[i + 8].y, hi[i + 8].x, hi[i + 8].y};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t wi = (j >> 1) ? ti1 : ti0, wj = (j >> 1) ? tj1 : tj0;
          const uint32_t ui = (j & 1) ? (wi >> 16) : (wi & 0xFFFFu);
          const uint32_t uj = (j & 1) ? (wj >> 16) : (wj & 0xFFFFu);
          w[j][0] |= e2m1_sr_bits(vi[j], ui) << (4 * i);
          w[j][1] |= e2m1_sr_bits(vj[j], uj) << (4 * i);
        }
        chain = b.x;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j][0] = w[j][1] = 0u;
#pragma unroll
      for (int k = 0; k < 16; k += 2) {
        const uint32_t sh = 8 * ((k >> 1) & 3);
        w[0][k >> 3] |= e2m1x2(lo[k].x, lo[k + 1].x) << sh;
        w[1][k >> 3] |= e2m1x2(lo[k].y, lo[k + 1].y) << sh;
        w[2][k >> 3] |= e2m1x2(hi[k].x, hi[k + 1].x) << sh;
        w[3][k >> 3] |= e2m1x2(hi[k].y, hi[k + 1].y) << sh;
      }
    }
    if (valid) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        *reinterpret_cast<uint2 *>(q_t + (c0 + j) * (tokens / 2) + t0 / 2) =
            make_uint2(w[j][0], w[j][1]);
        sf_t[scale_offset(c0 + j, t0 / 16, tokens / 16, scale_layout)] =
            static_cast<uint8_t>(sbyte[j]);
      }
    }
  }
  if (AMAX_ONLY) {
    amax_bits = __reduce_max_sync(0xFFFFFFFFu, amax_bits);
    if (lane == 0) atomicMax(amax_out, amax_bits);
  }
}

template <typename T, int N, bool SR, bool AMAX_ONLY>
cudaError_t launch_k(const T *dy, int64_t tokens, int64_t cols, int64_t ld, uint64_t seed,
                     const float *amax, float *s_dec_out, unsigned *amax_out, uint8_t *q_t,
                     uint8_t *sf_t, int scale_layout, float *rht_out, const Launch &L) {
  const void *kern = reinterpret_cast<const void *>(rht_kernel<T, N, SR, AMAX_ONLY>);
  static int per_sm = 0;
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0) != cudaSuccess ||
        per_sm < 1) {
      cudaGetLastError();
      per_sm = 1;
    }
  }
  const int64_t ntiles = ((cols + 15) / 16) * ((tokens + 127) / 128);
  const int64_t cap = static_cast<int64_t>(per_sm) * L.num_sms;
  const int64_t want = (ntiles + kWarps - 1) / kWarps;
  const int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
  rht_kernel<T, N, SR, AMAX_ONLY><<<grid, kThreads, 0, L.stream>>>(
      dy, tokens, cols, ld, seed, amax, s_dec_out, amax_out, q_t, sf_t, scale_layout, rht_out);
  return cudaGetLastError();
}

template <typename T, int N>
cudaError_t launch_n(const T *dy, int64_t tokens, int64_t cols, int64_t ld, int round,
                     uint64_t seed, const float *amax, float *s_dec_out, unsigned *amax_out,
                     uint8_t *q_t, uint8_t *sf_t, int scale_layout, float *rht_out,
                     bool amax_only, const Launch &L) {
  if (amax_only)
    return launch_k<T, N, false, true>(dy, tokens, cols, ld, seed, nullptr, nullptr, amax_out,
                                       nullptr, nullptr, 0, nullptr, L);
  if (round == FP4Q_SR)
    return launch_k<T, N, true, false>(dy, tokens, cols, ld, seed, amax, s_dec_out, nullptr, q_t,
                                       sf_t, scale_layout, rht_out, L);
  return launch_k<T, N, false, false>(dy, tokens, cols, ld, seed, amax, s_dec_out, nullptr, q_t,
                                      sf_t, scale_layout, rht_out, L);
}

template <typename T>
cudaError_t launch_t(const void *dy, int64_t tokens, int64_t cols, int64_t ld, int n, int round,
                     uint64_t seed, const float *amax, float *s_dec_out, unsigned *amax_out,
                     uint8_t *q_t, uint8_t *sf_t, int scale_layout, float *rht_out,
                     bool amax_only, const Launch &L) {
  const T *p = static_cast<const T *>(dy);
  if (n == 16)
    return launch_n<T, 16>(p, tokens, cols, ld, round, seed, amax, s_dec_out, amax_out, q_t, sf_t,
                           scale_layout, rht_out, amax_only, L);
  return launch_n<T, 128>(p, tokens, cols, ld, round, seed, amax, s_dec_out, amax_out, q_t, sf_t,
                          scale_layout, rht_out, amax_only, L);
}

}  // namespace

cudaError_t launch_rht_amax(const void *dy, int dtype, int64_t tokens, int64_t cols,
                            int64_t ld, int n, uint64_t seed, float *amax_out,
                            const Launch &L) {
  cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), L.stream);
  if (e != cudaSuccess) return e;
  unsigned *out = reinterpret_cast<unsigned *>(amax_out);
  if (dtype == FP4Q_BF16)
    return launch_t<__nv_bfloat16>(dy, tokens, cols, ld, n, 0, seed, nullptr, nullptr, out,
                                   nullptr, nullptr, 0, nullptr, true, L);
  return launch_t<float>(dy, tokens, cols, ld, n, 0, seed, nullptr, nullptr, out, nullptr,
                         nullptr, 0, nullptr, true, L);
}

cudaError_t launch_rht_quant(const void *dy, int dtype, int64_t tokens, int64_t cols,
                             int64_t ld, int n, int round, uint64_t seed, const float *amax,
                             float *s_dec_out, uint8_t *q_t, uint8_t *sf_t, int scale_layout,
                             float *rht_out, const Launch &L) {
  if (dtype == FP4Q_BF16)
    return launch_t<__nv_bfloat16>(dy, tokens, cols, ld, n, round, seed, amax, s_dec_out,
                                   nullptr, q_t, sf_t, scale_layout, rht_out, false, L);
  return launch_t<float>(dy, tokens, cols, ld, n, round, seed, amax, s_dec_out, nullptr, q_t,
                         sf_t, scale_layout, rht_out, false, L);
}

}  // namespace fp4q
