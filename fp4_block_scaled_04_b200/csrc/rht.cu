// rht.cu -- random Hadamard transform of a gradient along tokens, fused with
// column-wise NVFP4 1x16 quantization (stochastic rounding or RNE) of the
// transformed values, written as the Wgrad operand dY^T.
//
// Qiita note on NVFP4 training, "ランダムアダマール変換": Wgrad' =
// q(dY H) q(H^T x) with H H^T = I, the random version multiplying H by a
// diagonal of random signs; it helps Wgrad only.  "確率的丸め": stochastic
// rounding helps gradient quantization.
//
// One CTA handles 128 tokens x 64 columns, staged in shared memory as FP32:
//   A   each thread loads 16 tokens of 2 adjacent columns, flips signs and
//       runs the butterfly stages h = 1, 2, 4, 8 in registers;
//   A2  (n = 128) stages h = 16, 32, 64 across the eight 16-token groups;
//   B1  one E4M3 scale per (column, 16-token block);
//   B2  each thread encodes 4 tokens x 8 columns -- the 8 columns of one
//       Philox draw for stochastic rounding;
//   C   codes and scales go out as dY^T rows.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 256;
constexpr int kTT = 128;  // tokens per tile
constexpr int kTC = 64;   // columns per tile
constexpr int kLd = kTC + 4;

template <typename T> struct Pair;
template <> struct Pair<__nv_bfloat16> {
  __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float &a, float &b) {
    uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(p));
    a = bf16_lo(w);
    b = bf16_hi(w);
  }
};
template <> struct Pair<float> {
  __device__ __forceinline__ static void load(const float *p, float &a, float &b) {
    float2 v = __ldg(reinterpret_cast<const float2 *>(p));
    a = v.x;
    b = v.y;
  }
};

__device__ __forceinline__ float flip(float x, uint32_t bit) {
  return __uint_as_float(__float_as_uint(x) ^ (bit << 31));
}

// butterfly stage on 2*len values held as pairs (u[i], u[i+h])
template <int H>
__device__ __forceinline__ void stage16(float (&u)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if ((i & H) == 0) {
      float a = u[i], b = u[i + H];
      u[i] = __fadd_rn(a, b);
      u[i + H] = __fsub_rn(a, b);
    }
}

template <int H>
__device__ __forceinline__ void stage8(float (&u)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if ((i & H) == 0) {
      float a = u[i], b = u[i + H];
      u[i] = __fadd_rn(a, b);
      u[i + H] = __fsub_rn(a, b);
    }
}

struct Smem {
  float t[kTT][kLd];                 // transformed values
  float rf[kTT / 16][kTC];           // r = RN(s_enc / S) per (block, column)
  uint8_t sc[kTC][kTT / 16];         // E4M3 scale code per (column, block)
  __align__(16) uint8_t cs[kTC][kTT / 2 + 16];  // packed codes per column
  float rtab[128];
  uint32_t red[kThreads / 32];
};

template <typename T, int N, bool SR, bool AMAX_ONLY>
__global__ void __launch_bounds__(kThreads)
rht_kernel(const T *__restrict__ dy, int64_t tokens, int64_t cols, int64_t ld, uint64_t seed,
           const float *__restrict__ amax_ptr, float *__restrict__ s_dec_out,
           unsigned *__restrict__ amax_out, uint8_t *__restrict__ q_t,
           uint8_t *__restrict__ sf_t, int scale_layout, float *__restrict__ rht_out) {
  __shared__ __align__(16) Smem s;
  const int t = threadIdx.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kTT;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTC;

  TensorScale ts{1.0f, 1.0f};
  if (!AMAX_ONLY) {
    ts = tensor_scale(*amax_ptr);
    fill_factor_table(s.rtab, ts.enc);
    if (blockIdx.x == 0 && blockIdx.y == 0 && t == 0 && s_dec_out) *s_dec_out = ts.dec;
  }

  // ---- A: sign flip + in-group stages -----------------------------------
  {
    const int p = t & 31, g = t >> 5;
    const int64_t col = c0 + 2 * p, tok0 = t0 + 16 * g;
    const bool active = col < cols && tok0 < tokens;
    // the random diagonal: bit k of Philox(counter (0,0,1,0), key seed)
    const U32x4 sw = philox4x32_10(U32x4{0u, 0u, 1u, 0u}, static_cast<uint32_t>(seed),
                                   static_cast<uint32_t>(seed >> 32));
    uint32_t bits16;
    if (N == 16) {
      bits16 = sw.x & 0xFFFFu;
    } else {
      uint32_t word = (g >> 1) == 0 ? sw.x : (g >> 1) == 1 ? sw.y : (g >> 1) == 2 ? sw.z : sw.w;
      bits16 = (word >> ((g & 1) * 16)) & 0xFFFFu;
    }
    float u0[16], u1[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float a = 0.0f, b = 0.0f;
      if (active) Pair<T>::load(dy + (tok0 + k) * ld + col, a, b);
      uint32_t bit = (bits16 >> k) & 1u;
      u0[k] = flip(a, bit);
      u1[k] = flip(b, bit);
    }
    stage16<1>(u0); stage16<1>(u1);
    stage16<2>(u0); stage16<2>(u1);
    stage16<4>(u0); stage16<4>(u1);
    stage16<8>(u0); stage16<8>(u1);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float a = u0[k], b = u1[k];
      if (N == 16) {
        a = __fmul_rn(a, 0.25f);
        b = __fmul_rn(b, 0.25f);
      }
      *reinterpret_cast<float2 *>(&s.t[16 * g + k][2 * p]) = make_float2(a, b);
    }
  }
  __syncthreads();

  // ---- A2: cross-group stages for n = 128 ---------------------------------
  if (N == 128) {
    const float c128 = __frsqrt_rn(128.0f);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int id = t + kThreads * j;
      const int p = id & 31, o = id >> 5;
      float u0[8], u1[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float2 v = *reinterpret_cast<const float2 *>(&s.t[o + 16 * q][2 * p]);
        u0[q] = v.x;
        u1[q] = v.y;
      }
      stage8<1>(u0); stage8<1>(u1);   // h = 16
      stage8<2>(u0); stage8<2>(u1);   // h = 32
      stage8<4>(u0); stage8<4>(u1);   // h = 64
#pragma unroll
      for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float2 *>(&s.t[o + 16 * q][2 * p]) =
            make_float2(__fmul_rn(u0[q], c128), __fmul_rn(u1[q], c128));
    }
    __syncthreads();
  }

  if (AMAX_ONLY) {
    uint32_t m = 0;
    for (int id = t; id < kTT * kTC; id += kThreads) {
      float v = s.t[id / kTC][id % kTC];
      m = max(m, __float_as_uint(v) & 0x7FFFFFFFu);
    }
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if ((t & 31) == 0) s.red[t >> 5] = m;
    __syncthreads();
    if (t < 32) {
      uint32_t v = t < kThreads / 32 ? s.red[t] : 0u;
      v = __reduce_max_sync(0xFFFFFFFFu, v);
      if (t == 0) atomicMax(amax_out, v);
    }
    return;
  }

  if (rht_out) {
    for (int id = t; id < kTT * (kTC / 4); id += kThreads) {
      const int rr = id / (kTC / 4), cc = (id % (kTC / 4)) * 4;
      if (t0 + rr < tokens && c0 + cc < cols)
        *reinterpret_cast<float4 *>(rht_out + (t0 + rr) * cols + c0 + cc) =
            *reinterpret_cast<const float4 *>(&s.t[rr][cc]);
    }
  }

  // ---- B1: block scales ----------------------------------------------------
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int id = t + kThreads * j;
    const int cc = id & (kTC - 1), b = id >> 6;
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < 16; ++k) m = fmaxf(m, fabsf(s.t[16 * b + k][cc]));
    const uint32_t code = nvfp4_scale_code(m, ts.enc);
    s.sc[cc][b] = static_cast<uint8_t>(code);
    s.rf[b][cc] = s.rtab[code];
  }
  __syncthreads();

  // ---- B2: encode 4 tokens x 8 columns ------------------------------------
  {
    const int o = t & 7, q = t >> 3;
    const int b = q >> 2;
    const int64_t gcol = c0 + 8 * o;
    if (gcol < cols && t0 + 4 * q < tokens) {
      float f[8];
      {
        float4 a = *reinterpret_cast<const float4 *>(&s.rf[b][8 * o]);
        float4 c = *reinterpret_cast<const float4 *>(&s.rf[b][8 * o + 4]);
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = c.x; f[5] = c.y; f[6] = c.z; f[7] = c.w;
      }
      uint32_t packed[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) packed[j] = 0u;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float v[8];
        float4 a = *reinterpret_cast<const float4 *>(&s.t[4 * q + k][8 * o]);
        float4 c = *reinterpret_cast<const float4 *>(&s.t[4 * q + k][8 * o + 4]);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = __fmul_rn(v[j], f[j]);
        if (SR) {
          const uint64_t gt = static_cast<uint64_t>(t0 + 4 * q + k);
          const U32x4 bits = sr_bits_group(seed, (gt * static_cast<uint64_t>(cols) +
                                                  static_cast<uint64_t>(gcol)) / 8);
#pragma unroll
          for (int j = 0; j < 8; ++j) packed[j] |= e2m1_sr(v[j], half16(bits, j)) << (4 * k);
        } else {
#pragma unroll
          for (int j = 0; j < 8; j += 2) {
            uint32_t pr = e2m1x2(v[j], v[j + 1]);   // columns j, j+1 of token k
            packed[j] |= (pr & 0xFu) << (4 * k);
            packed[j + 1] |= ((pr >> 4) & 0xFu) << (4 * k);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint16_t *>(&s.cs[8 * o + j][2 * q]) = static_cast<uint16_t>(packed[j]);
    }
  }
  __syncthreads();

  // ---- C: store dY^T codes and scales ---------------------------------------
  {
    const int cc = t >> 2, ch = t & 3;
    const int64_t col = c0 + cc;
    if (col < cols) {
      uint8_t *dst = q_t + col * (tokens / 2) + t0 / 2 + 16 * ch;
      const int64_t tok = t0 + 32 * ch;
      if (tok + 16 <= tokens)
        *reinterpret_cast<uint2 *>(dst) = *reinterpret_cast<const uint2 *>(&s.cs[cc][16 * ch]);
      if (tok + 32 <= tokens)
        *reinterpret_cast<uint2 *>(dst + 8) =
            *reinterpret_cast<const uint2 *>(&s.cs[cc][16 * ch + 8]);
    }
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int id = t + kThreads * j;
    const int cc = id >> 3, b = id & 7;
    const int64_t col = c0 + cc, blk = t0 / 16 + b;
    if (col < cols && blk * 16 < tokens)
      sf_t[scale_offset(col, blk, tokens / 16, scale_layout)] = s.sc[cc][b];
  }
}

template <typename T, int N>
cudaError_t launch_n(const T *dy, int64_t tokens, int64_t cols, int64_t ld, int round,
                     uint64_t seed, const float *amax, float *s_dec_out, unsigned *amax_out,
                     uint8_t *q_t, uint8_t *sf_t, int scale_layout, float *rht_out,
                     bool amax_only, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>((cols + kTC - 1) / kTC),
            static_cast<unsigned>((tokens + kTT - 1) / kTT));
  if (amax_only)
    rht_kernel<T, N, false, true><<<grid, kThreads, 0, stream>>>(
        dy, tokens, cols, ld, seed, nullptr, nullptr, amax_out, nullptr, nullptr, 0, nullptr);
  else if (round == FP4Q_SR)
    rht_kernel<T, N, true, false><<<grid, kThreads, 0, stream>>>(
        dy, tokens, cols, ld, seed, amax, s_dec_out, nullptr, q_t, sf_t, scale_layout, rht_out);
  else
    rht_kernel<T, N, false, false><<<grid, kThreads, 0, stream>>>(
        dy, tokens, cols, ld, seed, amax, s_dec_out, nullptr, q_t, sf_t, scale_layout, rht_out);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const void *dy, int64_t tokens, int64_t cols, int64_t ld, int n, int round,
                     uint64_t seed, const float *amax, float *s_dec_out, unsigned *amax_out,
                     uint8_t *q_t, uint8_t *sf_t, int scale_layout, float *rht_out,
                     bool amax_only, cudaStream_t stream) {
  const T *p = static_cast<const T *>(dy);
  if (n == 16)
    return launch_n<T, 16>(p, tokens, cols, ld, round, seed, amax, s_dec_out, amax_out, q_t, sf_t,
                           scale_layout, rht_out, amax_only, stream);
  return launch_n<T, 128>(p, tokens, cols, ld, round, seed, amax, s_dec_out, amax_out, q_t, sf_t,
                          scale_layout, rht_out, amax_only, stream);
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
                                   nullptr, nullptr, 0, nullptr, true, L.stream);
  return launch_t<float>(dy, tokens, cols, ld, n, 0, seed, nullptr, nullptr, out, nullptr,
                         nullptr, 0, nullptr, true, L.stream);
}

cudaError_t launch_rht_quant(const void *dy, int dtype, int64_t tokens, int64_t cols,
                             int64_t ld, int n, int round, uint64_t seed, const float *amax,
                             float *s_dec_out, uint8_t *q_t, uint8_t *sf_t, int scale_layout,
                             float *rht_out, const Launch &L) {
  if (dtype == FP4Q_BF16)
    return launch_t<__nv_bfloat16>(dy, tokens, cols, ld, n, round, seed, amax, s_dec_out,
                                   nullptr, q_t, sf_t, scale_layout, rht_out, false, L.stream);
  return launch_t<float>(dy, tokens, cols, ld, n, round, seed, amax, s_dec_out, nullptr, q_t,
                         sf_t, scale_layout, rht_out, false, L.stream);
}

}  // namespace fp4q
