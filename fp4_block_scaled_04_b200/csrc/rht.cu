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
//   * each warp streams its tiles through a two-stage cp.async buffer in
//     shared memory, so the next tile is in flight while this one computes
//     (16-byte copies laid out so each warp write is a contiguous 512 bytes;
//     warp barriers order the copy, the reads and the refill);
//   * the sign flip is one LOP3 per packed word, the butterfly stages
//     h = 1, 2, 4, 8 run in registers on f32x2 column pairs;
//   * for n = 128 the stages h = 16, 32, 64 combine the eight groups of a
//     column quad: butterflies between lanes g and g ^ 1, g ^ 2, g ^ 4 by
//     shuffle, each output fma(own, +-1, partner) (an exact product, so one
//     rounding of the sum or difference).  With stochastic rounding, where
//     registers are short, the warp instead swaps values through an 8 KB
//     shared buffer (XOR-swizzled so the write and the transposed read both
//     spread over all banks), runs the three stages and swaps back;
//   * block maxima are in-thread; stochastic rounding needs one Philox call
//     per token per 8 columns, which two lanes share (each computes half of
//     the tokens and passes the other lane its 64 bits by shuffle).  The ten
//     Philox round keys and the 128 signs come in as kernel parameters.  The
//     values are rounded stochastically in place (e2m1_sr_value) and then
//     packed by the same round-to-nearest conversion as the RNE path;
//   * dY^T codes leave as 8 lanes x 8 bytes = 64 contiguous bytes per column.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 128;       // 4 warps
constexpr int kWarps = kThreads / 32;
// input buffer of one warp tile: 128 tokens x 4 column quads ("units" of 4
// elements); every 16 tokens are padded by 2 units, which makes the lanes'
// 8-byte reads (lane = group + 8 * quad, token 16 group + k) fall on 16
// distinct bank pairs per half-warp
constexpr int kUnits = 128 * 4 + 16;
__device__ __forceinline__ int unit_of(int t, int q) { return 4 * t + 2 * (t >> 4) + q; }

struct RhtParams {
  uint32_t k0[10], k1[10];   // Philox4x32-10 round keys of the seed
  uint32_t signs[4];         // bit k of word k/32: sign of token k of the diagonal
};

// The row-wise (Dgrad) output of the fused backward call: NVFP4 1x16 of dY
// itself, with its own tensor amax and its own stochastic-rounding seed.
struct RowArgs {
  const float *amax;         // tensor amax of dY
  float *s_dec_out;          // <- RN(amax / 2688) (may be NULL)
  uint8_t *q;                // codes [tokens, cols/2]
  uint8_t *sf;               // scales [tokens, cols/16]
  uint32_t k0[10], k1[10];   // Philox4x32-10 round keys of the row seed
};

// Philox4x32-10 of the counter (c0, c1, 0, 0) with the caller's round keys
template <typename K>
__device__ __forceinline__ U32x4 philox_rk(const K &P, uint32_t c0, uint32_t c1) {
  uint32_t c2 = 0u, c3 = 0u;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c0;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c2;
    const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ P.k0[i];
    const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ P.k1[i];
    c1 = static_cast<uint32_t>(p1);
    c3 = static_cast<uint32_t>(p0);
    c0 = n0;
    c2 = n2;
  }
  return U32x4{c0, c1, c2, c3};
}

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

// cross-group stage on (8 groups x 2 offsets) values, index 2 * group + offset
template <int H>
__device__ __forceinline__ void xstage(float2 (&lo)[16], float2 (&hi)[16]) {
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

template <typename T, int N, bool SR, bool AMAX_ONLY, bool ROW>
__global__ void __launch_bounds__(kThreads, (N == 16 && !SR && !ROW) ? 4 : 3)
rht_kernel(const T *__restrict__ dy, int64_t tokens, int64_t cols, int64_t ld,
           const RhtParams P, const float *__restrict__ amax_ptr, float *__restrict__ s_dec_out,
           unsigned *__restrict__ amax_out, uint8_t *__restrict__ q_t,
           uint8_t *__restrict__ sf_t, int scale_layout, float *__restrict__ rht_out,
           const RowArgs R) {
  constexpr int UB = 4 * sizeof(T);                       // bytes per input chunk
  constexpr int IN_BYTES = 2 * kUnits * UB;               // two stages
  // with stochastic rounding the 128-point cross-group stages go through a
  // shared exchange buffer (registers are short); otherwise through shuffles
  constexpr bool XSMEM = N == 128 && SR;
  constexpr int WARP_BYTES = IN_BYTES + (XSMEM ? 128 * 16 * 4 : 0);
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ float rtab[128];
  __shared__ float rtab_row[ROW ? 128 : 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane & 7, cq = lane >> 3;
  uint8_t *wbase = smem + warp * WARP_BYTES;
  const uint32_t in_s = static_cast<uint32_t>(__cvta_generic_to_shared(wbase));
  float4 *xbuf = reinterpret_cast<float4 *>(wbase + IN_BYTES);
  const int my_unit = unit_of(16 * g, cq);                // unit (16 g + k, cq) = my_unit + 4 k

  // signs of this lane's 16 tokens
  uint32_t signs;
  if (N == 16) {
    signs = P.signs[0] & 0xFFFFu;
  } else {
    const uint32_t w = (g >> 1) == 0 ? P.signs[0] : (g >> 1) == 1 ? P.signs[1]
                     : (g >> 1) == 2 ? P.signs[2] : P.signs[3];
    signs = (w >> ((g & 1) * 16)) & 0xFFFFu;
  }
  const float cn = N == 16 ? 0.25f : __frsqrt_rn(128.0f);

  const int64_t tiles_c = (cols + 15) / 16;
  const int64_t ntiles = tiles_c * ((tokens + 127) / 128);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  const int64_t dtt = nwarps / tiles_c, dtc = nwarps - dtt * tiles_c;
  TileCursor cur, nxt;                                    // this tile, the one being copied
  cur.init(static_cast<int64_t>(blockIdx.x) * kWarps + warp, tiles_c);
  nxt = cur;

  // the copy of a tile is spread differently from the reads: lane L moves the
  // 16-byte pieces L + 32 i (token (L + 32 i) / PPT, piece (L + 32 i) % PPT,
  // PPT = 16 columns * sizeof(T) / 16), so a warp writes whole
  // 512-byte stretches of shared memory; a __syncwarp after the wait hands
  // the data to the lanes that read it (PPT = pieces per token row)
  constexpr int PPT = sizeof(T);                          // 16-byte pieces per token row
  constexpr int UPP = 16 / UB;                            // units per piece
  // token (L + 32 i) / PPT = tok0 + TPI i and piece pc = L % PPT; the 16-token
  // group of copy i is TPI i / 16 for every lane, so the token bound (tokens
  // is a multiple of 16) is one test per i, and a piece is all-in or all-out
  // (cols % 8 == 0)
  constexpr int TPI = 32 / PPT;                           // tokens per copy step
  const int tok0 = lane / PPT, pc = lane % PPT;
  const uint32_t lane_dst = in_s + static_cast<uint32_t>(unit_of(tok0, pc * UPP) * UB);
  auto issue = [&](const TileCursor &t, int st) {
    const int64_t tbase = t.tt * 128;
    const int64_t col = t.tc * 16 + pc * (16 / static_cast<int>(sizeof(T)));
    if (col >= cols) return;
    const T *src = dy + (tbase + tok0) * ld + col;
    const uint32_t dst = lane_dst + static_cast<uint32_t>(st * kUnits * UB);
#pragma unroll
    for (int i = 0; i < 4 * PPT; ++i) {
      if (tbase + 16 * ((TPI * i) / 16) >= tokens) break;
      // unit_of(tok0 + TPI i, .) - unit_of(tok0, .) = 4 TPI i + 2 ((TPI i) / 16)
      cp_async16(dst + static_cast<uint32_t>((4 * TPI * i + 2 * ((TPI * i) / 16)) * UB), src);
      src += TPI * ld;
    }
  };

  uint32_t amax_bits = 0u;
  if (nxt.tile < ntiles) issue(nxt, 0);
  cp_async_commit();
  nxt.advance(nwarps, dtt, dtc, tiles_c);
  // the tensor scale and the factor table are set up while the first tile
  // is already in flight
  TensorScale ts{1.0f, 1.0f}, tsr{1.0f, 1.0f};
  if (!AMAX_ONLY) {
    ts = tensor_scale(*amax_ptr);
    fill_factor_table(rtab, ts.enc);
    if (blockIdx.x == 0 && threadIdx.x == 0 && s_dec_out) *s_dec_out = ts.dec;
  }
  if (ROW) {
    tsr = tensor_scale(*R.amax);
    fill_factor_table(rtab_row, tsr.enc);
    if (blockIdx.x == 0 && threadIdx.x == 0 && R.s_dec_out) *R.s_dec_out = tsr.dec;
  }
  __syncthreads();
  for (int st = 0; cur.tile < ntiles; cur.advance(nwarps, dtt, dtc, tiles_c), st ^= 1) {
    __syncwarp();   // every lane is done with stage st ^ 1 (last tile) before it is refilled
    if (nxt.tile < ntiles) issue(nxt, st ^ 1);
    cp_async_commit();
    nxt.advance(nwarps, dtt, dtc, tiles_c);
    cp_async_wait<1>();
    __syncwarp();
    // a column quad is all-in or all-out (cols % 8 == 0); a 16-token group
    // likewise (tokens % 16 == 0); for n = 128 all groups of a tile are in
    const int64_t t0 = cur.tt * 128 + 16 * g, c0 = cur.tc * 16 + 4 * cq;
    const bool valid = c0 < cols && t0 < tokens;

    // ---- sign flip and stages h = 1, 2, 4, 8 ----------------------------------
    float2 lo[16], hi[16];     // columns (c0, c0+1) and (c0+2, c0+3) per token
    const uint8_t *ib = wbase + (st * kUnits + my_unit) * UB;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      // 0 or 0xFFFFFFFF: token k's sign
      const uint32_t m = static_cast<uint32_t>(static_cast<int32_t>(signs << (31 - k)) >> 31);
      if (sizeof(T) == 2) {
        uint2 w = valid ? *reinterpret_cast<const uint2 *>(ib + 4 * k * UB) : make_uint2(0u, 0u);
        w.x ^= m & 0x80008000u;
        w.y ^= m & 0x80008000u;
        lo[k] = make_float2(bf16_lo(w.x), bf16_hi(w.x));
        hi[k] = make_float2(bf16_lo(w.y), bf16_hi(w.y));
      } else {
        uint4 w = valid ? *reinterpret_cast<const uint4 *>(ib + 4 * k * UB)
                        : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t s = m & 0x80000000u;
        lo[k] = make_float2(__uint_as_float(w.x ^ s), __uint_as_float(w.y ^ s));
        hi[k] = make_float2(__uint_as_float(w.z ^ s), __uint_as_float(w.w ^ s));
      }
    }
    stage<1>(lo, hi);
    stage<2>(lo, hi);
    stage<4>(lo, hi);
    stage<8>(lo, hi);

    if (N == 128 && !XSMEM) {
      // ---- stages h = 16, 32, 64 across the eight groups ------------------------
      // token 16 g + k meets token 16 (g ^ m) + k, m = 1, 2, 4: the lane with
      // bit m of g clear keeps RN(a + b), its partner RN(a - b); both are
      // fma(own, +-1, partner), whose product is exact
#pragma unroll
      for (int sgi = 0; sgi < 3; ++sgi) {
        const int m = 1 << sgi;
        const float sg = (g & m) ? -1.0f : 1.0f;
        const float2 sg2 = make_float2(sg, sg);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float2 pl = make_float2(__shfl_xor_sync(0xFFFFFFFFu, lo[k].x, m),
                                        __shfl_xor_sync(0xFFFFFFFFu, lo[k].y, m));
          const float2 ph = make_float2(__shfl_xor_sync(0xFFFFFFFFu, hi[k].x, m),
                                        __shfl_xor_sync(0xFFFFFFFFu, hi[k].y, m));
          lo[k] = fma2(lo[k], sg2, pl);
          hi[k] = fma2(hi[k], sg2, ph);
        }
      }
    }
    if (N == 128 && XSMEM) {
      // ---- stages h = 16, 32, 64 across the eight groups ------------------------
      // the 16-byte chunk of (token t, quad q) is 4t + q with its low three
      // bits XORed with (t/16 ^ t/2) mod 8; s = q ^ g is the lane's part of it
      const int s = cq ^ g;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int ck = (4 * (k & 1)) ^ ((k >> 1) & 7);
        xbuf[64 * g + 8 * (k >> 1) + (s ^ ck)] = make_float4(lo[k].x, lo[k].y, hi[k].x, hi[k].y);
      }
      __syncwarp();
#pragma unroll
      for (int gg = 0; gg < 8; ++gg)
#pragma unroll
        for (int o = 0; o < 2; ++o) {
          const float4 c = xbuf[64 * gg + 8 * g + (s ^ ((4 * o) ^ gg))];
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
          xbuf[64 * gg + 8 * g + (s ^ ((4 * o) ^ gg))] =
              make_float4(lo[i].x, lo[i].y, hi[i].x, hi[i].y);
        }
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int ck = (4 * (k & 1)) ^ ((k >> 1) & 7);
        const float4 c = xbuf[64 * g + 8 * (k >> 1) + (s ^ ck)];
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
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      lo[k] = mul2(lo[k], make_float2(f[0], f[1]));
      hi[k] = mul2(hi[k], make_float2(f[2], f[3]));
    }

    // ---- encode -----------------------------------------------------------------
    uint32_t w[4][2];
    if (SR) {
      // element (t, c) draws from the Philox call (t * cols + c) / 8, covering
      // this lane's quad and its neighbour's (lane ^ 8): the even quad computes
      // tokens 0..7, the odd one 8..15, and each sends the other its half.
      // The values are rounded in place; the RNE packing below encodes them.
      const int half = cq & 1;
      const uint64_t row0 = (static_cast<uint64_t>(t0) * static_cast<uint64_t>(cols) +
                             static_cast<uint64_t>(c0 - 4 * half)) / 8;
      const uint64_t rstep = static_cast<uint64_t>(cols) / 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint64_t gidx = row0 + static_cast<uint64_t>(i + 8 * half) * rstep;
        const U32x4 b = philox_rk(P, static_cast<uint32_t>(gidx), static_cast<uint32_t>(gidx >> 32));
        // words 0,1 serve the even quad (columns 0-3), words 2,3 the odd quad
        const uint32_t keep0 = half ? b.z : b.x, keep1 = half ? b.w : b.y;
        const uint32_t send0 = half ? b.x : b.z, send1 = half ? b.y : b.w;
        const uint32_t got0 = __shfl_xor_sync(0xFFFFFFFFu, send0, 8);
        const uint32_t got1 = __shfl_xor_sync(0xFFFFFFFFu, send1, 8);
        // this lane computed token i + 8 half, the partner token i + 8 (1 - half)
        const uint32_t ti0 = half ? got0 : keep0, ti1 = half ? got1 : keep1;
        const uint32_t tj0 = half ? keep0 : got0, tj1 = half ? keep1 : got1;
        lo[i].x = e2m1_sr_value(lo[i].x, sr_z_lo(ti0));
        lo[i].y = e2m1_sr_value(lo[i].y, sr_z_hi(ti0));
        hi[i].x = e2m1_sr_value(hi[i].x, sr_z_lo(ti1));
        hi[i].y = e2m1_sr_value(hi[i].y, sr_z_hi(ti1));
        lo[i + 8].x = e2m1_sr_value(lo[i + 8].x, sr_z_lo(tj0));
        lo[i + 8].y = e2m1_sr_value(lo[i + 8].y, sr_z_hi(tj0));
        hi[i + 8].x = e2m1_sr_value(hi[i + 8].x, sr_z_lo(tj1));
        hi[i + 8].y = e2m1_sr_value(hi[i + 8].y, sr_z_hi(tj1));
      }
    }
    {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float a[8], b[8], c[8], d[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          a[k] = lo[8 * h + k].x; b[k] = lo[8 * h + k].y;
          c[k] = hi[8 * h + k].x; d[k] = hi[8 * h + k].y;
        }
        w[0][h] = e2m1x8(a);
        w[1][h] = e2m1x8(b);
        w[2][h] = e2m1x8(c);
        w[3][h] = e2m1x8(d);
      }
    }
    if (valid) {
      // columns c0..c0+3 (c0 % 4 == 0): code rows tokens/2 bytes apart, scale
      // rows 16 bytes apart in the swizzled layout, tokens/16 in the linear one
      uint8_t *qp = q_t + c0 * (tokens / 2) + t0 / 2;
      uint8_t *sp = sf_t + scale_offset(c0, t0 / 16, tokens / 16, scale_layout);
      const int64_t sstep = scale_layout == FP4Q_SCALE_SWIZZLED_128x4 ? 16 : tokens / 16;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        *reinterpret_cast<uint2 *>(qp + j * (tokens / 2)) = make_uint2(w[j][0], w[j][1]);
        sp[j * sstep] = static_cast<uint8_t>(sbyte[j]);
      }
    }
    if (ROW) {
      // ---- row-wise NVFP4 of dY itself (the Dgrad operand) ----------------------
      // The stage buffer still holds this tile's raw values (it is refilled
      // only after the next tile), so the row blocks are read from it again
      // with a row-friendly split: lane L takes tokens L, L + 32, L + 64,
      // L + 96, each a whole 16-column block (32 bytes, BF16) held by one
      // lane -- the block maximum needs no shuffles and each code row leaves
      // as one 8-byte store.  With BF16 input, lanes L and L ^ 4 read the two
      // 16-byte halves of their tokens in opposite order, so eight consecutive
      // lanes hit eight distinct bank groups.
      const uint8_t *sb0 = wbase + st * kUnits * UB;
      const int64_t tile_t0 = cur.tt * 128, col0 = cur.tc * 16;
      const bool cvalid = col0 < cols;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        const int tok = lane + 32 * j;
        const int64_t t = tile_t0 + tok;
        const bool tv = cvalid && t < tokens;
        const uint8_t *src = sb0 + unit_of(tok, 0) * UB;    // 16 values, 16 * sizeof(T) bytes
        float x[16];
        if (sizeof(T) == 2) {
          // two 16-byte pieces, read in lane-dependent order and put back by select
          const int sw = (lane >> 2) & 1;
          uint4 w0 = tv ? *reinterpret_cast<const uint4 *>(src + 16 * sw) : make_uint4(0u, 0u, 0u, 0u);
          uint4 w1 = tv ? *reinterpret_cast<const uint4 *>(src + 16 * (sw ^ 1)) : make_uint4(0u, 0u, 0u, 0u);
          const uint4 p0 = sw ? w1 : w0, p1 = sw ? w0 : w1;
          const uint32_t ws[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            x[2 * i] = bf16_lo(ws[i]);
            x[2 * i + 1] = bf16_hi(ws[i]);
          }
        } else {
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const uint4 w = tv ? *reinterpret_cast<const uint4 *>(src + 16 * p) : make_uint4(0u, 0u, 0u, 0u);
            x[4 * p + 0] = __uint_as_float(w.x); x[4 * p + 1] = __uint_as_float(w.y);
            x[4 * p + 2] = __uint_as_float(w.z); x[4 * p + 3] = __uint_as_float(w.w);
          }
        }
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < 16; ++k) m = fmaxf(m, fabsf(x[k]));
        const uint32_t sbr = nvfp4_scale_code(m, tsr.enc);
        const float f = rtab_row[sbr];
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          const float2 v = mul2(make_float2(x[k], x[k + 1]), make_float2(f, f));
          x[k] = v.x;
          x[k + 1] = v.y;
        }
        if (SR) {
          // element (t, c) draws 16 bits from Philox call (t * cols + c) / 8
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint64_t gidx = (static_cast<uint64_t>(t) * static_cast<uint64_t>(cols) +
                                   static_cast<uint64_t>(col0 + 8 * h)) / 8;
            const U32x4 b = philox_rk(R, static_cast<uint32_t>(gidx), static_cast<uint32_t>(gidx >> 32));
            const uint32_t wd[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int k = 0; k < 8; ++k)
              x[8 * h + k] = e2m1_sr_value(x[8 * h + k], (k & 1) ? sr_z_hi(wd[k >> 1]) : sr_z_lo(wd[k >> 1]));
          }
        }
        float lo8[8], hi8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) { lo8[k] = x[k]; hi8[k] = x[8 + k]; }
        if (tv) {
          *reinterpret_cast<uint2 *>(R.q + t * (cols / 2) + col0 / 2) = make_uint2(e2m1x8(lo8), e2m1x8(hi8));
          R.sf[scale_offset(t, cur.tc, cols / 16, scale_layout)] = static_cast<uint8_t>(sbr);
        }
      }
    }
  }
  cp_async_wait<0>();
  if (AMAX_ONLY) {
    amax_bits = __reduce_max_sync(0xFFFFFFFFu, amax_bits);
    if (lane == 0) atomicMax(amax_out, amax_bits);
  }
}

// host side: Philox4x32-10 (Salmon et al., SC'11) for the signs, and the
// round keys the kernel consumes
void host_philox(uint32_t c[4], uint32_t k0, uint32_t k1) {
  for (int i = 0; i < 10; ++i) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c[0];
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c[2];
    const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c[1] ^ k0;
    const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c[3] ^ k1;
    c[1] = static_cast<uint32_t>(p1);
    c[3] = static_cast<uint32_t>(p0);
    c[0] = n0;
    c[2] = n2;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
}

RhtParams make_params(uint64_t seed) {
  RhtParams P;
  uint32_t a = static_cast<uint32_t>(seed), b = static_cast<uint32_t>(seed >> 32);
  for (int i = 0; i < 10; ++i) {
    P.k0[i] = a;
    P.k1[i] = b;
    a += 0x9E3779B9u;
    b += 0xBB67AE85u;
  }
  uint32_t c[4] = {0u, 0u, 1u, 0u};
  host_philox(c, static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
  for (int i = 0; i < 4; ++i) P.signs[i] = c[i];
  return P;
}

RowArgs make_row_args(const float *amax, float *s_dec_out, uint8_t *q, uint8_t *sf,
                      uint64_t seed) {
  RowArgs R;
  R.amax = amax;
  R.s_dec_out = s_dec_out;
  R.q = q;
  R.sf = sf;
  uint32_t a = static_cast<uint32_t>(seed), b = static_cast<uint32_t>(seed >> 32);
  for (int i = 0; i < 10; ++i) {
    R.k0[i] = a;
    R.k1[i] = b;
    a += 0x9E3779B9u;
    b += 0xBB67AE85u;
  }
  return R;
}

template <typename T, int N, bool SR, bool AMAX_ONLY, bool ROW = false>
cudaError_t launch_k(const T *dy, int64_t tokens, int64_t cols, int64_t ld, uint64_t seed,
                     const float *amax, float *s_dec_out, unsigned *amax_out, uint8_t *q_t,
                     uint8_t *sf_t, int scale_layout, float *rht_out, const Launch &L,
                     const RowArgs &R = RowArgs{}) {
  constexpr int UB = 4 * sizeof(T);
  constexpr int WARP_BYTES = 2 * kUnits * UB + ((N == 128 && SR) ? 128 * 16 * 4 : 0);
  constexpr int SMEM = kWarps * WARP_BYTES;
  const void *kern = reinterpret_cast<const void *>(rht_kernel<T, N, SR, AMAX_ONLY, ROW>);
  static KernelSetup setup;
  int per_sm = 0;
  const cudaError_t e = kernel_setup(setup, kern, kThreads, SMEM, &per_sm);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = ((cols + 15) / 16) * ((tokens + 127) / 128);
  const int64_t cap = static_cast<int64_t>(per_sm) * L.num_sms;
  const int64_t want = (ntiles + kWarps - 1) / kWarps;
  const int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
  rht_kernel<T, N, SR, AMAX_ONLY, ROW><<<grid, kThreads, SMEM, L.stream>>>(
      dy, tokens, cols, ld, make_params(seed), amax, s_dec_out, amax_out, q_t, sf_t, scale_layout,
      rht_out, R);
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

template <typename T, int N>
cudaError_t launch_bwd_n(const T *dy, int64_t tokens, int64_t cols, int64_t ld, int round,
                         uint64_t seed_col, const float *amax_rht, float *s_dec_col,
                         uint8_t *q_t, uint8_t *sf_t, int scale_layout, const RowArgs &R,
                         const Launch &L) {
  if (round == FP4Q_SR)
    return launch_k<T, N, true, false, true>(dy, tokens, cols, ld, seed_col, amax_rht, s_dec_col,
                                             nullptr, q_t, sf_t, scale_layout, nullptr, L, R);
  return launch_k<T, N, false, false, true>(dy, tokens, cols, ld, seed_col, amax_rht, s_dec_col,
                                            nullptr, q_t, sf_t, scale_layout, nullptr, L, R);
}

template <typename T>
cudaError_t launch_bwd_t(const void *dy, int64_t tokens, int64_t cols, int64_t ld, int n,
                         int round, uint64_t seed_col, const float *amax_rht, float *s_dec_col,
                         uint8_t *q_t, uint8_t *sf_t, int scale_layout, const RowArgs &R,
                         const Launch &L) {
  const T *p = static_cast<const T *>(dy);
  if (n == 16)
    return launch_bwd_n<T, 16>(p, tokens, cols, ld, round, seed_col, amax_rht, s_dec_col, q_t,
                               sf_t, scale_layout, R, L);
  return launch_bwd_n<T, 128>(p, tokens, cols, ld, round, seed_col, amax_rht, s_dec_col, q_t,
                              sf_t, scale_layout, R, L);
}

}  // namespace

cudaError_t launch_rht_backward(const void *dy, int dtype, int64_t tokens, int64_t cols,
                                int64_t ld, int n, int round, uint64_t seed_row,
                                uint64_t seed_col, const float *amax_row, const float *amax_rht,
                                float *s_dec_row, float *s_dec_col, uint8_t *q_row,
                                uint8_t *sf_row, uint8_t *q_t, uint8_t *sf_t, int scale_layout,
                                const Launch &L) {
  const RowArgs R = make_row_args(amax_row, s_dec_row, q_row, sf_row, seed_row);
  if (dtype == FP4Q_BF16)
    return launch_bwd_t<__nv_bfloat16>(dy, tokens, cols, ld, n, round, seed_col, amax_rht,
                                       s_dec_col, q_t, sf_t, scale_layout, R, L);
  return launch_bwd_t<float>(dy, tokens, cols, ld, n, round, seed_col, amax_rht, s_dec_col, q_t,
                             sf_t, scale_layout, R, L);
}

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
