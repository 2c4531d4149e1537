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
//   * the sign flip rides on the BF16 unpacking (one multiply-add and one
//     LOP3 per packed pair), the butterfly stages h = 1, 2, 4, 8 run in
//     registers on f32x2 column pairs;
//   * for n = 128 the stages h = 16, 32, 64 combine the eight groups of a
//     column quad, which sit in lanes g ^ 1, g ^ 2, g ^ 4: each stage is a
//     warp shuffle of the partner's values and one exact fused multiply-add
//     per pair, so the lane keeps its own tokens in registers throughout;
//   * three CTAs per SM for n = 128, stochastic rounding and the fused
//     backward (the register budget that avoids spills), four for the
//     16-point transform with round to nearest;
//   * the rest runs in two passes over the lane's two column pairs (for
//     n = 16 each pass also transforms its pair, which halves the values live
//     at once): scaling by the transform's factor, block maxima (three-input
//     maximum), block scales, stochastic rounding or RNE, packing and the
//     stores of the pair's two code rows and scales;
//   * stochastic rounding needs one Philox call per token per 8 columns,
//     256 per tile: each lane computes 8 of them and stores their four words
//     in a per-warp table in shared memory, from which both passes read the
//     words of their own columns (for n = 128 the table takes the input
//     stage the tile has finished reading, so the warp's shared memory does
//     not grow).  The ten Philox round keys and the 128 signs come in as
//     kernel parameters, and the counters are 32-bit arithmetic wherever the
//     tensor has fewer than 2^35 elements (the high counter word is then 0).
//     The values are dithered in place (e2m1_sr_dithered2: the rounding by
//     scaling with 2^-126) and then packed by the truncating conversion,
//     which drops the bits below the kept one;
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

// stages h = 1, 2, 4, 8 of one column pair over 16 tokens
__device__ __forceinline__ void stages16(float2 (&v)[16]) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1)
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if ((i & h) == 0) {
        const float2 a = v[i], b = v[i + h];
        v[i] = add2(a, b);
        v[i + h] = sub2(a, b);
      }
}

// The Philox table of a warp tile: the four words of the call for token t
// (0..127) and column octet o (0, 1) at byte (2 t + o) * 16 + (t / 16) * 16;
// the pad puts the eight 16-byte writes of a quarter warp (tokens 16 g + i,
// g = 0..7) on eight distinct bank groups.
constexpr int kPTabBytes = (2 * 127 + 1) * 16 + (127 / 16) * 16 + 16;
static_assert(kPTabBytes <= kUnits * 8, "the table fits in one BF16 input stage");
__host__ __device__ constexpr int ptab_off(int t, int o) { return (2 * t + o) * 16 + (t >> 4) * 16; }


// Coordinates (tile row tt, tile column tc) of a linear tile index over a grid
// of tiles_c tile columns, stepped by a fixed number of tiles without
// dividing; 32-bit.
struct TileCursor32 {
  int tile, tt, tc;
  __device__ __forceinline__ void init(int t, int tiles_c) {
    tile = t;
    tt = t / tiles_c;
    tc = t - tt * tiles_c;
  }
  __device__ __forceinline__ void advance(int step, int dtt, int dtc, int tiles_c) {
    tile += step;
    tt += dtt;
    tc += dtc;
    if (tc >= tiles_c) {
      tc -= tiles_c;
      ++tt;
    }
  }
};

// EVEN: tokens % 128 == 0 and cols % 16 == 0, so every warp tile lies wholly
// inside the matrix and the bound tests of the copies and stores drop out.
template <typename T, int N, bool SR, bool AMAX_ONLY, bool ROW, bool I32, bool EVEN>
__global__ void __launch_bounds__(kThreads, (ROW || SR || N == 128) ? 3 : 4)
rht_kernel(const T *__restrict__ dy, int64_t tokens, int64_t cols, int64_t ld,
           const RhtParams P, const float *__restrict__ amax_ptr, float *__restrict__ s_dec_out,
           unsigned *__restrict__ amax_out, uint8_t *__restrict__ q_t,
           uint8_t *__restrict__ sf_t, int scale_layout, float *__restrict__ rht_out,
           const RowArgs R) {
  constexpr int UB = 4 * sizeof(T);                       // bytes per input chunk
  constexpr int IN_BYTES = 2 * kUnits * UB;               // two stages
  constexpr bool PTAB_IN_STAGE = SR && N == 128 && !ROW;
  constexpr int WARP_BYTES = IN_BYTES + ((SR && !PTAB_IN_STAGE) ? kPTabBytes : 0);
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ float rtab[128];
  __shared__ float rtab_row[ROW ? 128 : 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane & 7, cq = lane >> 3;
  uint8_t *wbase = smem + warp * WARP_BYTES;
  const uint32_t in_s = static_cast<uint32_t>(__cvta_generic_to_shared(wbase));
  uint8_t *const ptab_own = wbase + IN_BYTES;
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

  // tile counts fit in 32 bits (the launcher checks): a tile is 2048 elements
  const int tiles_c = static_cast<int>((cols + 15) / 16);
  const int ntiles = tiles_c * static_cast<int>((tokens + 127) / 128);
  const int nwarps = static_cast<int>(gridDim.x) * kWarps;
  const int dtt = nwarps / tiles_c, dtc = nwarps - dtt * tiles_c;
  TileCursor32 cur, nxt;                                  // this tile, the one being copied
  cur.init(static_cast<int>(blockIdx.x) * kWarps + warp, tiles_c);
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
  auto issue = [&](const TileCursor32 &t, int st) {
    const int64_t tbase = static_cast<int64_t>(t.tt) * 128;
    const int64_t col = static_cast<int64_t>(t.tc) * 16 + pc * (16 / static_cast<int>(sizeof(T)));
    if (!EVEN && col >= cols) return;
    const T *src = dy + (tbase + tok0) * ld + col;
    const uint32_t dst = lane_dst + static_cast<uint32_t>(st * kUnits * UB);
#pragma unroll
    for (int i = 0; i < 4 * PPT; ++i) {
      if (!EVEN && tbase + 16 * ((TPI * i) / 16) >= tokens) break;
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
  const int half = cq & 1;
  for (int st = 0; cur.tile < ntiles; cur.advance(nwarps, dtt, dtc, tiles_c), st ^= 1) {
    __syncwarp();   // every lane is done with stage st ^ 1 (last tile) before it is refilled
    if (nxt.tile < ntiles) issue(nxt, st ^ 1);
    cp_async_commit();
    nxt.advance(nwarps, dtt, dtc, tiles_c);
    cp_async_wait<1>();
    __syncwarp();
    // a column quad is all-in or all-out (cols % 8 == 0); a 16-token group
    // likewise (tokens % 16 == 0); for n = 128 all groups of a tile are in
    const int64_t t0 = static_cast<int64_t>(cur.tt) * 128 + 16 * g;
    const int64_t c0 = static_cast<int64_t>(cur.tc) * 16 + 4 * cq;
    const bool valid = EVEN || (c0 < cols && t0 < tokens);
    const uint8_t *ib = wbase + (st * kUnits + my_unit) * UB;
    // The tile's stochastic-rounding bits: element (t, c) draws from Philox
    // call (t cols + c) / 8, one call per token and column octet, 256 per
    // tile.  This lane computes tokens 16 g + 8 (cq & 1) + i of octet cq / 2
    // and stores the four words of each in the warp's table; the passes read
    // back the words of their own columns.  For n = 128 the table sits in the
    // input stage this tile has finished reading (written after the
    // transform, so that no transformed values are live meanwhile).
    uint8_t *const ptab = PTAB_IN_STAGE ? wbase + st * kUnits * UB : ptab_own;
    auto philox_phase = [&]() {
      const int o = cq >> 1, tb = 16 * g + 8 * half;
      const int64_t orow = (static_cast<int64_t>(cur.tt) * 128 + tb) * cols +
                           static_cast<int64_t>(cur.tc) * 16 + 8 * o;
      const uint32_t rstep = static_cast<uint32_t>(cols / 8);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        U32x4 b;
        if (I32) {
          b = philox_rk(P, static_cast<uint32_t>(orow / 8) + static_cast<uint32_t>(i) * rstep, 0u);
        } else {
          const uint64_t gidx = static_cast<uint64_t>(orow / 8) + static_cast<uint64_t>(i) * rstep;
          b = philox_rk(P, static_cast<uint32_t>(gidx), static_cast<uint32_t>(gidx >> 32));
        }
        *reinterpret_cast<uint4 *>(ptab + ptab_off(tb + i, o)) = make_uint4(b.x, b.y, b.z, b.w);
      }
      __syncwarp();
    };
    if (SR && !PTAB_IN_STAGE) philox_phase();
    // token k's sign as a mask for the BF16 / FP32 sign bits
    auto sign_of = [&](int k) -> uint32_t {
      return static_cast<uint32_t>(static_cast<int32_t>(signs << (31 - k)) >> 31) & 0x80000000u;
    };
    // sign-flipped FP32 values of a raw column pair: for BF16 the low value is
    // w * 2^16 + s (adding the sign bit flips it), the high one
    // (w & 0xFFFF0000) ^ s -- one multiply-add and one LOP3 per pair
    auto unpack_bf16 = [](uint32_t w, uint32_t sg) -> float2 {
      return make_float2(__uint_as_float(w * 65536u + sg), __uint_as_float((w & 0xFFFF0000u) ^ sg));
    };
    auto unpack_f32 = [](uint2 w, uint32_t sg) -> float2 {
      return make_float2(__uint_as_float(w.x ^ sg), __uint_as_float(w.y ^ sg));
    };

    // The lane works on its four columns as two column pairs, one per pass.
    uint32_t raw1[sizeof(T) == 2 ? 16 : 1];   // BF16: the pass-1 pair, still packed
    float2 lo[16], hi[16];   // n = 128: the lane's four columns (unused for n = 16)
    if (N == 128) {
      // ---- the whole 128-point transform on all four columns --------------------
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const uint32_t sg = sign_of(k);
        // (a lane outside the matrix reads stale shared memory: it shares no
        // values with lanes inside, and its results are never stored)
        if (sizeof(T) == 2) {
          const uint2 w = *reinterpret_cast<const uint2 *>(ib + 4 * k * UB);
          lo[k] = unpack_bf16(w.x, sg);
          hi[k] = unpack_bf16(w.y, sg);
        } else {
          const uint4 w = *reinterpret_cast<const uint4 *>(ib + 4 * k * UB);
          lo[k] = unpack_f32(make_uint2(w.x, w.y), sg);
          hi[k] = unpack_f32(make_uint2(w.z, w.w), sg);
        }
      }
      stages16(lo);
      stages16(hi);
    }
    if (N == 128) {
      // ---- stages h = 16, 32, 64 across the eight groups, by warp shuffles -------
      // token 16 g + k meets token 16 (g ^ m) + k, m = 1, 2, 4, which sits in
      // lane ^ m: the lane with bit m of g clear keeps RN(a + b), its partner
      // RN(a - b); both are fma(own, +-1, partner), whose product is exact, so
      // the lane keeps its own 16 tokens and nothing is written back
#pragma unroll
      for (int sgi = 0; sgi < 3; ++sgi) {
        const int m = 1 << sgi;
        const float sgn = (g & m) ? -1.0f : 1.0f;
        const float2 sg2 = make_float2(sgn, sgn);
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
    if (PTAB_IN_STAGE) {   // the stage's raw values are all read
      __syncwarp();
      philox_phase();
    }

    // ---- two passes over the column pairs ---------------------------------------
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const int pp = p;                      // the column pair of this pass
      float2 v[16];
      if (N == 128) {
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = p == 0 ? lo[k] : hi[k];
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint32_t sg = sign_of(k);
          if (sizeof(T) == 2) {
            uint32_t w;
            if (p == 0) {
              const uint2 u = *reinterpret_cast<const uint2 *>(ib + 4 * k * UB);
              w = u.x;
              raw1[k] = u.y;
            } else {
              w = raw1[k];
            }
            v[k] = unpack_bf16(w, sg);
          } else {
            const uint2 u = *reinterpret_cast<const uint2 *>(ib + 4 * k * UB + 8 * pp);
            v[k] = unpack_f32(u, sg);
          }
        }
        stages16(v);
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) v[k] = mul2(v[k], make_float2(cn, cn));

      // ---- block maxima (16 tokens of each column) ------------------------------
      float ma, mb;
      {
        float a[16], b[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) { a[k] = v[k].x; b[k] = v[k].y; }
        ma = absmax_n(a);
        mb = absmax_n(b);
      }
      if (AMAX_ONLY) {
        if (valid) amax_bits = max(amax_bits, __float_as_uint(fmaxf(ma, mb)));
        continue;
      }
      const int64_t c = c0 + 2 * pp;
      if (rht_out && valid) {
#pragma unroll
        for (int k = 0; k < 16; ++k)
          *reinterpret_cast<float2 *>(rht_out + (t0 + k) * cols + c) = v[k];
      }
      const uint32_t sa = nvfp4_scale_code(ma, ts.enc), sb = nvfp4_scale_code(mb, ts.enc);
      const float2 f = make_float2(rtab[sa], rtab[sb]);
#pragma unroll
      for (int k = 0; k < 16; ++k) v[k] = mul2(v[k], f);

      if (SR) {
        // words 0, 1 of a call serve the even quad's pairs, 2, 3 the odd quad's;
        // token 16 g + k of octet o is at ptab_off(16 g, o) + 32 k
        const uint8_t *pw = ptab + ptab_off(16 * g, cq >> 1) + 4 * (2 * (cq & 1) + pp);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint32_t w = *reinterpret_cast<const uint32_t *>(pw + 32 * k);
          v[k] = e2m1_sr_dithered2(v[k], sr_x_lo(w), sr_x_hi(w));
        }
      }
      uint32_t wa[2], wb[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float a[8], b[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) { a[k] = v[8 * h + k].x; b[k] = v[8 * h + k].y; }
        wa[h] = SR ? e2m1x8_rz(a) : e2m1x8(a);
        wb[h] = SR ? e2m1x8_rz(b) : e2m1x8(b);
      }
      if (valid) {
        // columns c, c + 1: code rows tokens/2 bytes apart, scale rows 16 bytes
        // apart in the swizzled layout, tokens/16 in the linear one
        uint8_t *qp = q_t + c * (tokens / 2) + t0 / 2;
        uint8_t *sp = sf_t + scale_offset(c, t0 / 16, tokens / 16, scale_layout);
        const int64_t sstep = scale_layout == FP4Q_SCALE_SWIZZLED_128x4 ? 16 : tokens / 16;
        *reinterpret_cast<uint2 *>(qp) = make_uint2(wa[0], wa[1]);
        *reinterpret_cast<uint2 *>(qp + tokens / 2) = make_uint2(wb[0], wb[1]);
        sp[0] = static_cast<uint8_t>(sa);
        sp[sstep] = static_cast<uint8_t>(sb);
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
      const int64_t tile_t0 = static_cast<int64_t>(cur.tt) * 128;
      const int64_t col0 = static_cast<int64_t>(cur.tc) * 16;
      const bool cvalid = EVEN || col0 < cols;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        const int tok = lane + 32 * j;
        const int64_t t = tile_t0 + tok;
        const bool tv = cvalid && (EVEN || t < tokens);
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
        const float m = absmax_n(x);
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
            const U32x4 b = philox_rk(R, static_cast<uint32_t>(gidx),
                                      I32 ? 0u : static_cast<uint32_t>(gidx >> 32));
            const uint32_t wd[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int k = 0; k < 8; k += 2) {
              const float2 r = e2m1_sr_dithered2(make_float2(x[8 * h + k], x[8 * h + k + 1]),
                                                 sr_x_lo(wd[k >> 1]), sr_x_hi(wd[k >> 1]));
              x[8 * h + k] = r.x;
              x[8 * h + k + 1] = r.y;
            }
          }
        }
        float lo8[8], hi8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) { lo8[k] = x[k]; hi8[k] = x[8 + k]; }
        if (tv) {
          *reinterpret_cast<uint2 *>(R.q + t * (cols / 2) + col0 / 2) =
              SR ? make_uint2(e2m1x8_rz(lo8), e2m1x8_rz(hi8)) : make_uint2(e2m1x8(lo8), e2m1x8(hi8));
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

template <typename T, int N, bool SR, bool AMAX_ONLY, bool ROW, bool I32, bool EVEN>
cudaError_t launch_k2(const T *dy, int64_t tokens, int64_t cols, int64_t ld, uint64_t seed,
                      const float *amax, float *s_dec_out, unsigned *amax_out, uint8_t *q_t,
                      uint8_t *sf_t, int scale_layout, float *rht_out, const Launch &L,
                      const RowArgs &R) {
  constexpr int UB = 4 * sizeof(T);
  constexpr int WARP_BYTES = 2 * kUnits * UB +
                             ((SR && !(N == 128 && !ROW)) ? kPTabBytes : 0);
  constexpr int SMEM = kWarps * WARP_BYTES;
  const void *kern =
      reinterpret_cast<const void *>(rht_kernel<T, N, SR, AMAX_ONLY, ROW, I32, EVEN>);
  static KernelSetup setup;
  int per_sm = 0;
  const cudaError_t e = kernel_setup(setup, kern, kThreads, SMEM, &per_sm);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = ((cols + 15) / 16) * ((tokens + 127) / 128);
  if (ntiles > INT32_MAX / 2) return cudaErrorInvalidValue;   // the kernel counts tiles in 32 bits
  const int64_t cap = static_cast<int64_t>(per_sm) * L.num_sms;
  const int64_t want = (ntiles + kWarps - 1) / kWarps;
  const int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
  rht_kernel<T, N, SR, AMAX_ONLY, ROW, I32, EVEN><<<grid, kThreads, SMEM, L.stream>>>(
      dy, tokens, cols, ld, make_params(seed), amax, s_dec_out, amax_out, q_t, sf_t, scale_layout,
      rht_out, R);
  return cudaGetLastError();
}

// Stochastic rounding draws Philox calls (t * cols + c) / 8: with fewer than
// 2^35 elements every counter fits in 32 bits.
template <typename T, int N, bool SR, bool AMAX_ONLY, bool ROW = false>
cudaError_t launch_k(const T *dy, int64_t tokens, int64_t cols, int64_t ld, uint64_t seed,
                     const float *amax, float *s_dec_out, unsigned *amax_out, uint8_t *q_t,
                     uint8_t *sf_t, int scale_layout, float *rht_out, const Launch &L,
                     const RowArgs &R = RowArgs{}) {
  const bool i32 = SR && tokens * cols < (int64_t{1} << 35);
  // whole warp tiles only; not for the 128-point transform with stochastic
  // rounding, whose even form spills registers and measured no faster
  if constexpr (!(N == 128 && SR)) {
    if (tokens % 128 == 0 && cols % 16 == 0) {
      if (i32)
        return launch_k2<T, N, SR, AMAX_ONLY, ROW, true, true>(
            dy, tokens, cols, ld, seed, amax, s_dec_out, amax_out, q_t, sf_t, scale_layout,
            rht_out, L, R);
      return launch_k2<T, N, SR, AMAX_ONLY, ROW, false, true>(
          dy, tokens, cols, ld, seed, amax, s_dec_out, amax_out, q_t, sf_t, scale_layout,
          rht_out, L, R);
    }
  }
  if (i32)
    return launch_k2<T, N, SR, AMAX_ONLY, ROW, true, false>(
        dy, tokens, cols, ld, seed, amax, s_dec_out, amax_out, q_t, sf_t, scale_layout, rht_out,
        L, R);
  return launch_k2<T, N, SR, AMAX_ONLY, ROW, false, false>(
      dy, tokens, cols, ld, seed, amax, s_dec_out, amax_out, q_t, sf_t, scale_layout, rht_out, L,
      R);
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
