// nvfp4.cu -- NVFP4 1x16 and MXFP4 1x32 quantization, row-wise and/or
// column-wise (the transposed copy the backward pass needs) from one read.
//
// Qiita note on NVFP4 training: "Blockwise" (16 values share one 8-bit
// scale), "誤差逆伝播と転置" (Wgrad / Dgrad consume transposed operands),
// "scaleの導出" (global scale 6*448/amax, local scale = block max / 6 in
// E4M3).  Ultralytics glossary "FP4", "FP4の仕組み" (MXFP4: 32 values per
// power-of-two E8M0 scale).
//
// rowwise_kernel  one thread per block of 16 (NVFP4) or 32 (MXFP4) values of
//                 a row, two blocks per iteration; 128-bit loads.
// rowcol_kernel   register tiles fed by a two-stage cp.async buffer.  A
//                 warp owns 64 rows x 128 bytes (8 16-byte chunks of 8 BF16
//                 or 4 FP32 columns) and copies the next such tile into
//                 shared memory while it computes this one; each warp copy
//                 instruction moves four whole 128-byte row segments.  A
//                 thread works on 16 rows x one chunk (lane = chunk + 8 * row
//                 band).  Pass 1 takes row and column block maxima on the
//                 packed data (row blocks span 2..8 lanes: shuffle), pass 2
//                 reads the rows again and scales and encodes every element
//                 twice.  Row codes of a warp instruction are 8 lanes x 4
//                 bytes of one row, column codes 4 lanes x 8 bytes of one
//                 column: whole 32-byte sectors.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

// ----------------------------------------------------------------------------
// row-wise only
// ----------------------------------------------------------------------------
constexpr int kRowThreads = 256;

template <typename T, int BLK>
__device__ __forceinline__ void load_block(const T *p, uint4 (&u)[BLK * sizeof(T) / 16]) {
#pragma unroll
  for (int i = 0; i < BLK * static_cast<int>(sizeof(T)) / 16; ++i)
    u[i] = __ldg(reinterpret_cast<const uint4 *>(p) + i);
}

template <typename T, int BLK>
__device__ __forceinline__ void unpack_block(const uint4 (&u)[BLK * sizeof(T) / 16],
                                             float (&v)[BLK]) {
  if (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < BLK / 8; ++i) {
      v[8 * i + 0] = bf16_lo(u[i].x); v[8 * i + 1] = bf16_hi(u[i].x);
      v[8 * i + 2] = bf16_lo(u[i].y); v[8 * i + 3] = bf16_hi(u[i].y);
      v[8 * i + 4] = bf16_lo(u[i].z); v[8 * i + 5] = bf16_hi(u[i].z);
      v[8 * i + 6] = bf16_lo(u[i].w); v[8 * i + 7] = bf16_hi(u[i].w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < BLK / 4; ++i) {
      v[4 * i + 0] = __uint_as_float(u[i].x); v[4 * i + 1] = __uint_as_float(u[i].y);
      v[4 * i + 2] = __uint_as_float(u[i].z); v[4 * i + 3] = __uint_as_float(u[i].w);
    }
  }
}

template <typename T, int BLK>
__device__ __forceinline__ float block_absmax(const uint4 (&u)[BLK * sizeof(T) / 16]) {
  constexpr int N = BLK * sizeof(T) / 16;
  if (sizeof(T) == 2) {
    uint32_t m = maxabs_bf16x2(u[0].x, u[0].y);
    m = maxabs_bf16x2(m, maxabs_bf16x2(u[0].z, u[0].w));
#pragma unroll
    for (int i = 1; i < N; ++i)
      m = maxabs_bf16x2(m, maxabs_bf16x2(maxabs_bf16x2(u[i].x, u[i].y),
                                         maxabs_bf16x2(u[i].z, u[i].w)));
    return bf16x2_hmax(m);
  } else {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < N; ++i) {
      m = fmaxf(m, fmaxf(fabsf(__uint_as_float(u[i].x)), fabsf(__uint_as_float(u[i].y))));
      m = fmaxf(m, fmaxf(fabsf(__uint_as_float(u[i].z)), fabsf(__uint_as_float(u[i].w))));
    }
    return m;
  }
}

// 16 values scaled by f, stochastic rounding with the bits of one Philox call
// per 8 values: calls g0 and g0 + 1 (the high counter word g_hi)
__device__ __forceinline__ void encode_sr16(const float (&v)[16], float f, const PhiloxKey &K,
                                            uint32_t g0, uint32_t g_hi, uint32_t (&w)[2]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const U32x4 bits = philox(K, g0 + h, g_hi, 0u, 0u);
    const uint32_t words[4] = {bits.x, bits.y, bits.z, bits.w};
    float t[8];
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const float2 r = e2m1_sr_dithered2(
          mul2(make_float2(v[8 * h + k], v[8 * h + k + 1]), make_float2(f, f)),
          sr_x_lo(words[k >> 1]), sr_x_hi(words[k >> 1]));
      t[k] = r.x;
      t[k + 1] = r.y;
    }
    w[h] = e2m1x8_rz(t);
  }
}

template <int BLK>
__device__ __forceinline__ void encode_rne(const float (&v)[BLK], float f,
                                           uint32_t (&w)[BLK / 8]) {
#pragma unroll
  for (int i = 0; i < BLK / 8; ++i) {
    float t[8];
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const float2 p = mul2(make_float2(v[8 * i + k], v[8 * i + k + 1]), make_float2(f, f));
      t[k] = p.x;
      t[k + 1] = p.y;
    }
    w[i] = e2m1x8(t);
  }
}

template <typename T, bool MX, bool SR, int QMAX, bool I32>
__global__ void __launch_bounds__(kRowThreads)
rowwise_kernel(const T *__restrict__ x, int64_t rows_, int64_t cols_, int64_t ld_,
               const float *__restrict__ amax_ptr, int e8m0_mode, uint64_t seed,
               float *__restrict__ s_dec_out, uint8_t *__restrict__ q,
               uint8_t *__restrict__ sf, int scale_layout) {
  constexpr int BLK = MX ? 32 : 16;
  constexpr int NV = BLK * sizeof(T) / 16;   // uint4 per block
  // 32-bit indices where the launcher has checked that they fit
  using I = typename std::conditional<I32, int32_t, int64_t>::type;
  const I rows = static_cast<I>(rows_), cols = static_cast<I>(cols_), ld = static_cast<I>(ld_);
  __shared__ float rtab[128];
  TensorScale ts{1.0f, 1.0f};
  if (!MX) {
    ts = tensor_scale_q<QMAX>(*amax_ptr);
    fill_factor_table(rtab, ts.enc);
    if (blockIdx.x == 0 && threadIdx.x == 0 && s_dec_out) *s_dec_out = ts.dec;
    __syncthreads();
  }
  const PhiloxKey K(seed);
  const I bpr = cols / BLK, nblk = rows * bpr;
  const I stride = static_cast<I>(gridDim.x) * kRowThreads;
  I b = static_cast<I>(blockIdx.x) * kRowThreads + threadIdx.x;
  // two independent blocks per iteration keep 2 x BLK x sizeof(T) bytes in flight
  for (; b < nblk; b += 2 * stride) {
    const I b1 = b + stride;
    const bool two = b1 < nblk;
    uint4 u0[NV], u1[NV];
    const I r0 = b / bpr, cb0 = b - r0 * bpr;
    const I r1 = two ? b1 / bpr : r0, cb1 = two ? b1 - r1 * bpr : cb0;
    load_block<T, BLK>(x + r0 * ld + cb0 * BLK, u0);
    load_block<T, BLK>(x + r1 * ld + cb1 * BLK, u1);
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (s == 1 && !two) break;
      const uint4(&u)[NV] = s == 0 ? u0 : u1;
      const I r = s == 0 ? r0 : r1, cb = s == 0 ? cb0 : cb1;
      const float m = block_absmax<T, BLK>(u);
      uint32_t sbyte;
      float f;
      if (MX) {
        sbyte = e8m0_biased(m, e8m0_mode);
        f = e8m0_inverse(sbyte);
      } else {
        sbyte = scale_code_q<QMAX>(m, ts.enc);
        f = rtab[sbyte];
      }
      float v[BLK];
      unpack_block<T, BLK>(u, v);
      uint8_t *qp = q + r * (cols / 2) + cb * (BLK / 2);
      if (BLK == 16) {
        uint32_t w[2];
        if (SR) {
          // Philox call (r cols + c) / 8; with fewer than 2^35 elements the
          // counter's high word is 0
          const uint64_t g0 = static_cast<uint64_t>(r * cols + cb * 16) / 8;
          encode_sr16(*reinterpret_cast<const float(*)[16]>(v), f, K, static_cast<uint32_t>(g0),
                      I32 ? 0u : static_cast<uint32_t>(g0 >> 32), w);
        }
        else encode_rne<16>(*reinterpret_cast<const float(*)[16]>(v), f,
                            *reinterpret_cast<uint32_t(*)[2]>(w));
        *reinterpret_cast<uint2 *>(qp) = make_uint2(w[0], w[1]);
      } else {
        uint32_t w[4];
        encode_rne<32>(*reinterpret_cast<const float(*)[32]>(v), f,
                       *reinterpret_cast<uint32_t(*)[4]>(w));
        *reinterpret_cast<uint4 *>(qp) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      sf[scale_offset_t<I>(r, cb, bpr, scale_layout)] = static_cast<uint8_t>(sbyte);
    }
  }
}

// ----------------------------------------------------------------------------
// row-wise and column-wise from one read, register tiles
// ----------------------------------------------------------------------------
constexpr int kRCThreads = 128;

template <typename T, bool MX>
struct RCGeom {
  static constexpr int CPT = 16 / sizeof(T);   // columns per thread: 8 (BF16) or 4 (FP32)
  static constexpr int BLK = MX ? 32 : 16;
  static constexpr int WR = 64;                // warp tile rows (4 bands of 16)
  static constexpr int WC = 8 * CPT;           // warp tile columns
  static constexpr int GR = BLK / CPT;         // lanes per row block
};

template <typename T>
__device__ __forceinline__ void unpack_chunk(uint4 u, float (&v)[16 / sizeof(T)]) {
  if (sizeof(T) == 2) {
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4 % (16 / sizeof(T))] = bf16_lo(u.z); v[5 % (16 / sizeof(T))] = bf16_hi(u.z);
    v[6 % (16 / sizeof(T))] = bf16_lo(u.w); v[7 % (16 / sizeof(T))] = bf16_hi(u.w);
  } else {
    v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
  }
}

// |x| maxima of the chunk: per column lane pair for BF16 (as a packed word
// per column pair), per column for FP32
template <typename T>
__device__ __forceinline__ void chunk_colmax(uint4 u, uint32_t (&cm)[4]) {
  if (sizeof(T) == 2) {
    cm[0] = maxabs_bf16x2(cm[0], u.x); cm[1] = maxabs_bf16x2(cm[1], u.y);
    cm[2] = maxabs_bf16x2(cm[2], u.z); cm[3] = maxabs_bf16x2(cm[3], u.w);
  } else {
    cm[0] = __float_as_uint(fmaxf(__uint_as_float(cm[0]), fabsf(__uint_as_float(u.x))));
    cm[1] = __float_as_uint(fmaxf(__uint_as_float(cm[1]), fabsf(__uint_as_float(u.y))));
    cm[2] = __float_as_uint(fmaxf(__uint_as_float(cm[2]), fabsf(__uint_as_float(u.z))));
    cm[3] = __float_as_uint(fmaxf(__uint_as_float(cm[3]), fabsf(__uint_as_float(u.w))));
  }
}

template <typename T>
__device__ __forceinline__ float chunk_rowmax(uint4 u) {
  if (sizeof(T) == 2) return absmax8(u);
  return fmaxf(fmaxf(fabsf(__uint_as_float(u.x)), fabsf(__uint_as_float(u.y))),
               fmaxf(fabsf(__uint_as_float(u.z)), fabsf(__uint_as_float(u.w))));
}

// packed |x| maxima of rows k and k+1 of a BF16 chunk pair -> (M_k, M_k+1)
__device__ __forceinline__ uint32_t rowpair_max_bf16(uint4 a, uint4 b) {
  const uint32_t ma = maxabs_bf16x2(maxabs_bf16x2(a.x, a.y), maxabs_bf16x2(a.z, a.w));
  const uint32_t mb = maxabs_bf16x2(maxabs_bf16x2(b.x, b.y), maxabs_bf16x2(b.z, b.w));
  // (lo_a, lo_b) and (hi_a, hi_b)
  return maxabs_bf16x2(__byte_perm(ma, mb, 0x5410), __byte_perm(ma, mb, 0x7632));
}

template <typename T, bool MX, int QMAX>
__device__ __forceinline__ uint32_t block_scale(float m, const TensorScale &ts, const float *rtab,
                                                int mode, float &f) {
  if (MX) {
    const uint32_t be = e8m0_biased(m, mode);
    f = e8m0_inverse(be);
    return be;
  }
  const uint32_t code = scale_code_q<QMAX>(m, ts.enc);
  f = rtab[code];
  return code;
}


constexpr int kRCTileBytes = 64 * 128;            // one warp tile: 64 rows x 128 bytes
constexpr int kRCSmem = (kRCThreads / 32) * 2 * kRCTileBytes;

// EVEN: rows % 64 == 0 and cols % WC == 0, so every warp tile lies wholly
// inside the matrix and the bound tests of the copies and stores drop out.
template <typename T, bool MX, bool SR, int QMAX, bool I32, bool EVEN>
__global__ void __launch_bounds__(kRCThreads, SR ? 2 : 3)
rowcol_kernel(const T *__restrict__ x, int64_t rows_, int64_t cols_, int64_t ld_, unsigned layouts,
              const float *__restrict__ amax_ptr, int e8m0_mode, uint64_t seed,
              float *__restrict__ s_dec_out, uint8_t *__restrict__ q_row,
              uint8_t *__restrict__ sf_row, uint8_t *__restrict__ q_col,
              uint8_t *__restrict__ sf_col, int scale_layout) {
  using G = RCGeom<T, MX>;
  constexpr int CPT = G::CPT, BLK = G::BLK, GR = G::GR;
  // 32-bit indices where the launcher has checked that they fit
  using I = typename std::conditional<I32, int32_t, int64_t>::type;
  const I rows = static_cast<I>(rows_), cols = static_cast<I>(cols_), ld = static_cast<I>(ld_);
  __shared__ float rtab[128];
  const PhiloxKey K(seed);
  const bool do_row = (layouts & FP4Q_ROWWISE) != 0;
  const bool do_col = (layouts & FP4Q_COLWISE) != 0;
  const int lane = threadIdx.x & 31, cc = lane & 7, band = lane >> 3;
  const I tiles_c = (cols + G::WC - 1) / G::WC;
  const I ntiles = tiles_c * ((rows + G::WR - 1) / G::WR);
  const I nwarps = static_cast<I>(gridDim.x) * (kRCThreads / 32);
  const bool swz = scale_layout == FP4Q_SCALE_SWIZZLED_128x4;
  extern __shared__ __align__(16) uint8_t rc_smem[];
  const int warp = threadIdx.x >> 5;
  const uint32_t stage_s = static_cast<uint32_t>(__cvta_generic_to_shared(rc_smem)) +
                           static_cast<uint32_t>(warp * 2 * kRCTileBytes);
  const uint4 *stage_g = reinterpret_cast<const uint4 *>(rc_smem + warp * 2 * kRCTileBytes);
  // lane L copies the 16-byte pieces L + 32 i: row (L + 32 i) / 8, chunk L % 8
  // row (L >> 3) + 4 i lies in the 16-row band i / 4 for every lane, and rows
  // is a multiple of 16, so the row bound is one test per band
  auto issue = [&](const TileCursorT<I> &t, int st) {
    const I col = t.tc * G::WC + cc * CPT;
    if (!EVEN && col >= cols) return;
    const I row0 = t.tt * G::WR;
    const T *src = x + (row0 + (lane >> 3)) * ld + col;
    const uint32_t dst =
        stage_s + static_cast<uint32_t>(st * kRCTileBytes + (lane >> 3) * 128 + cc * 16);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (!EVEN && row0 + 16 * (i / 4) >= rows) break;
      cp_async16(dst + static_cast<uint32_t>(i * 512), src);
      src += 4 * ld;
    }
  };
  const I dtr = nwarps / tiles_c, dtc = nwarps - dtr * tiles_c;
  TileCursorT<I> cur, nxt;                                    // this tile, the one being copied
  cur.init(static_cast<I>(blockIdx.x) * (kRCThreads / 32) + warp, tiles_c);
  nxt = cur;
  if (nxt.tile < ntiles) issue(nxt, 0);
  cp_async_commit();
  nxt.advance(nwarps, dtr, dtc, tiles_c);
  // the tensor scale and the factor table are set up while the first tile
  // is already in flight
  TensorScale ts{1.0f, 1.0f};
  if (!MX) {
    ts = tensor_scale_q<QMAX>(*amax_ptr);
    fill_factor_table(rtab, ts.enc);
    if (blockIdx.x == 0 && threadIdx.x == 0 && s_dec_out) *s_dec_out = ts.dec;
  }
  __syncthreads();
  for (int st = 0; cur.tile < ntiles; cur.advance(nwarps, dtr, dtc, tiles_c), st ^= 1) {
    __syncwarp();   // every lane is done with stage st ^ 1 before it is refilled
    if (nxt.tile < ntiles) issue(nxt, st ^ 1);
    cp_async_commit();
    nxt.advance(nwarps, dtr, dtc, tiles_c);
    cp_async_wait<1>();
    __syncwarp();
    const I tr = cur.tt, tc = cur.tc;
    const I r0 = tr * G::WR + band * 16, c0 = tc * G::WC + cc * CPT;
    const bool valid = EVEN || (r0 < rows && c0 < cols);
    // row k of this thread's 16: tb[8 * k] (rows outside the matrix are never
    // copied; their lanes' values only meet other outside lanes and are not stored)
    const uint4 *tb = stage_g + st * (kRCTileBytes / 16) + band * 16 * 8 + cc;
    // ---- pass 1: block maxima --------------------------------------------
    float rmax[16];
    uint32_t cm[4] = {0u, 0u, 0u, 0u};
    if (sizeof(T) == 2) {
#pragma unroll
      for (int k = 0; k < 16; k += 2) {
        const uint4 a = tb[8 * k], b = tb[8 * k + 8];
        chunk_colmax<T>(a, cm);
        chunk_colmax<T>(b, cm);
        uint32_t pm = rowpair_max_bf16(a, b);
#pragma unroll
        for (int o = 1; o < GR; o <<= 1) pm = maxabs_bf16x2(pm, __shfl_xor_sync(0xFFFFFFFFu, pm, o));
        pm &= 0x7FFF7FFFu;
        rmax[k] = __uint_as_float(pm << 16);
        rmax[k + 1] = __uint_as_float(pm & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const uint4 a = tb[8 * k];
        chunk_colmax<T>(a, cm);
        rmax[k] = chunk_rowmax<T>(a);
      }
#pragma unroll
      for (int o = 1; o < GR; o <<= 1)
#pragma unroll
        for (int k = 0; k < 16; ++k)
          rmax[k] = fmaxf(rmax[k], __shfl_xor_sync(0xFFFFFFFFu, rmax[k], o));
    }
    float cmax[CPT];
    if (sizeof(T) == 2) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t m = cm[j] & 0x7FFF7FFFu;
        cmax[(2 * j) % CPT] = __uint_as_float(m << 16);
        cmax[(2 * j + 1) % CPT] = __uint_as_float(m & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int j = 0; j < CPT; ++j) cmax[j] = __uint_as_float(cm[j % 4]);
    }
    if (MX) {   // a 32-row column block spans two row bands
#pragma unroll
      for (int j = 0; j < CPT; ++j) cmax[j] = fmaxf(cmax[j], __shfl_xor_sync(0xFFFFFFFFu, cmax[j], 8));
    }

    // ---- scales --------------------------------------------------------------
    // the GR lanes of a row block share its 16 row maxima: lane gi of the
    // group computes the scales of rows gi, gi + GR, ... and the factors are
    // gathered back by shuffles
    constexpr int RPL = 16 / GR;                      // rows per lane
    const int gi = cc % GR;
    float rf[16], cf[CPT], own_f[RPL];
    uint32_t cbyte[CPT];
    {
      // rows r0..r0+15 of one block column: in the swizzled layout they are
      // 16 bytes apart (r0 is a multiple of 16), in the linear one cols/BLK
      const I step = swz ? 16 : cols / BLK;
      uint8_t *srow = sf_row + scale_offset_t<I>(r0, c0 / BLK, cols / BLK, scale_layout) + gi * step;
      float mrow[RPL];
#pragma unroll
      for (int i = 0; i < RPL; ++i) {
        float m = rmax[i * GR];
#pragma unroll
        for (int g = 1; g < GR; ++g)
          if (g == gi) m = rmax[i * GR + g];
        mrow[i] = m;
      }
      if (!MX && QMAX == 6 && RPL % 2 == 0) {
#pragma unroll
        for (int i = 0; i < RPL; i += 2) {
          const uint32_t c2 = nvfp4_scale_code2(mrow[i], mrow[i + 1], ts.enc);
          own_f[i] = rtab[c2 & 0xFFu];
          own_f[i + 1] = rtab[c2 >> 8];
          if (valid && do_row) {
            srow[i * GR * step] = static_cast<uint8_t>(c2);
            srow[(i + 1) * GR * step] = static_cast<uint8_t>(c2 >> 8);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
          const uint32_t b = block_scale<T, MX, QMAX>(mrow[i], ts, rtab, e8m0_mode, own_f[i]);
          if (valid && do_row) srow[i * GR * step] = static_cast<uint8_t>(b);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 16; ++k)
      rf[k] = GR == 1 ? own_f[k] : __shfl_sync(0xFFFFFFFFu, own_f[k / GR], lane - gi + k % GR);
    if (!MX && QMAX == 6) {
#pragma unroll
      for (int j = 0; j < CPT; j += 2) {
        const uint32_t c2 = nvfp4_scale_code2(cmax[j], cmax[j + 1], ts.enc);
        cbyte[j] = c2 & 0xFFu;
        cbyte[j + 1] = c2 >> 8;
        cf[j] = rtab[cbyte[j]];
        cf[j + 1] = rtab[cbyte[j + 1]];
      }
    } else {
#pragma unroll
      for (int j = 0; j < CPT; ++j) cbyte[j] = block_scale<T, MX, QMAX>(cmax[j], ts, rtab, e8m0_mode, cf[j]);
    }
    if (valid && do_col && (!MX || (band & 1) == 0)) {
      const I base = scale_offset_t<I>(c0, r0 / BLK, rows / BLK, scale_layout);
      const I step = swz ? 16 : rows / BLK;
#pragma unroll
      for (int j = 0; j < CPT; ++j) sf_col[base + j * step] = static_cast<uint8_t>(cbyte[j]);
    }

    // ---- pass 2: encode, four rows at a time ----------------------------------
    // read the rows from shared memory again rather than keeping all 16 live
    // (the warp barrier keeps the second reads from being hoisted into pass 1)
    __syncwarp();
    uint32_t colw[CPT][2];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      float v[4][CPT];
#pragma unroll
      for (int i = 0; i < 4; ++i) unpack_chunk<T>(tb[8 * (4 * q4 + i)], v[i]);
      uint32_t u[4][CPT];
      if (SR) {
        // one Philox call covers the 8 columns of a row from a multiple of 8
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint64_t idx = static_cast<uint64_t>((r0 + 4 * q4 + i) * cols + c0);
          const uint64_t gi = idx / 8;
          const U32x4 bits = philox(K, static_cast<uint32_t>(gi),
                                    I32 ? 0u : static_cast<uint32_t>(gi >> 32), 0u, 0u);
          const uint32_t words[4] = {bits.x, bits.y, bits.z, bits.w};
#pragma unroll
          for (int j = 0; j < CPT; ++j) {
            const int e = static_cast<int>(idx % 8) + j;
            const uint32_t wv = words[(e >> 1) & 3];
            u[i][j] = (e & 1) ? sr_x_hi(wv) : sr_x_lo(wv);   // 64 times the 16-bit uniform
          }
        }
      }
      if (do_row) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k = 4 * q4 + i;
          uint32_t wr = 0u;
          float t[8];
#pragma unroll
          for (int j = 0; j < CPT; j += 2) {
            const float2 p = mul2(make_float2(v[i][j], v[i][j + 1]), make_float2(rf[k], rf[k]));
            const float2 q = SR ? e2m1_sr_dithered2(p, u[i][j], u[i][j + 1]) : p;
            t[j] = q.x;
            t[j + 1] = q.y;
          }
          if (SR)
            wr = CPT == 8 ? e2m1x8_rz(t) : e2m1x4_rz(t[0], t[1], t[2 % CPT], t[3 % CPT]);
          else
            wr = CPT == 8 ? e2m1x8(t) : e2m1x4(t[0], t[1], t[2 % CPT], t[3 % CPT]);
          if (valid) {
            uint8_t *qa = q_row + (r0 + k) * (cols / 2) + c0 / 2;
            if (CPT == 8) *reinterpret_cast<uint32_t *>(qa) = wr;
            else *reinterpret_cast<uint16_t *>(qa) = static_cast<uint16_t>(wr);
          }
        }
      }
      if (do_col) {
#pragma unroll
        for (int j = 0; j < CPT; j += 2) {
          float2 p[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            p[i] = mul2(make_float2(v[i][j], v[i][j + 1]), make_float2(cf[j], cf[j + 1]));
          if (SR) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              p[i] = e2m1_sr_dithered2(p[i], u[i][j], u[i][j + 1]);
          }
          // column j, rows 4q4..4q4+3, and column j + 1
          const uint32_t h0 = SR ? e2m1x4_rz(p[0].x, p[1].x, p[2].x, p[3].x)
                                 : e2m1x4(p[0].x, p[1].x, p[2].x, p[3].x);
          const uint32_t h1 = SR ? e2m1x4_rz(p[0].y, p[1].y, p[2].y, p[3].y)
                                 : e2m1x4(p[0].y, p[1].y, p[2].y, p[3].y);
          if (q4 & 1) {
            colw[j][q4 >> 1] |= h0 << 16;
            colw[j + 1][q4 >> 1] |= h1 << 16;
          } else {
            colw[j][q4 >> 1] = h0;
            colw[j + 1][q4 >> 1] = h1;
          }
        }
      }
    }
    if (do_col && valid) {
#pragma unroll
      for (int j = 0; j < CPT; ++j)
        *reinterpret_cast<uint2 *>(q_col + (c0 + j) * (rows / 2) + r0 / 2) =
            make_uint2(colw[j][0], colw[j][1]);
    }
  }
  cp_async_wait<0>();
}


template <typename T, bool MX, bool SR, int QMAX, bool I32>
cudaError_t launch_typed2(const T *x, int64_t rows, int64_t cols, int64_t ld, unsigned layouts,
                         const float *amax, int e8m0_mode, uint64_t seed, float *s_dec_out,
                         uint8_t *q_row, uint8_t *sf_row, uint8_t *q_col, uint8_t *sf_col,
                         int scale_layout, const Launch &L) {
  constexpr int BLK = MX ? 32 : 16;
  if (layouts == FP4Q_ROWWISE) {
    const int64_t nblk = rows * (cols / BLK);
    static KernelSetup setup;
    int per_sm = 0;
    const cudaError_t e = kernel_setup(
        setup, reinterpret_cast<const void *>(rowwise_kernel<T, MX, SR, QMAX, I32>), kRowThreads, 0,
        &per_sm);
    if (e != cudaSuccess) return e;
    const int64_t cap = static_cast<int64_t>(per_sm) * L.num_sms;
    const int64_t want = (nblk + 2 * kRowThreads - 1) / (2 * kRowThreads);
    const int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
    rowwise_kernel<T, MX, SR, QMAX, I32><<<grid, kRowThreads, 0, L.stream>>>(
        x, rows, cols, ld, amax, e8m0_mode, seed, s_dec_out, q_row, sf_row, scale_layout);
  } else {
    using G = RCGeom<T, MX>;
    const int64_t ntiles = ((cols + G::WC - 1) / G::WC) * ((rows + G::WR - 1) / G::WR);
    const bool even = rows % G::WR == 0 && cols % G::WC == 0;   // whole warp tiles only
    const void *kern = even
        ? reinterpret_cast<const void *>(rowcol_kernel<T, MX, SR, QMAX, I32, true>)
        : reinterpret_cast<const void *>(rowcol_kernel<T, MX, SR, QMAX, I32, false>);
    static KernelSetup setup, setup_e;
    int per_sm = 0;
    const cudaError_t e = kernel_setup(even ? setup_e : setup, kern, kRCThreads, kRCSmem, &per_sm);
    if (e != cudaSuccess) return e;
    const int64_t cap = static_cast<int64_t>(per_sm) * L.num_sms;
    const int64_t want = (ntiles + kRCThreads / 32 - 1) / (kRCThreads / 32);
    const int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
    if (even)
      rowcol_kernel<T, MX, SR, QMAX, I32, true><<<grid, kRCThreads, kRCSmem, L.stream>>>(
          x, rows, cols, ld, layouts, amax, e8m0_mode, seed, s_dec_out, q_row, sf_row, q_col,
          sf_col, scale_layout);
    else
      rowcol_kernel<T, MX, SR, QMAX, I32, false><<<grid, kRCThreads, kRCSmem, L.stream>>>(
          x, rows, cols, ld, layouts, amax, e8m0_mode, seed, s_dec_out, q_row, sf_row, q_col,
          sf_col, scale_layout);
  }
  return cudaGetLastError();
}

// 32-bit index arithmetic where every element and input offset fits (then
// every stochastic-rounding counter (r * cols + c) / 8 fits in 32 bits too).
template <typename T, bool MX, bool SR, int QMAX = 6>
cudaError_t launch_typed(const T *x, int64_t rows, int64_t cols, int64_t ld, unsigned layouts,
                         const float *amax, int e8m0_mode, uint64_t seed, float *s_dec_out,
                         uint8_t *q_row, uint8_t *sf_row, uint8_t *q_col, uint8_t *sf_col,
                         int scale_layout, const Launch &L) {
  constexpr int64_t kLim = (int64_t{1} << 31) - (int64_t{1} << 24);
  if (rows * ld < kLim && rows * cols < kLim)
    return launch_typed2<T, MX, SR, QMAX, true>(x, rows, cols, ld, layouts, amax, e8m0_mode, seed,
                                               s_dec_out, q_row, sf_row, q_col, sf_col,
                                               scale_layout, L);
  return launch_typed2<T, MX, SR, QMAX, false>(x, rows, cols, ld, layouts, amax, e8m0_mode, seed,
                                              s_dec_out, q_row, sf_row, q_col, sf_col,
                                              scale_layout, L);
}

}  // namespace

cudaError_t launch_nvfp4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                         unsigned layouts, int round, uint64_t seed, const float *amax,
                         float *s_dec_out, uint8_t *q_row, uint8_t *sf_row, uint8_t *q_col,
                         uint8_t *sf_col, int scale_layout, const Launch &L) {
  const bool sr = round == FP4Q_SR;
  if (dtype == FP4Q_BF16) {
    auto *p = static_cast<const __nv_bfloat16 *>(x);
    return sr ? launch_typed<__nv_bfloat16, false, true>(p, rows, cols, ld, layouts, amax, 0, seed,
                                                         s_dec_out, q_row, sf_row, q_col, sf_col,
                                                         scale_layout, L)
              : launch_typed<__nv_bfloat16, false, false>(p, rows, cols, ld, layouts, amax, 0,
                                                          seed, s_dec_out, q_row, sf_row, q_col,
                                                          sf_col, scale_layout, L);
  }
  auto *p = static_cast<const float *>(x);
  return sr ? launch_typed<float, false, true>(p, rows, cols, ld, layouts, amax, 0, seed, s_dec_out,
                                               q_row, sf_row, q_col, sf_col, scale_layout, L)
            : launch_typed<float, false, false>(p, rows, cols, ld, layouts, amax, 0, seed,
                                                s_dec_out, q_row, sf_row, q_col, sf_col,
                                                scale_layout, L);
}

cudaError_t launch_four_over_six(const void *x, int dtype, int64_t rows, int64_t cols,
                                 int64_t ld, unsigned layouts, const float *amax,
                                 float *s_dec_out, uint8_t *q_row, uint8_t *sf_row,
                                 uint8_t *q_col, uint8_t *sf_col, int scale_layout,
                                 const Launch &L) {
  if (dtype == FP4Q_BF16)
    return launch_typed<__nv_bfloat16, false, false, 4>(
        static_cast<const __nv_bfloat16 *>(x), rows, cols, ld, layouts, amax, 0, 0, s_dec_out,
        q_row, sf_row, q_col, sf_col, scale_layout, L);
  return launch_typed<float, false, false, 4>(static_cast<const float *>(x), rows, cols, ld,
                                              layouts, amax, 0, 0, s_dec_out, q_row, sf_row,
                                              q_col, sf_col, scale_layout, L);
}

cudaError_t launch_mxfp4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                         unsigned layouts, int e8m0_mode, uint8_t *q_row, uint8_t *sf_row,
                         uint8_t *q_col, uint8_t *sf_col, int scale_layout, const Launch &L) {
  if (dtype == FP4Q_BF16)
    return launch_typed<__nv_bfloat16, true, false>(static_cast<const __nv_bfloat16 *>(x), rows,
                                                    cols, ld, layouts, nullptr, e8m0_mode, 0,
                                                    nullptr, q_row, sf_row, q_col, sf_col,
                                                    scale_layout, L);
  return launch_typed<float, true, false>(static_cast<const float *>(x), rows, cols, ld, layouts,
                                          nullptr, e8m0_mode, 0, nullptr, q_row, sf_row, q_col,
                                          sf_col, scale_layout, L);
}

}  // namespace fp4q
