// quant2d.cu -- NVFP4 with 16x16 2D block scaling for weights.
//
// Qiita note on NVFP4 training, "2D scaling": with 1x16 blocks q(W) differs
// from q(W^T)^T because the scaling direction changes under transposition;
// square 16x16 tiles give both the same scales, so W and W^T codes come out
// of one pass.
//
// Register tiles fed by a two-stage cp.async buffer: a warp owns 64 rows x
// 128 bytes (8 16-byte chunks of 4 FP32 or 8 BF16 columns) and copies the
// next such tile into shared memory while it encodes this one.  A thread
// owns 16 rows x one chunk; a 16x16 tile spans 4 (FP32) or 2 (BF16) lanes,
// whose partial maxima meet by shuffle (lane = chunk + 8 * row band), so a
// warp instruction writes W^T codes as whole 32-byte sectors (4 bands x 8
// bytes of one column).
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int kThreads = 128;
constexpr int kTileBytes = 64 * 128;               // one warp tile: 64 rows x 128 bytes
constexpr int kSmem = (kThreads / 32) * 2 * kTileBytes;

template <typename T>
__device__ __forceinline__ void unpack4or8(uint4 u, float (&v)[16 / sizeof(T)]) {
  if (sizeof(T) == 2) {
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4 % (16 / sizeof(T))] = bf16_lo(u.z); v[5 % (16 / sizeof(T))] = bf16_hi(u.z);
    v[6 % (16 / sizeof(T))] = bf16_lo(u.w); v[7 % (16 / sizeof(T))] = bf16_hi(u.w);
  } else {
    v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
quant2d_kernel(const T *__restrict__ w, int64_t rows, int64_t cols, int64_t ld,
               const float *__restrict__ amax_ptr, float *__restrict__ s_dec_out,
               uint8_t *__restrict__ q_w, uint8_t *__restrict__ q_wt,
               uint8_t *__restrict__ sf_tiles, uint8_t *__restrict__ sf_w_1x16,
               uint8_t *__restrict__ sf_wt_1x16, int scale_layout) {
  constexpr int CPT = 16 / sizeof(T);       // columns per thread
  constexpr int LPT = 16 / CPT;             // lanes per tile
  constexpr int WC = 8 * CPT;               // warp tile columns
  __shared__ float rtab[128];

  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, cc = lane & 7, band = lane >> 3, warp = threadIdx.x >> 5;
  const int li = cc % LPT;                  // lane index within the tile
  const int64_t tiles_c = (cols + WC - 1) / WC;
  const int64_t ntiles = tiles_c * ((rows + 63) / 64);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  const int64_t dtr = nwarps / tiles_c, dtc = nwarps - dtr * tiles_c;
  const uint32_t stage_s = static_cast<uint32_t>(__cvta_generic_to_shared(smem)) +
                           static_cast<uint32_t>(warp * 2 * kTileBytes);
  const uint4 *stage_g = reinterpret_cast<const uint4 *>(smem + warp * 2 * kTileBytes);
  // lane L copies the 16-byte pieces L + 32 i: row (L + 32 i) / 8, chunk L % 8;
  // each warp copy instruction moves four whole 128-byte row segments
  // row (L >> 3) + 4 i lies in the 16-row band i / 4 for every lane, and rows
  // is a multiple of 16, so the row bound is one test per band
  auto issue = [&](const TileCursor &t, int st) {
    const int64_t col = t.tc * WC + cc * CPT;
    if (col >= cols) return;
    const int64_t row0 = t.tt * 64;
    const T *src = w + (row0 + (lane >> 3)) * ld + col;
    const uint32_t dst =
        stage_s + static_cast<uint32_t>(st * kTileBytes + (lane >> 3) * 128 + cc * 16);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (row0 + 16 * (i / 4) >= rows) break;
      cp_async16(dst + static_cast<uint32_t>(i * 512), src);
      src += 4 * ld;
    }
  };
  TileCursor cur, nxt;                                    // this tile, the one being copied
  cur.init(static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + warp, tiles_c);
  nxt = cur;
  if (nxt.tile < ntiles) issue(nxt, 0);
  cp_async_commit();
  nxt.advance(nwarps, dtr, dtc, tiles_c);
  // the tensor scale and the factor table are set up while the first tile
  // is already in flight
  const TensorScale ts = tensor_scale(*amax_ptr);
  fill_factor_table(rtab, ts.enc);
  if (blockIdx.x == 0 && threadIdx.x == 0 && s_dec_out) *s_dec_out = ts.dec;
  __syncthreads();
  for (int st = 0; cur.tile < ntiles; cur.advance(nwarps, dtr, dtc, tiles_c), st ^= 1) {
    __syncwarp();   // every lane is done with stage st ^ 1 before it is refilled
    if (nxt.tile < ntiles) issue(nxt, st ^ 1);
    cp_async_commit();
    nxt.advance(nwarps, dtr, dtc, tiles_c);
    cp_async_wait<1>();
    __syncwarp();
    const int64_t r0 = cur.tt * 64 + band * 16, c0 = cur.tc * WC + cc * CPT;
    const bool valid = r0 < rows && c0 < cols;   // the whole 16x16 tile shares validity
    // rows outside the matrix are never copied; their lanes' values only meet
    // other outside lanes and are not stored
    const uint4 *tb = stage_g + st * (kTileBytes / 16) + band * 16 * 8 + cc;
    uint4 d[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) d[k] = tb[8 * k];
    float m;
    if (sizeof(T) == 2) {
      uint32_t mm = 0u;
#pragma unroll
      for (int k = 0; k < 16; ++k)
        mm = maxabs_bf16x2(mm, maxabs_bf16x2(maxabs_bf16x2(d[k].x, d[k].y),
                                             maxabs_bf16x2(d[k].z, d[k].w)));
      m = bf16x2_hmax(mm);
    } else {
      m = 0.0f;
#pragma unroll
      for (int k = 0; k < 16; ++k)
        m = fmaxf(m, fmaxf(fmaxf(fabsf(__uint_as_float(d[k].x)), fabsf(__uint_as_float(d[k].y))),
                           fmaxf(fabsf(__uint_as_float(d[k].z)), fabsf(__uint_as_float(d[k].w)))));
    }
#pragma unroll
    for (int o = 1; o < LPT; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (!valid) continue;

    const uint32_t sbyte = nvfp4_scale_code(m, ts.enc);
    const float f = rtab[sbyte];
    const int64_t gr = r0, gc = c0 - li * CPT;        // tile origin
    uint32_t colw[CPT][2];
#pragma unroll
    for (int j = 0; j < CPT; ++j) colw[j][0] = colw[j][1] = 0u;
#pragma unroll
    for (int k = 0; k < 16; k += 2) {
      float a[CPT], b[CPT];
      unpack4or8<T>(d[k], a);
      unpack4or8<T>(d[k + 1], b);
#pragma unroll
      for (int j = 0; j < CPT; j += 2) {
        const float2 pa = mul2(make_float2(a[j], a[j + 1]), make_float2(f, f));
        const float2 pb = mul2(make_float2(b[j], b[j + 1]), make_float2(f, f));
        a[j] = pa.x; a[j + 1] = pa.y; b[j] = pb.x; b[j + 1] = pb.y;
      }
      if (q_w) {
        uint32_t wa = 0u, wb = 0u;
#pragma unroll
        for (int j = 0; j < CPT; j += 2) {
          wa |= e2m1x2(a[j], a[j + 1]) << (4 * j);
          wb |= e2m1x2(b[j], b[j + 1]) << (4 * j);
        }
        uint8_t *qa = q_w + (r0 + k) * (cols / 2) + c0 / 2;
        if (CPT == 8) {
          *reinterpret_cast<uint32_t *>(qa) = wa;
          *reinterpret_cast<uint32_t *>(qa + cols / 2) = wb;
        } else {
          *reinterpret_cast<uint16_t *>(qa) = static_cast<uint16_t>(wa);
          *reinterpret_cast<uint16_t *>(qa + cols / 2) = static_cast<uint16_t>(wb);
        }
      }
      if (q_wt) {
#pragma unroll
        for (int j = 0; j < CPT; ++j)   // column j: rows k (low nibble), k + 1
          colw[j][k >> 3] |= e2m1x2(a[j], b[j]) << (8 * ((k >> 1) & 3));
      }
    }
    if (q_wt) {
#pragma unroll
      for (int j = 0; j < CPT; ++j)
        *reinterpret_cast<uint2 *>(q_wt + (c0 + j) * (rows / 2) + r0 / 2) =
            make_uint2(colw[j][0], colw[j][1]);
    }
    const uint8_t sb = static_cast<uint8_t>(sbyte);
    if (li == 0) sf_tiles[(gr / 16) * (cols / 16) + gc / 16] = sb;
    if (sf_w_1x16) {
#pragma unroll
      for (int k = 0; k < 16 / LPT; ++k)
        sf_w_1x16[scale_offset(gr + li * (16 / LPT) + k, gc / 16, cols / 16, scale_layout)] = sb;
    }
    if (sf_wt_1x16) {
#pragma unroll
      for (int j = 0; j < CPT; ++j)
        sf_wt_1x16[scale_offset(c0 + j, gr / 16, rows / 16, scale_layout)] = sb;
    }
  }
  cp_async_wait<0>();
}

}  // namespace

cudaError_t launch_2d(const void *w, int dtype, int64_t rows, int64_t cols, int64_t ld,
                      const float *amax, float *s_dec_out, uint8_t *q_w, uint8_t *q_wt,
                      uint8_t *sf_tiles, uint8_t *sf_w_1x16, uint8_t *sf_wt_1x16,
                      int scale_layout, const Launch &L) {
  const int cpt = dtype == FP4Q_BF16 ? 8 : 4;
  const int64_t ntiles = ((cols + 8 * cpt - 1) / (8 * cpt)) * ((rows + 63) / 64);
  const bool bf = dtype == FP4Q_BF16;
  const void *kern = bf ? reinterpret_cast<const void *>(quant2d_kernel<__nv_bfloat16>)
                        : reinterpret_cast<const void *>(quant2d_kernel<float>);
  static KernelSetup setup_t[2];
  int per_sm = 0;
  const cudaError_t e = kernel_setup(setup_t[bf ? 1 : 0], kern, kThreads, kSmem, &per_sm);
  if (e != cudaSuccess) return e;
  const int64_t cap = static_cast<int64_t>(per_sm) * L.num_sms;
  const int64_t want = (ntiles + kThreads / 32 - 1) / (kThreads / 32);
  const int grid = static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
  if (dtype == FP4Q_BF16)
    quant2d_kernel<__nv_bfloat16><<<grid, kThreads, kSmem, L.stream>>>(
        static_cast<const __nv_bfloat16 *>(w), rows, cols, ld, amax, s_dec_out, q_w, q_wt,
        sf_tiles, sf_w_1x16, sf_wt_1x16, scale_layout);
  else
    quant2d_kernel<float><<<grid, kThreads, kSmem, L.stream>>>(
        static_cast<const float *>(w), rows, cols, ld, amax, s_dec_out, q_w, q_wt, sf_tiles,
        sf_w_1x16, sf_wt_1x16, scale_layout);
  return cudaGetLastError();
}

}  // namespace fp4q
