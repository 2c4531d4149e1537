// gemm.cu -- block-scaled NVFP4 GEMM on the sm_100a tensor cores: the
// consumer of the quantized operands.
//
// Qiita note on NVFP4 training: the NVFP4 operands feed FP4 GEMMs (Fprop
// X W^T from the row-wise copies, Wgrad dY^T X from the column-wise ones),
// each 16-value block's E2M1 codes times its E4M3 block scale, the two
// FP32 tensor scales applied to the product.  This kernel reads the
// library's outputs as they are: codes [rows, K/2] (K-major) and block
// scales in the 128x4 tile layout, which is the layout the tensor core's
// scale-factor copy expects, so nothing is repacked.
//
//   C[m, n] = RN(acc[m, n] * RN(s_a * s_b)),
//   acc[m, n] = sum_k (g_a[m,k] S_a[m,k/16]) (g_b[n,k] S_b[n,k/16])   (FP32)
//
// The kernel is persistent: one CTA per SM walks the 128 x BN output tiles
// (BN = 256, or 128 when N is not a multiple of 256) in row-major order,
// taking every gridDim-th tile, with six warps in three roles:
//  - one thread of warp 0 is the producer: for every K-tile of 256 values of
//    every tile it loads the A and B code tiles with TMA (cp.async.bulk.tensor,
//    128-byte swizzle, which is the K-major layout the MMA descriptors
//    describe) and the 2 KiB scale blocks with plain bulk copies (the 128x4
//    tiles of one K-tile are contiguous in the swizzled layout), completing on
//    the stage's "full" mbarrier; four stages, one stream across tiles, so the
//    next tile's first K-tiles load while the current one finishes;
//  - one thread of warp 1 issues the tensor-core work: tcgen05.cp
//    32x128b.warpx4 of each 512-byte scale tile into tensor memory (4
//    columns per 64-value K step and 128 rows), then four tcgen05.mma
//    kind::mxf4nvf4 block16 (M = 128, N = BN, K = 64) accumulating in tensor
//    memory, then tcgen05.commit to the stage's "empty" mbarrier; after the
//    last K-tile it commits to "acc_full", and it starts the next tile only
//    once the epilogue has signalled "acc_empty";
//  - warps 2-5 are the epilogue: each reads its 32 accumulator rows with
//    tcgen05.ld (warp w reaches lanes 32 (w % 4) .. + 31), scales by
//    RN(s_a s_b), hands tensor memory back (for BF16 output as soon as the
//    row is in registers) and writes C.
// No load uses cluster multicast.  Every mbarrier wait is bounded (about a
// second of clock cycles); a wait that runs out sets *status, the roles stop
// issuing, and the CTA waits (bounded) for its tensor-core work, frees its
// tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int BM = 128;
constexpr int KTILE = 256;                       // K values per stage
constexpr int KTB = KTILE / 2;                   // 128 code bytes per row per stage
constexpr int kThreads = 192;                    // producer warp, MMA warp, 4 epilogue warps
constexpr int SF_TILE = 512;                     // 128 rows x 4 scales
constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at the B200's clock

// NA A operands per output tile: 1 (NVFP4), or 3 (the IF4 split: the FP4
// blocks accumulate into one accumulator, the two E2M1 parts of the INT4
// blocks into a second; all three share the A scales).  VS is the scale
// block: 16 values with E4M3 scales (NVFP4, kind::mxf4nvf4 block16) or 32
// values with E8M0 scales (MXFP4, kind::mxf4 block32).
template <int BN, int NA = 1, int VS = 16>
struct Tile {
  static constexpr int STAGES = NA == 1 ? 4 : 3;
  static constexpr int NACC = NA == 1 ? 1 : 2;
  // one 512-byte 128x4 scale tile covers 4 VS-value blocks of K
  static constexpr int SF_TILES = KTILE / (4 * VS);            // per K-tile: 4 or 2
  static constexpr int SF_BYTES = SF_TILES * SF_TILE;          // one operand row tile, one K-tile
  static constexpr int A_BYTES = BM * KTB;                      // 16384 per A operand
  static constexpr int B_BYTES = BN * KTB;                      // 16384 or 32768
  static constexpr int B_OFF = NA * A_BYTES;
  static constexpr int SFB_BYTES = (BN / 128) * SF_BYTES;       // [row tile][K step][512]
  static constexpr int STAGE_BYTES = NA * A_BYTES + B_BYTES + SF_BYTES + SFB_BYTES;
  static constexpr int BAR_BYTES = 128;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  // tensor memory: NACC accumulators of BN columns, then per stage 4 columns
  // per A scale tile and 4 per B scale tile
  static constexpr uint32_t SF_COL0 = NACC * BN;
  static constexpr uint32_t SFA_COLS = 4 * SF_TILES;
  static constexpr uint32_t SFB_COLS = 4 * SF_TILES * (BN / 128);
  static constexpr uint32_t STAGE_COLS = SFA_COLS + SFB_COLS;
  static constexpr uint32_t COLS_USED = NACC * BN + STAGES * STAGE_COLS;
  static constexpr uint32_t TMEM_COLS = COLS_USED <= 256 ? 256 : 512;
  // Instruction descriptor of the block-scaled tcgen05.mma: A and B E2M1
  // (format 1), K-major, N (bits 17-22 = N/8), M = 128 (bits 24-28 = M/16),
  // dense, K = 64, scale format in bit 23 (0 = E4M3, 1 = E8M0); the scale
  // byte within each 32-bit tensor-memory cell goes in bits 29-30 (A) and
  // 4-5 (B) per instruction.
  static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                                    (VS == 32 ? (1u << 23) : 0u) | (uint32_t(BM >> 4) << 24);
  static_assert(VS == 16 || VS == 32, "scale block of 16 (NVFP4) or 32 (MXFP4)");
  static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static_assert(COLS_USED <= 512, "tensor memory");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory matrix descriptor, K-major with 128-byte swizzle: rows of
// 128 bytes, 8-row groups 1024 bytes apart (SBO), LBO 1 (unused for this
// layout), descriptor version 1, layout type 2.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (uint64_t{1} << 16) |
         (uint64_t{1024 >> 4} << 32) | (uint64_t{1} << 46) | (uint64_t{2} << 61);
}

// Descriptor of one 512-byte scale tile for the 32x128b copy: 32 rows of 16
// bytes, no swizzle, 8-row groups 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (uint64_t{128 >> 4} << 32) |
         (uint64_t{1} << 46);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// true once the phase with this parity has completed; false after about a
// second without completion
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_test(bar, parity))
    if (clock64() - t0 > kWaitCycles) return false;
  return true;
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tc_copy_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}
template <int VS>
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  if (VS == 16)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], "
        "[%6], p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], "
        "[%6], p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// 16 consecutive FP32 accumulator columns of this thread's row (warp w reads
// lanes 32 (w % 4) .. + 31); the wait is separate so that loads can overlap
__device__ __forceinline__ void tc_load16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// TMA tile load of a 2-D box (x in bytes along the row, y rows), completing
// on an mbarrier; no multicast
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// contiguous bulk copy (16-byte aligned, size a multiple of 16) completing
// on an mbarrier; no multicast
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

template <typename OutT, int BN, int NA, int VS>
__global__ void __launch_bounds__(kThreads, 1)
gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap map_a,
                  const __grid_constant__ CUtensorMap map_a1,
                  const __grid_constant__ CUtensorMap map_a2,
                  const __grid_constant__ CUtensorMap map_b, const uint8_t *__restrict__ sfa,
                  const float *__restrict__ s_a, const uint8_t *__restrict__ sfb,
                  const float *__restrict__ s_b, int K, int n_tiles_n, int n_tiles,
                  OutT *__restrict__ c, int64_t ldc, int *__restrict__ status,
                  GemmOptions opt) {
  using T = Tile<BN, NA, VS>;
  constexpr int STAGES = T::STAGES;
  constexpr int SF_BYTES = T::SF_BYTES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t full = base + STAGES * T::STAGE_BYTES;   // STAGES "full" barriers
  const uint32_t empty = full + 8 * STAGES;               // STAGES "empty" barriers
  const uint32_t acc_full = empty + 8 * STAGES;           // accumulator written
  const uint32_t acc_empty = acc_full + 8;                // accumulator read out
  const uint32_t tmem_slot = acc_empty + 8;
  const uint32_t err_slot = tmem_slot + 4;
  volatile uint32_t *slot_ptr = reinterpret_cast<volatile uint32_t *>(smem_raw + (tmem_slot - raw));
  volatile int *err_ptr = reinterpret_cast<volatile int *>(smem_raw + (err_slot - raw));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KT = K / KTILE;
  // bytes of the scales of one 128-row tile: K / (4 VS) tiles of 512 bytes
  const int64_t sf_rowtile = static_cast<int64_t>(K / (4 * VS)) * SF_TILE;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     tmem_slot),
                 "r"(T::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(full + 8 * i, 1);
      mbar_init(empty + 8 * i, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);                              // one arrival per epilogue warp
    *err_ptr = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot_ptr;

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer: the K-tiles of this CTA's output tiles, one stream ----
      int g = 0;                                          // K-tiles issued so far
      // withhold (a failure-detection test hook): issue nothing, so that the
      // MMA thread's first wait runs out
      for (int tile = blockIdx.x; tile < n_tiles && !*err_ptr && !opt.withhold;
           tile += gridDim.x) {
        const int m0 = (tile / n_tiles_n) * BM, n0 = (tile % n_tiles_n) * BN;
        const uint8_t *sfa_tile = sfa + static_cast<int64_t>(m0 / BM) * sf_rowtile;
        const uint8_t *sfb_tile = sfb + static_cast<int64_t>(n0 / 128) * sf_rowtile;
        for (int kt = 0; kt < KT; ++kt, ++g) {
          const int s = g % STAGES;
          if (g >= STAGES &&
              !mbar_wait(empty + 8 * s, static_cast<uint32_t>((g / STAGES - 1) & 1))) {
            *err_ptr = 1;
            break;
          }
          const uint32_t st = base + s * T::STAGE_BYTES;
          const uint32_t bar = full + 8 * s;
          mbar_expect_tx(bar, T::STAGE_BYTES);
          tma_load_2d(st, &map_a, kt * KTB, m0, bar);
          if (NA == 3) {
            tma_load_2d(st + T::A_BYTES, &map_a1, kt * KTB, m0, bar);
            tma_load_2d(st + 2 * T::A_BYTES, &map_a2, kt * KTB, m0, bar);
          }
          tma_load_2d(st + T::B_OFF, &map_b, kt * KTB, n0, bar);
          bulk_load(st + T::B_OFF + T::B_BYTES, sfa_tile + static_cast<int64_t>(kt) * SF_BYTES,
                    SF_BYTES, bar);
#pragma unroll
          for (int h = 0; h < BN / 128; ++h)
            bulk_load(st + T::B_OFF + T::B_BYTES + SF_BYTES + h * SF_BYTES,
                      sfb_tile + h * sf_rowtile + static_cast<int64_t>(kt) * SF_BYTES, SF_BYTES,
                      bar);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- tensor-core issue ----
      int g = 0, i = 0;                                   // K-tiles consumed, tiles done
      for (int tile = blockIdx.x; tile < n_tiles && !*err_ptr; tile += gridDim.x, ++i) {
        // the epilogue must have read the previous tile's accumulator
        if (i > 0 && !mbar_wait(acc_empty, static_cast<uint32_t>((i - 1) & 1))) {
          *err_ptr = 1;
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < KT; ++kt, ++g) {
          const int s = g % STAGES;
          if (!mbar_wait(full + 8 * s, static_cast<uint32_t>((g / STAGES) & 1))) {
            *err_ptr = 1;
            break;
          }
          tc_fence_after();
          const uint32_t st = base + s * T::STAGE_BYTES;
          const uint32_t sfa_col = tmem + T::SF_COL0 + T::STAGE_COLS * s;
          const uint32_t sfb_col = sfa_col + T::SFA_COLS;
          // scale tile t (4 VS-value blocks of K) of every operand row tile
          // into 4 tensor-memory columns: A at sfa_col + 4 t, B rows
          // 128 h .. 128 h + 127 at sfb_col + 4 (BN / 128) t + 4 h
#pragma unroll
          for (int t = 0; t < T::SF_TILES; ++t) {
            tc_copy_sf(sfa_col + 4u * t, desc_sf(st + T::B_OFF + T::B_BYTES + t * SF_TILE));
#pragma unroll
            for (int h = 0; h < BN / 128; ++h)
              tc_copy_sf(sfb_col + 4u * (BN / 128) * t + 4u * h,
                         desc_sf(st + T::B_OFF + T::B_BYTES + SF_BYTES + h * SF_BYTES +
                                 t * SF_TILE));
          }
          const uint64_t da = desc_sw128(st), db = desc_sw128(st + T::B_OFF);
#pragma unroll
          for (int kb = 0; kb < KTILE / 64; ++kb) {     // 64 values = 32 bytes = 2 descriptor units
            // the scales of these 64 values: all four bytes of tile kb
            // (VS 16), or bytes 2 (kb % 2) and up of tile kb / 2 (VS 32); the
            // byte goes in the address's top bits and in the descriptor
            const uint32_t t = VS == 16 ? kb : kb / 2, id = VS == 16 ? 0u : 2u * (kb & 1);
            const uint32_t sa = (sfa_col + 4u * t) | (id << 30);
            const uint32_t sb = (sfb_col + 4u * (BN / 128) * t) | (id << 30);
            const uint32_t idesc = T::IDESC | (id << 29) | (id << 4);
            tc_mma<VS>(tmem, da + 2u * kb, db + 2u * kb, idesc, sa, sb, (kt | kb) != 0);
            if (NA == 3) {                              // both INT4 parts into accumulator 1
              const uint64_t da1 = desc_sw128(st + T::A_BYTES), da2 = desc_sw128(st + 2 * T::A_BYTES);
              tc_mma<VS>(tmem + BN, da1 + 2u * kb, db + 2u * kb, idesc, sa, sb, (kt | kb) != 0);
              tc_mma<VS>(tmem + BN, da2 + 2u * kb, db + 2u * kb, idesc, sa, sb, 1u);
            }
          }
          tc_commit(empty + 8 * s);
        }
        tc_commit(acc_full);                            // this tile's accumulator is complete
      }
    }
  } else {
    // ---- epilogue: warp w reads accumulator lanes 32 (w % 4) .. + 31 ----
    const int quarter = warp & 3;
    const float a0 =
        __fmul_rn(__fmul_rn(s_a ? *s_a : 1.0f, s_b ? *s_b : 1.0f), opt.alpha_mul);
    const float a1 = __fmul_rn(a0, opt.alpha_int);     // the second accumulator's factor
    // with two accumulators the combined value is formed first and then
    // multiplied by 1 (exact) in the conversions below
    const float alpha = NA == 3 ? 1.0f : a0;
    // 16 columns of this thread's row, combined from both accumulators (NA 3)
    auto load_chunk = [&](uint32_t taddr, int j, uint32_t (&r)[16]) {
      tc_load16(taddr + 16u * j, r);
      if (NA == 3) {
        uint32_t r1[16];
        tc_load16(taddr + BN + 16u * j, r1);
        tc_wait_ld();
#pragma unroll
        for (int q = 0; q < 16; ++q)
          r[q] = __float_as_uint(__fadd_rn(__fmul_rn(__uint_as_float(r[q]), a0),
                                           __fmul_rn(__uint_as_float(r1[q]), a1)));
      } else {
        tc_wait_ld();
      }
    };
    int i = 0;
    for (int tile = blockIdx.x; tile < n_tiles && !*err_ptr; tile += gridDim.x, ++i) {
      const int ok = mbar_wait(acc_full, static_cast<uint32_t>(i & 1)) ? 1 : 0;
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        *err_ptr = 1;
        break;
      }
      tc_fence_after();
      const int m0 = (tile / n_tiles_n) * BM, n0 = (tile % n_tiles_n) * BN;
      OutT *row = c + (static_cast<int64_t>(m0) + quarter * 32 + lane) * ldc + n0;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
      if (sizeof(OutT) == 2) {
        // BF16: the whole converted row (BN / 2 words) stays in registers, so
        // tensor memory is handed back before the stores
        uint32_t w[BN / 2];
#pragma unroll
        for (int j = 0; j < BN / 16; ++j) {
          uint32_t r[16];
          load_chunk(taddr, j, r);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[2 * q]), alpha),
                                                      __fmul_rn(__uint_as_float(r[2 * q + 1]), alpha));
            memcpy(&w[8 * j + q], &b2, sizeof(uint32_t));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(acc_empty) : "memory");
        uint4 *d = reinterpret_cast<uint4 *>(row);
#pragma unroll
        for (int q = 0; q < BN / 8; ++q) d[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      } else {
        // FP32: chunk by chunk; tensor memory is handed back after the last load
        float4 *d = reinterpret_cast<float4 *>(row);
#pragma unroll
        for (int j = 0; j < BN / 16; ++j) {
          uint32_t r[16];
          load_chunk(taddr, j, r);
          if (j == BN / 16 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
              asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(acc_empty) : "memory");
          }
#pragma unroll
          for (int q = 0; q < 4; ++q)
            d[4 * j + q] = make_float4(__fmul_rn(__uint_as_float(r[4 * q]), alpha),
                                       __fmul_rn(__uint_as_float(r[4 * q + 1]), alpha),
                                       __fmul_rn(__uint_as_float(r[4 * q + 2]), alpha),
                                       __fmul_rn(__uint_as_float(r[4 * q + 3]), alpha));
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && status && *err_ptr) atomicExch(status, 1);
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(T::TMEM_COLS)
                 : "memory");
}

// cuTensorMapEncodeTiled, reached through the runtime (no link to the driver
// library)
PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    cudaGetLastError();
  });
  return fn;
}

// A [rows, row_bytes] byte matrix read as boxes of 128 bytes x box_rows rows
// into 128-byte-swizzled shared memory.
bool make_map(CUtensorMap *map, const uint8_t *base, int64_t rows, int64_t row_bytes,
              int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(KTB), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename OutT, int BN, int NA, int VS = 16>
cudaError_t launch_t(const uint8_t *const (&qa)[3], const uint8_t *sfa, const float *s_a,
                     const uint8_t *qb, const uint8_t *sfb, const float *s_b, int64_t M,
                     int64_t N, int64_t K, void *c, int64_t ldc, int *status, GemmOptions opt,
                     const Launch &L) {
  using T = Tile<BN, NA, VS>;
  static KernelSetup setup;
  int per_sm = 0;
  const cudaError_t e =
      kernel_setup(setup, reinterpret_cast<const void *>(gemm_nvfp4_kernel<OutT, BN, NA, VS>),
                   kThreads, T::SMEM_BYTES, &per_sm);
  if (e != cudaSuccess) return e;
  CUtensorMap map_a[3], map_b;
  for (int i = 0; i < 3; ++i)
    if (!make_map(&map_a[i], qa[NA == 3 ? i : 0], M, K / 2, BM)) return cudaErrorInvalidValue;
  if (!make_map(&map_b, qb, N, K / 2, BN)) return cudaErrorInvalidValue;
  // persistent: one CTA per SM (the stages fill its shared memory), output
  // tiles in row-major order, each CTA taking every gridDim-th tile
  const int64_t n_tiles_n = N / BN, n_tiles = (M / BM) * n_tiles_n;
  const int grid = static_cast<int>(n_tiles < L.num_sms ? n_tiles : L.num_sms);
  gemm_nvfp4_kernel<OutT, BN, NA, VS><<<grid, kThreads, T::SMEM_BYTES, L.stream>>>(
      map_a[0], map_a[1], map_a[2], map_b, sfa, s_a, sfb, s_b, static_cast<int>(K),
      static_cast<int>(n_tiles_n), static_cast<int>(n_tiles), static_cast<OutT *>(c), ldc,
      status, opt);
  return cudaGetLastError();
}

template <typename OutT, int VS = 16>
cudaError_t launch_o(const uint8_t *qa, const uint8_t *sfa, const float *s_a, const uint8_t *qb,
                     const uint8_t *sfb, const float *s_b, int64_t M, int64_t N, int64_t K,
                     void *c, int64_t ldc, int *status, GemmOptions opt, const Launch &L) {
  const uint8_t *const a[3] = {qa, qa, qa};
  if (N % 256 == 0)
    return launch_t<OutT, 256, 1, VS>(a, sfa, s_a, qb, sfb, s_b, M, N, K, c, ldc, status, opt, L);
  return launch_t<OutT, 128, 1, VS>(a, sfa, s_a, qb, sfb, s_b, M, N, K, c, ldc, status, opt, L);
}

}  // namespace

cudaError_t launch_gemm_if4_split(const uint8_t *q_fp, const uint8_t *q_k1, const uint8_t *q_k2,
                                  const uint8_t *sfa, const float *s_a, const uint8_t *qb,
                                  const uint8_t *sfb, const float *s_b, int64_t M, int64_t N,
                                  int64_t K, float *c, int64_t ldc, int *status,
                                  const Launch &L) {
  const uint8_t *const a[3] = {q_fp, q_k1, q_k2};
  GemmOptions opt;
  opt.alpha_int = 6.0f / 7.0f;                         // RN(6/7)
  return launch_t<float, 128, 3>(a, sfa, s_a, qb, sfb, s_b, M, N, K, c, ldc, status, opt, L);
}

cudaError_t launch_gemm_nvfp4(const uint8_t *qa, const uint8_t *sfa, const float *s_a,
                              const uint8_t *qb, const uint8_t *sfb, const float *s_b, int64_t M,
                              int64_t N, int64_t K, void *c, int c_dtype, int64_t ldc,
                              int *status, GemmOptions opt, const Launch &L) {
  if (c_dtype == FP4Q_BF16)
    return launch_o<__nv_bfloat16>(qa, sfa, s_a, qb, sfb, s_b, M, N, K, c, ldc, status, opt, L);
  return launch_o<float>(qa, sfa, s_a, qb, sfb, s_b, M, N, K, c, ldc, status, opt, L);
}

cudaError_t launch_gemm_mxfp4(const uint8_t *qa, const uint8_t *sfa, const uint8_t *qb,
                              const uint8_t *sfb, int64_t M, int64_t N, int64_t K, void *c,
                              int c_dtype, int64_t ldc, int *status, const Launch &L) {
  GemmOptions opt;
  if (c_dtype == FP4Q_BF16)
    return launch_o<__nv_bfloat16, 32>(qa, sfa, nullptr, qb, sfb, nullptr, M, N, K, c, ldc,
                                       status, opt, L);
  return launch_o<float, 32>(qa, sfa, nullptr, qb, sfb, nullptr, M, N, K, c, ldc, status, opt,
                             L);
}

}  // namespace fp4q
