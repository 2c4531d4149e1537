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
// One CTA computes a 128x128 tile of C with 4 warps:
//  - all threads stage K-tiles of 256 values (128 code bytes per row) of A
//    and B into shared memory with cp.async, in the 128-byte-swizzled
//    K-major layout, plus the 4 scale tiles (512 bytes each) of A and B;
//    four stages, loads running two K-tiles ahead of the tensor core;
//  - one thread copies the scale tiles into tensor memory (tcgen05.cp
//    32x128b.warpx4: one 512-byte tile per 64-value K step) and issues four
//    tcgen05.mma kind::mxf4nvf4 block16 (M=128, N=128, K=64), accumulating
//    in tensor memory, then tcgen05.commit to the stage's mbarrier, which
//    tells the loaders that the stage may be refilled;
//  - at the end every warp reads its 32 accumulator rows with tcgen05.ld
//    and writes C (FP32 or BF16).
// Every wait on an mbarrier is bounded (about a second of clock cycles);
// a wait that runs out sets *status and the CTA leaves the K loop, waits
// (bounded) for its tensor-core work, frees its tensor memory and returns.
#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr int BM = 128, BN = 128;
constexpr int KTILE = 256;                       // K values per stage
constexpr int KTB = KTILE / 2;                   // 128 code bytes per row per stage
constexpr int STAGES = 4;
constexpr int kThreads = 128;
constexpr int A_BYTES = BM * KTB;                // 16384
constexpr int B_BYTES = BN * KTB;                // 16384
constexpr int SF_TILE = 512;                     // 128 rows x 4 scales
constexpr int SF_BYTES = (KTILE / 64) * SF_TILE; // 2048 per operand per stage
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + 2 * SF_BYTES;   // 36864 = 36 KiB
constexpr int BAR_BYTES = 128;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 256;              // 128 accumulator + 4 x 32 scale columns
constexpr uint32_t SF_COL0 = 128;
constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at the B200's clock

static_assert(STAGE_BYTES % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");

// Instruction descriptor of tcgen05.mma kind::mxf4nvf4 (block-scaled):
// A and B E2M1 (format 1), K-major, E4M3 scales (bit 23 = 0), N = 128
// (bits 17-22 = N/8), M = 128 (bits 24-28 = M/16), dense, K = 64.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                            (uint32_t(BM >> 4) << 24);

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
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], "
      "[%6], p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// 32 consecutive FP32 accumulator columns of this thread's row (warp w reads
// lanes 32w .. 32w + 31)
__device__ __forceinline__ void tc_load32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Stage K-tile kt of this CTA's A rows, B rows and their scale tiles.
__device__ __forceinline__ void load_stage(uint32_t st, const uint8_t *qa, const uint8_t *qb,
                                           const uint8_t *sfa, const uint8_t *sfb, int64_t ldk,
                                           int kt) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int j = 0; j < 8; ++j) {                  // 1024 16-byte pieces per operand
    const int i = tid + kThreads * j;
    const int r = i >> 3, c = i & 7;
    const uint32_t so = static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
    const int64_t go = r * ldk + static_cast<int64_t>(kt) * KTB + c * 16;
    cp_async16(st + so, qa + go);
    cp_async16(st + A_BYTES + so, qb + go);
  }
  // the four 512-byte scale tiles of this K-tile are contiguous
  cp_async16(st + A_BYTES + B_BYTES + tid * 16, sfa + static_cast<int64_t>(kt) * SF_BYTES + tid * 16);
  cp_async16(st + A_BYTES + B_BYTES + SF_BYTES + tid * 16,
             sfb + static_cast<int64_t>(kt) * SF_BYTES + tid * 16);
}

template <typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
gemm_nvfp4_kernel(const uint8_t *__restrict__ qa, const uint8_t *__restrict__ sfa,
                  const float *__restrict__ s_a, const uint8_t *__restrict__ qb,
                  const uint8_t *__restrict__ sfb, const float *__restrict__ s_b, int K,
                  OutT *__restrict__ c, int64_t ldc, int *__restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t bars = base + STAGES * STAGE_BYTES;   // STAGES empty barriers, then done
  const uint32_t done_bar = bars + 8 * STAGES;
  const uint32_t tmem_slot = done_bar + 8;
  uint8_t *const slot_ptr = smem_raw + (tmem_slot - raw);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  const int64_t ldk = K / 2;                           // code bytes per row
  const int KT = K / KTILE;
  const int64_t sf_per_rowtile = static_cast<int64_t>(K / 64) * SF_TILE;
  const uint8_t *a_rows = qa + m0 * ldk, *b_rows = qb + n0 * ldk;
  const uint8_t *a_sf = sfa + (m0 / BM) * sf_per_rowtile, *b_sf = sfb + (n0 / BN) * sf_per_rowtile;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     tmem_slot),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(bars + 8 * s, 1);
    mbar_init(done_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(slot_ptr);

  // prologue: K-tiles 0 .. STAGES-3
#pragma unroll
  for (int t = 0; t < STAGES - 2; ++t) {
    if (t < KT) load_stage(base + t * STAGE_BYTES, a_rows, b_rows, a_sf, b_sf, ldk, t);
    cp_async_commit();
  }
  int err = 0;
  for (int kt = 0; kt < KT; ++kt) {
    const int t = kt + STAGES - 2;                     // the K-tile loaded now
    if (t < KT) {
      const int s = t % STAGES;
      // its stage last held K-tile kt - 2: wait until the MMAs reading it are done
      if (kt >= 2 && !mbar_wait(bars + 8 * s, static_cast<uint32_t>(((kt - 2) / STAGES) & 1)))
        err = 1;
      if (!err) load_stage(base + s * STAGE_BYTES, a_rows, b_rows, a_sf, b_sf, ldk, t);
    }
    cp_async_commit();
    cp_async_wait<STAGES - 2>();                        // K-tile kt has landed
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (__syncthreads_or(err)) {
      err = 1;
      break;
    }
    if (tid == 0) {
      tc_fence_after();
      const int s = kt % STAGES;
      const uint32_t st = base + s * STAGE_BYTES;
      const uint32_t sfa_col = tmem + SF_COL0 + 32u * s, sfb_col = sfa_col + 16u;
#pragma unroll
      for (int kb = 0; kb < KTILE / 64; ++kb) {
        tc_copy_sf(sfa_col + 4u * kb, desc_sf(st + A_BYTES + B_BYTES + kb * SF_TILE));
        tc_copy_sf(sfb_col + 4u * kb, desc_sf(st + A_BYTES + B_BYTES + SF_BYTES + kb * SF_TILE));
      }
      const uint64_t da = desc_sw128(st), db = desc_sw128(st + A_BYTES);
#pragma unroll
      for (int kb = 0; kb < KTILE / 64; ++kb)          // 64 values = 32 bytes = 2 descriptor units
        tc_mma(tmem, da + 2u * kb, db + 2u * kb, sfa_col + 4u * kb, sfb_col + 4u * kb,
               (kt | kb) != 0);
      tc_commit(bars + 8 * s);
    }
  }
  cp_async_wait<0>();
  if (tid == 0) tc_commit(done_bar);                    // all MMAs issued so far
  const int late = mbar_wait(done_bar, 0) ? 0 : 1;
  err = __syncthreads_or(err | late);
  tc_fence_after();
  if (!err && KT > 0) {
    const float alpha = __fmul_rn(s_a ? *s_a : 1.0f, s_b ? *s_b : 1.0f);
    OutT *row = c + (m0 + warp * 32 + lane) * ldc + n0;
#pragma unroll 1
    for (int j = 0; j < BN / 32; ++j) {
      uint32_t r[32];
      tc_load32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + 32u * j, r);
      if (sizeof(OutT) == 4) {
        float4 *d = reinterpret_cast<float4 *>(row + 32 * j);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          d[q] = make_float4(__fmul_rn(__uint_as_float(r[4 * q]), alpha),
                             __fmul_rn(__uint_as_float(r[4 * q + 1]), alpha),
                             __fmul_rn(__uint_as_float(r[4 * q + 2]), alpha),
                             __fmul_rn(__uint_as_float(r[4 * q + 3]), alpha));
      } else {
        uint4 *d = reinterpret_cast<uint4 *>(row + 32 * j);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(
                __fmul_rn(__uint_as_float(r[8 * q + 2 * h]), alpha),
                __fmul_rn(__uint_as_float(r[8 * q + 2 * h + 1]), alpha));
            memcpy(&w[h], &b2, sizeof(uint32_t));
          }
          d[q] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }
  if (err && tid == 0 && status) atomicExch(status, 1);
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(TMEM_COLS)
                 : "memory");
}

template <typename OutT>
cudaError_t launch_t(const uint8_t *qa, const uint8_t *sfa, const float *s_a, const uint8_t *qb,
                     const uint8_t *sfb, const float *s_b, int64_t M, int64_t N, int64_t K,
                     void *c, int64_t ldc, int *status, const Launch &L) {
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(
        gemm_nvfp4_kernel<OutT>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const dim3 grid(static_cast<unsigned>(N / BN), static_cast<unsigned>(M / BM));
  gemm_nvfp4_kernel<OutT><<<grid, kThreads, SMEM_BYTES, L.stream>>>(
      qa, sfa, s_a, qb, sfb, s_b, static_cast<int>(K), static_cast<OutT *>(c), ldc, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_nvfp4(const uint8_t *qa, const uint8_t *sfa, const float *s_a,
                              const uint8_t *qb, const uint8_t *sfb, const float *s_b, int64_t M,
                              int64_t N, int64_t K, void *c, int c_dtype, int64_t ldc,
                              int *status, const Launch &L) {
  if (c_dtype == FP4Q_BF16)
    return launch_t<__nv_bfloat16>(qa, sfa, s_a, qb, sfb, s_b, M, N, K, c, ldc, status, L);
  return launch_t<float>(qa, sfa, s_a, qb, sfb, s_b, M, N, K, c, ldc, status, L);
}

}  // namespace fp4q
