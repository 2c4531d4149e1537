// api.cu -- the extern "C" entry points declared in include/fp4q.h.
//
// Each entry point checks its arguments on the host (returning a status and
// enqueueing nothing on error), makes the device that owns the input current,
// and enqueues its kernels on the caller's stream.
#include <cstdint>
#include <cstring>
#include <initializer_list>

#include "common.cuh"
#include "launch.h"

namespace fp4q {
namespace {

constexpr size_t kWorkspaceBytes = 256;  // one float amax, padded

int g_num_sms[64];

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_size(int dtype) { return dtype == FP4Q_BF16 ? 2 : 4; }

bool valid_dtype(int d) { return d == FP4Q_BF16 || d == FP4Q_FP32; }
bool valid_layout(int l) { return l == FP4Q_SCALE_LINEAR || l == FP4Q_SCALE_SWIZZLED_128x4; }

// The device owning `p` becomes current; host memory is rejected.
fp4q_status bind_device(const void *p, void *stream, Launch *L) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return FP4Q_ERR_INVALID_ARG;
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return FP4Q_ERR_INVALID_ARG;
  int dev = attr.device;
  if (dev < 0 || dev >= 64) return FP4Q_ERR_INVALID_ARG;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != dev)
    if (cudaSetDevice(dev) != cudaSuccess) return FP4Q_ERR_CUDA;
  if (g_num_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FP4Q_ERR_CUDA;
    g_num_sms[dev] = n;
  }
  L->stream = static_cast<cudaStream_t>(stream);
  L->num_sms = g_num_sms[dev];
  cudaGetLastError();  // start from a clean error state of this runtime
  return FP4Q_OK;
}

// Bind to the first non-NULL pointer of the call (an empty tensor may have a
// NULL data pointer).  *nothing is set when every pointer is NULL.
fp4q_status bind_first(std::initializer_list<const void *> ptrs, void *stream, Launch *L,
                       bool *nothing) {
  *nothing = false;
  for (const void *p : ptrs)
    if (p != nullptr) return bind_device(p, stream, L);
  *nothing = true;
  return FP4Q_OK;
}

// A pointer that must live on the device (NULL allowed when optional).
fp4q_status check_dev(const void *p, bool optional) {
  if (p == nullptr) return optional ? FP4Q_OK : FP4Q_ERR_INVALID_ARG;
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return FP4Q_ERR_INVALID_ARG;
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return FP4Q_ERR_INVALID_ARG;
  return FP4Q_OK;
}

fp4q_status check_matrix(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld) {
  if (!valid_dtype(dtype)) return FP4Q_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0 || ld < cols) return FP4Q_ERR_INVALID_ARG;
  if (x == nullptr) return (rows == 0 || cols == 0) ? FP4Q_OK : FP4Q_ERR_INVALID_ARG;
  if (!aligned16(x) || (ld * elem_size(dtype)) % 16 != 0) return FP4Q_ERR_MISALIGNED;
  return FP4Q_OK;
}

fp4q_status check_swizzle(int layout, int64_t srows, int64_t scols) {
  if (layout == FP4Q_SCALE_SWIZZLED_128x4 && (srows % 128 != 0 || scols % 4 != 0))
    return FP4Q_ERR_UNSUPPORTED_SHAPE;
  return FP4Q_OK;
}

fp4q_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FP4Q_OK : FP4Q_ERR_CUDA; }

template <int QMAX = 6>
__global__ void write_s_dec_kernel(const float *amax, float *out) {
  if (threadIdx.x == 0) *out = tensor_scale_q<QMAX>(*amax).dec;
}

// s_dec = RN(amax / top) for a grid whose largest magnitude times 448 is top
// (1 when amax is 0)
__global__ void write_s_dec_top_kernel(const float *amax, float top, float *out) {
  if (threadIdx.x == 0) *out = *amax == 0.0f ? 1.0f : __fdiv_rn(*amax, top);
}

// Resolve the tensor amax: the caller's pointer, or one computed into the
// workspace by a pre-pass.
fp4q_status resolve_amax(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                         const float *amax, void *ws, size_t ws_bytes, const Launch &L,
                         const float **out) {
  if (amax != nullptr) {
    *out = amax;
    return FP4Q_OK;
  }
  if (ws == nullptr || ws_bytes < kWorkspaceBytes) return FP4Q_ERR_WORKSPACE_TOO_SMALL;
  if ((reinterpret_cast<uintptr_t>(ws) & 3u) != 0) return FP4Q_ERR_MISALIGNED;
  float *a = static_cast<float *>(ws);
  fp4q_status s = cuda_status(launch_amax(x, dtype, rows, cols, ld, a, L));
  *out = a;
  return s;
}

#define FP4Q_TRY(expr)                     \
  do {                                     \
    fp4q_status s_ = (expr);               \
    if (s_ != FP4Q_OK) return s_;          \
  } while (0)

}  // namespace
}  // namespace fp4q

using namespace fp4q;

namespace fp4q {
namespace {

fp4q_status quantize_if4_mode(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                              const float *amax, float *tensor_scale_out, uint8_t *q,
                              uint8_t *sf, int scale_layout, void *workspace, size_t ws_bytes,
                              void *stream, int int4_mode) {
  FP4Q_TRY(check_matrix(x, dtype, rows, cols, ld));
  if (!valid_layout(scale_layout)) return FP4Q_ERR_INVALID_ARG;
  if (cols % 16 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if ((!q || !sf) && rows > 0 && cols > 0) return FP4Q_ERR_INVALID_ARG;
  if (!aligned16(q)) return FP4Q_ERR_MISALIGNED;
  FP4Q_TRY(check_swizzle(scale_layout, rows, cols / 16));
  Launch L;
  bool none = false;
  FP4Q_TRY(bind_first({x, tensor_scale_out, amax}, stream, &L, &none));
  if (none) return FP4Q_OK;
  if (rows > 0 && cols > 0) {
    FP4Q_TRY(check_dev(q, false));
    FP4Q_TRY(check_dev(sf, false));
  }
  FP4Q_TRY(check_dev(amax, true));
  FP4Q_TRY(check_dev(tensor_scale_out, true));
  const float *a = nullptr;
  FP4Q_TRY(resolve_amax(x, dtype, rows, cols, ld, amax, workspace, ws_bytes, L, &a));
  if (rows == 0 || cols == 0) {
    if (tensor_scale_out) write_s_dec_kernel<<<1, 1, 0, L.stream>>>(a, tensor_scale_out);
    return cuda_status(cudaGetLastError());
  }
  return cuda_status(
      launch_if4(x, dtype, rows, cols, ld, a, tensor_scale_out, q, sf, scale_layout, int4_mode,
                 L));
}

}  // namespace

int check_nvfp4_args(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                     unsigned layouts, int round, const uint8_t *q_row, const uint8_t *sf_row,
                     const uint8_t *q_col, const uint8_t *sf_col, int scale_layout) {
  FP4Q_TRY(check_matrix(x, dtype, rows, cols, ld));
  if (layouts == 0 || (layouts & ~(FP4Q_ROWWISE | FP4Q_COLWISE)) != 0) return FP4Q_ERR_INVALID_ARG;
  if (round != FP4Q_RNE && round != FP4Q_SR) return FP4Q_ERR_INVALID_ARG;
  if (!valid_layout(scale_layout)) return FP4Q_ERR_INVALID_ARG;
  if (cols % 16 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if ((layouts & FP4Q_COLWISE) && rows % 16 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  const bool nonempty = rows > 0 && cols > 0;
  if (layouts & FP4Q_ROWWISE) {
    if ((!q_row || !sf_row) && nonempty) return FP4Q_ERR_INVALID_ARG;
    if (!aligned16(q_row)) return FP4Q_ERR_MISALIGNED;
    FP4Q_TRY(check_swizzle(scale_layout, rows, cols / 16));
  }
  if (layouts & FP4Q_COLWISE) {
    if ((!q_col || !sf_col) && nonempty) return FP4Q_ERR_INVALID_ARG;
    if (!aligned16(q_col)) return FP4Q_ERR_MISALIGNED;
    FP4Q_TRY(check_swizzle(scale_layout, cols, rows / 16));
  }
  return FP4Q_OK;
}

}  // namespace fp4q

extern "C" {

const char *fp4q_status_string(int status) {
  switch (status) {
    case FP4Q_OK: return "FP4Q_OK";
    case FP4Q_ERR_INVALID_ARG: return "FP4Q_ERR_INVALID_ARG";
    case FP4Q_ERR_UNSUPPORTED_SHAPE: return "FP4Q_ERR_UNSUPPORTED_SHAPE";
    case FP4Q_ERR_MISALIGNED: return "FP4Q_ERR_MISALIGNED";
    case FP4Q_ERR_WORKSPACE_TOO_SMALL: return "FP4Q_ERR_WORKSPACE_TOO_SMALL";
    case FP4Q_ERR_CUDA: return "FP4Q_ERR_CUDA";
    default: return "FP4Q_ERR_UNKNOWN";
  }
}

const char *fp4q_version(void) { return "fp4q 0.1 (sm_100a)"; }

size_t fp4q_workspace_bytes(int64_t rows, int64_t cols) {
  return (rows < 0 || cols < 0) ? 0 : kWorkspaceBytes;
}

size_t fp4q_scale_bytes(int64_t rows, int64_t cols, int block, int scale_layout) {
  if (rows < 0 || cols < 0 || block <= 0 || cols % block != 0 || !valid_layout(scale_layout))
    return 0;
  int64_t sc = cols / block;
  if (scale_layout == FP4Q_SCALE_LINEAR) return static_cast<size_t>(rows * sc);
  return static_cast<size_t>(((rows + 127) / 128 * 128) * ((sc + 3) / 4 * 4));
}

fp4q_status fp4q_amax(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                      float *amax_out, void *stream) {
  DeviceGuard guard;
  FP4Q_TRY(check_matrix(x, dtype, rows, cols, ld));
  if (cols % 16 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  Launch L;
  bool none = false;
  FP4Q_TRY(bind_first({x, amax_out}, stream, &L, &none));
  FP4Q_TRY(check_dev(amax_out, false));
  if (rows == 0 || cols == 0)
    return cuda_status(cudaMemsetAsync(amax_out, 0, sizeof(float), L.stream));
  return cuda_status(launch_amax(x, dtype, rows, cols, ld, amax_out, L));
}

fp4q_status fp4q_quantize_nvfp4(const void *x, int dtype, int64_t rows, int64_t cols,
                                int64_t ld, unsigned layouts, int round, uint64_t seed,
                                const float *amax, float *tensor_scale_out, uint8_t *q_row,
                                uint8_t *sf_row, uint8_t *q_col, uint8_t *sf_col,
                                int scale_layout, void *workspace, size_t ws_bytes,
                                void *stream) {
  DeviceGuard guard;
  FP4Q_TRY(static_cast<fp4q_status>(check_nvfp4_args(x, dtype, rows, cols, ld, layouts, round,
                                                     q_row, sf_row, q_col, sf_col,
                                                     scale_layout)));
  Launch L;
  bool none = false;
  FP4Q_TRY(bind_first({x, tensor_scale_out, amax}, stream, &L, &none));
  if (none) return FP4Q_OK;
  FP4Q_TRY(check_dev(amax, true));
  FP4Q_TRY(check_dev(tensor_scale_out, true));
  FP4Q_TRY(check_dev((layouts & FP4Q_ROWWISE) ? q_row : nullptr, true));
  FP4Q_TRY(check_dev((layouts & FP4Q_COLWISE) ? q_col : nullptr, true));
  const float *a = nullptr;
  FP4Q_TRY(resolve_amax(x, dtype, rows, cols, ld, amax, workspace, ws_bytes, L, &a));
  if (rows == 0 || cols == 0) {
    if (tensor_scale_out) write_s_dec_kernel<<<1, 1, 0, L.stream>>>(a, tensor_scale_out);
    return cuda_status(cudaGetLastError());
  }
  return cuda_status(launch_nvfp4(x, dtype, rows, cols, ld, layouts, round, seed, a,
                                  tensor_scale_out, q_row, sf_row, q_col, sf_col, scale_layout,
                                  L));
}

fp4q_status fp4q_quantize_mxfp4(const void *x, int dtype, int64_t rows, int64_t cols,
                                int64_t ld, unsigned layouts, int e8m0_mode, uint8_t *q_row,
                                uint8_t *sf_row, uint8_t *q_col, uint8_t *sf_col,
                                int scale_layout, void *stream) {
  DeviceGuard guard;
  FP4Q_TRY(check_matrix(x, dtype, rows, cols, ld));
  if (layouts == 0 || (layouts & ~(FP4Q_ROWWISE | FP4Q_COLWISE)) != 0) return FP4Q_ERR_INVALID_ARG;
  if (e8m0_mode < FP4Q_E8M0_RNE || e8m0_mode > FP4Q_E8M0_OCP_FLOOR) return FP4Q_ERR_INVALID_ARG;
  if (!valid_layout(scale_layout)) return FP4Q_ERR_INVALID_ARG;
  if (cols % 32 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if ((layouts & FP4Q_COLWISE) && rows % 32 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if (layouts & FP4Q_ROWWISE) {
    if (!q_row || !sf_row) return FP4Q_ERR_INVALID_ARG;
    if (!aligned16(q_row)) return FP4Q_ERR_MISALIGNED;
    FP4Q_TRY(check_swizzle(scale_layout, rows, cols / 32));
  }
  if (layouts & FP4Q_COLWISE) {
    if (!q_col || !sf_col) return FP4Q_ERR_INVALID_ARG;
    if (!aligned16(q_col)) return FP4Q_ERR_MISALIGNED;
    FP4Q_TRY(check_swizzle(scale_layout, cols, rows / 32));
  }
  if (rows == 0 || cols == 0) return FP4Q_OK;
  Launch L;
  FP4Q_TRY(bind_device(x, stream, &L));
  FP4Q_TRY(check_dev((layouts & FP4Q_ROWWISE) ? q_row : nullptr, true));
  FP4Q_TRY(check_dev((layouts & FP4Q_COLWISE) ? q_col : nullptr, true));
  return cuda_status(launch_mxfp4(x, dtype, rows, cols, ld, layouts, e8m0_mode, q_row, sf_row,
                                  q_col, sf_col, scale_layout, L));
}

fp4q_status fp4q_quantize_2d(const void *w, int dtype, int64_t rows, int64_t cols, int64_t ld,
                             const float *amax, float *tensor_scale_out, uint8_t *q_w,
                             uint8_t *q_wt, uint8_t *sf_tiles, uint8_t *sf_w_1x16,
                             uint8_t *sf_wt_1x16, int scale_layout, void *workspace,
                             size_t ws_bytes, void *stream) {
  DeviceGuard guard;
  FP4Q_TRY(check_matrix(w, dtype, rows, cols, ld));
  if (!valid_layout(scale_layout)) return FP4Q_ERR_INVALID_ARG;
  if (rows % 16 != 0 || cols % 16 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if (!sf_tiles && rows > 0 && cols > 0) return FP4Q_ERR_INVALID_ARG;
  if ((q_w && !aligned16(q_w)) || (q_wt && !aligned16(q_wt))) return FP4Q_ERR_MISALIGNED;
  if (sf_w_1x16) FP4Q_TRY(check_swizzle(scale_layout, rows, cols / 16));
  if (sf_wt_1x16) FP4Q_TRY(check_swizzle(scale_layout, cols, rows / 16));
  Launch L;
  bool none = false;
  FP4Q_TRY(bind_first({w, tensor_scale_out, amax}, stream, &L, &none));
  if (none) return FP4Q_OK;
  if (rows > 0 && cols > 0) FP4Q_TRY(check_dev(sf_tiles, false));
  FP4Q_TRY(check_dev(q_w, true));
  FP4Q_TRY(check_dev(q_wt, true));
  FP4Q_TRY(check_dev(amax, true));
  FP4Q_TRY(check_dev(tensor_scale_out, true));
  const float *a = nullptr;
  FP4Q_TRY(resolve_amax(w, dtype, rows, cols, ld, amax, workspace, ws_bytes, L, &a));
  if (rows == 0 || cols == 0) {
    if (tensor_scale_out) write_s_dec_kernel<<<1, 1, 0, L.stream>>>(a, tensor_scale_out);
    return cuda_status(cudaGetLastError());
  }
  return cuda_status(launch_2d(w, dtype, rows, cols, ld, a, tensor_scale_out, q_w, q_wt,
                               sf_tiles, sf_w_1x16, sf_wt_1x16, scale_layout, L));
}

fp4q_status fp4q_rht_amax(const void *dy, int dtype, int64_t tokens, int64_t cols, int64_t ld,
                          int hadamard_n, uint64_t seed, float *amax_out, void *stream) {
  DeviceGuard guard;
  FP4Q_TRY(check_matrix(dy, dtype, tokens, cols, ld));
  if (hadamard_n != 16 && hadamard_n != 128) return FP4Q_ERR_INVALID_ARG;
  if (tokens % hadamard_n != 0 || cols % 8 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  Launch L;
  bool none = false;
  FP4Q_TRY(bind_first({dy, amax_out}, stream, &L, &none));
  FP4Q_TRY(check_dev(amax_out, false));
  if (tokens == 0 || cols == 0)
    return cuda_status(cudaMemsetAsync(amax_out, 0, sizeof(float), L.stream));
  return cuda_status(launch_rht_amax(dy, dtype, tokens, cols, ld, hadamard_n, seed, amax_out, L));
}

fp4q_status fp4q_quantize_rht_sr(const void *dy, int dtype, int64_t tokens, int64_t cols,
                                 int64_t ld, int hadamard_n, int round, uint64_t seed,
                                 const float *amax_rht, float *tensor_scale_out, uint8_t *q_t,
                                 uint8_t *sf_t, int scale_layout, float *rht_debug_out,
                                 void *workspace, size_t ws_bytes, void *stream) {
  DeviceGuard guard;
  FP4Q_TRY(check_matrix(dy, dtype, tokens, cols, ld));
  if (hadamard_n != 16 && hadamard_n != 128) return FP4Q_ERR_INVALID_ARG;
  if (round != FP4Q_RNE && round != FP4Q_SR) return FP4Q_ERR_INVALID_ARG;
  if (!valid_layout(scale_layout)) return FP4Q_ERR_INVALID_ARG;
  if (tokens % hadamard_n != 0 || cols % 8 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if ((!q_t || !sf_t) && tokens > 0 && cols > 0) return FP4Q_ERR_INVALID_ARG;
  if (!aligned16(q_t) || (rht_debug_out && !aligned16(rht_debug_out))) return FP4Q_ERR_MISALIGNED;
  FP4Q_TRY(check_swizzle(scale_layout, cols, tokens / 16));
  Launch L;
  bool none = false;
  FP4Q_TRY(bind_first({dy, tensor_scale_out, amax_rht}, stream, &L, &none));
  if (none) return FP4Q_OK;
  if (tokens > 0 && cols > 0) {
    FP4Q_TRY(check_dev(q_t, false));
    FP4Q_TRY(check_dev(sf_t, false));
  }
  FP4Q_TRY(check_dev(amax_rht, true));
  FP4Q_TRY(check_dev(tensor_scale_out, true));
  FP4Q_TRY(check_dev(rht_debug_out, true));
  const float *a = amax_rht;
  if (a == nullptr) {
    if (workspace == nullptr || ws_bytes < kWorkspaceBytes) return FP4Q_ERR_WORKSPACE_TOO_SMALL;
    if ((reinterpret_cast<uintptr_t>(workspace) & 3u) != 0) return FP4Q_ERR_MISALIGNED;
    float *w = static_cast<float *>(workspace);
    if (tokens == 0 || cols == 0) {
      FP4Q_TRY(cuda_status(cudaMemsetAsync(w, 0, sizeof(float), L.stream)));
    } else {
      FP4Q_TRY(cuda_status(launch_rht_amax(dy, dtype, tokens, cols, ld, hadamard_n, seed, w, L)));
    }
    a = w;
  }
  if (tokens == 0 || cols == 0) {
    if (tensor_scale_out) write_s_dec_kernel<<<1, 1, 0, L.stream>>>(a, tensor_scale_out);
    return cuda_status(cudaGetLastError());
  }
  return cuda_status(launch_rht_quant(dy, dtype, tokens, cols, ld, hadamard_n, round, seed, a,
                                      tensor_scale_out, q_t, sf_t, scale_layout, rht_debug_out,
                                      L));
}

fp4q_status fp4q_quantize_backward(const void *dy, int dtype, int64_t tokens, int64_t cols,
                                   int64_t ld, int hadamard_n, int round, uint64_t seed_row,
                                   uint64_t seed_col, const float *amax_row,
                                   const float *amax_rht, float *s_dec_row_out,
                                   float *s_dec_col_out, uint8_t *q_row, uint8_t *sf_row,
                                   uint8_t *q_t, uint8_t *sf_t, int scale_layout, void *workspace,
                                   size_t ws_bytes, void *stream) {
  DeviceGuard guard;
  FP4Q_TRY(check_matrix(dy, dtype, tokens, cols, ld));
  if (hadamard_n != 16 && hadamard_n != 128) return FP4Q_ERR_INVALID_ARG;
  if (round != FP4Q_RNE && round != FP4Q_SR) return FP4Q_ERR_INVALID_ARG;
  if (!valid_layout(scale_layout)) return FP4Q_ERR_INVALID_ARG;
  if (tokens % hadamard_n != 0 || cols % 16 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  const bool nonempty = tokens > 0 && cols > 0;
  if ((!q_row || !sf_row || !q_t || !sf_t) && nonempty) return FP4Q_ERR_INVALID_ARG;
  if (!aligned16(q_row) || !aligned16(q_t)) return FP4Q_ERR_MISALIGNED;
  FP4Q_TRY(check_swizzle(scale_layout, tokens, cols / 16));
  FP4Q_TRY(check_swizzle(scale_layout, cols, tokens / 16));
  Launch L;
  bool none = false;
  FP4Q_TRY(bind_first({dy, s_dec_row_out, s_dec_col_out, amax_row, amax_rht}, stream, &L, &none));
  if (none) return FP4Q_OK;
  if (nonempty) {
    FP4Q_TRY(check_dev(q_row, false));
    FP4Q_TRY(check_dev(sf_row, false));
    FP4Q_TRY(check_dev(q_t, false));
    FP4Q_TRY(check_dev(sf_t, false));
  }
  FP4Q_TRY(check_dev(amax_row, true));
  FP4Q_TRY(check_dev(amax_rht, true));
  FP4Q_TRY(check_dev(s_dec_row_out, true));
  FP4Q_TRY(check_dev(s_dec_col_out, true));
  // missing amaxes are computed into the workspace: the row amax at byte 0,
  // the amax of the transform at byte 128
  const float *ar = amax_row, *ac = amax_rht;
  if (ar == nullptr || ac == nullptr) {
    if (workspace == nullptr || ws_bytes < kWorkspaceBytes) return FP4Q_ERR_WORKSPACE_TOO_SMALL;
    if ((reinterpret_cast<uintptr_t>(workspace) & 3u) != 0) return FP4Q_ERR_MISALIGNED;
  }
  if (ar == nullptr) {
    float *w = static_cast<float *>(workspace);
    if (nonempty)
      FP4Q_TRY(cuda_status(launch_amax(dy, dtype, tokens, cols, ld, w, L)));
    else
      FP4Q_TRY(cuda_status(cudaMemsetAsync(w, 0, sizeof(float), L.stream)));
    ar = w;
  }
  if (ac == nullptr) {
    float *w = static_cast<float *>(workspace) + 32;
    if (nonempty)
      FP4Q_TRY(cuda_status(launch_rht_amax(dy, dtype, tokens, cols, ld, hadamard_n, seed_col, w, L)));
    else
      FP4Q_TRY(cuda_status(cudaMemsetAsync(w, 0, sizeof(float), L.stream)));
    ac = w;
  }
  if (!nonempty) {
    if (s_dec_row_out) write_s_dec_kernel<<<1, 1, 0, L.stream>>>(ar, s_dec_row_out);
    if (s_dec_col_out) write_s_dec_kernel<<<1, 1, 0, L.stream>>>(ac, s_dec_col_out);
    return cuda_status(cudaGetLastError());
  }
  return cuda_status(launch_rht_backward(dy, dtype, tokens, cols, ld, hadamard_n, round, seed_row,
                                         seed_col, ar, ac, s_dec_row_out, s_dec_col_out, q_row,
                                         sf_row, q_t, sf_t, scale_layout, L));
}

fp4q_status fp4q_quantize_if4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                              const float *amax, float *tensor_scale_out, uint8_t *q,
                              uint8_t *sf, int scale_layout, void *workspace, size_t ws_bytes,
                              void *stream) {
  DeviceGuard guard;
  return quantize_if4_mode(x, dtype, rows, cols, ld, amax, tensor_scale_out, q, sf, scale_layout,
                           workspace, ws_bytes, stream, 1);
}

fp4q_status fp4q_quantize_nvint4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                                 const float *amax, float *tensor_scale_out, uint8_t *q,
                                 uint8_t *sf, int scale_layout, void *workspace,
                                 size_t ws_bytes, void *stream) {
  DeviceGuard guard;
  return quantize_if4_mode(x, dtype, rows, cols, ld, amax, tensor_scale_out, q, sf, scale_layout,
                           workspace, ws_bytes, stream, 2);
}

fp4q_status fp4q_quantize_four_over_six(const void *x, int dtype, int64_t rows, int64_t cols,
                                        int64_t ld, unsigned layouts, const float *amax,
                                        float *tensor_scale_out, uint8_t *q_row, uint8_t *sf_row,
                                        uint8_t *q_col, uint8_t *sf_col, int scale_layout,
                                        void *workspace, size_t ws_bytes, void *stream) {
  DeviceGuard guard;
  FP4Q_TRY(check_matrix(x, dtype, rows, cols, ld));
  if (layouts == 0 || (layouts & ~(FP4Q_ROWWISE | FP4Q_COLWISE)) != 0) return FP4Q_ERR_INVALID_ARG;
  if (!valid_layout(scale_layout)) return FP4Q_ERR_INVALID_ARG;
  if (cols % 16 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if ((layouts & FP4Q_COLWISE) && rows % 16 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  const bool nonempty = rows > 0 && cols > 0;
  if (layouts & FP4Q_ROWWISE) {
    if ((!q_row || !sf_row) && nonempty) return FP4Q_ERR_INVALID_ARG;
    if (!aligned16(q_row)) return FP4Q_ERR_MISALIGNED;
    FP4Q_TRY(check_swizzle(scale_layout, rows, cols / 16));
  }
  if (layouts & FP4Q_COLWISE) {
    if ((!q_col || !sf_col) && nonempty) return FP4Q_ERR_INVALID_ARG;
    if (!aligned16(q_col)) return FP4Q_ERR_MISALIGNED;
    FP4Q_TRY(check_swizzle(scale_layout, cols, rows / 16));
  }
  Launch L;
  bool none = false;
  FP4Q_TRY(bind_first({x, tensor_scale_out, amax}, stream, &L, &none));
  if (none) return FP4Q_OK;
  FP4Q_TRY(check_dev(amax, true));
  FP4Q_TRY(check_dev(tensor_scale_out, true));
  FP4Q_TRY(check_dev((layouts & FP4Q_ROWWISE) ? q_row : nullptr, true));
  FP4Q_TRY(check_dev((layouts & FP4Q_COLWISE) ? q_col : nullptr, true));
  const float *a = nullptr;
  FP4Q_TRY(resolve_amax(x, dtype, rows, cols, ld, amax, workspace, ws_bytes, L, &a));
  if (!nonempty) {
    if (tensor_scale_out) write_s_dec_kernel<4><<<1, 1, 0, L.stream>>>(a, tensor_scale_out);
    return cuda_status(cudaGetLastError());
  }
  return cuda_status(launch_four_over_six(x, dtype, rows, cols, ld, layouts, a, tensor_scale_out,
                                          q_row, sf_row, q_col, sf_col, scale_layout, L));
}

fp4q_status fp4q_quantize_if6(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                              const float *amax, float *tensor_scale_out, uint8_t *q, uint8_t *sf,
                              int scale_layout, void *workspace, size_t ws_bytes, void *stream) {
  DeviceGuard guard;
  FP4Q_TRY(check_matrix(x, dtype, rows, cols, ld));
  if (!valid_layout(scale_layout)) return FP4Q_ERR_INVALID_ARG;
  if (cols % 16 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if ((!q || !sf) && rows > 0 && cols > 0) return FP4Q_ERR_INVALID_ARG;
  if (!aligned16(q)) return FP4Q_ERR_MISALIGNED;
  FP4Q_TRY(check_swizzle(scale_layout, rows, cols / 16));
  Launch L;
  bool none = false;
  FP4Q_TRY(bind_first({x, tensor_scale_out, amax}, stream, &L, &none));
  if (none) return FP4Q_OK;
  if (rows > 0 && cols > 0) {
    FP4Q_TRY(check_dev(q, false));
    FP4Q_TRY(check_dev(sf, false));
  }
  FP4Q_TRY(check_dev(amax, true));
  FP4Q_TRY(check_dev(tensor_scale_out, true));
  const float *a = nullptr;
  FP4Q_TRY(resolve_amax(x, dtype, rows, cols, ld, amax, workspace, ws_bytes, L, &a));
  if (rows == 0 || cols == 0) {
    if (tensor_scale_out) write_s_dec_top_kernel<<<1, 1, 0, L.stream>>>(a, 3360.0f, tensor_scale_out);
    return cuda_status(cudaGetLastError());
  }
  return cuda_status(
      launch_if6(x, dtype, rows, cols, ld, a, tensor_scale_out, q, sf, scale_layout, L));
}

fp4q_status fp4q_quantize_if3(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                              const float *amax, float *tensor_scale_out, uint8_t *q, uint8_t *sf,
                              int scale_layout, void *workspace, size_t ws_bytes, void *stream) {
  DeviceGuard guard;
  FP4Q_TRY(check_matrix(x, dtype, rows, cols, ld));
  if (!valid_layout(scale_layout)) return FP4Q_ERR_INVALID_ARG;
  if (cols % 16 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if ((!q || !sf) && rows > 0 && cols > 0) return FP4Q_ERR_INVALID_ARG;
  if (!aligned16(q)) return FP4Q_ERR_MISALIGNED;
  FP4Q_TRY(check_swizzle(scale_layout, rows, cols / 16));
  Launch L;
  bool none = false;
  FP4Q_TRY(bind_first({x, tensor_scale_out, amax}, stream, &L, &none));
  if (none) return FP4Q_OK;
  if (rows > 0 && cols > 0) {
    FP4Q_TRY(check_dev(q, false));
    FP4Q_TRY(check_dev(sf, false));
  }
  FP4Q_TRY(check_dev(amax, true));
  FP4Q_TRY(check_dev(tensor_scale_out, true));
  const float *a = nullptr;
  FP4Q_TRY(resolve_amax(x, dtype, rows, cols, ld, amax, workspace, ws_bytes, L, &a));
  if (rows == 0 || cols == 0) {
    if (tensor_scale_out) write_s_dec_top_kernel<<<1, 1, 0, L.stream>>>(a, 1792.0f, tensor_scale_out);
    return cuda_status(cudaGetLastError());
  }
  return cuda_status(
      launch_if3(x, dtype, rows, cols, ld, a, tensor_scale_out, q, sf, scale_layout, L));
}

fp4q_status fp4q_quantize_mxfp6(const void *x, int dtype, int64_t rows, int64_t cols,
                                int64_t ld, int fp6_format, int e8m0_mode, uint8_t *q,
                                uint8_t *sf, int scale_layout, void *stream) {
  DeviceGuard guard;
  FP4Q_TRY(check_matrix(x, dtype, rows, cols, ld));
  if (fp6_format != FP4Q_FP6_E2M3 && fp6_format != FP4Q_FP6_E3M2) return FP4Q_ERR_INVALID_ARG;
  if (e8m0_mode < FP4Q_E8M0_RNE || e8m0_mode > FP4Q_E8M0_OCP_FLOOR) return FP4Q_ERR_INVALID_ARG;
  if (!valid_layout(scale_layout)) return FP4Q_ERR_INVALID_ARG;
  if (cols % 32 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  FP4Q_TRY(check_swizzle(scale_layout, rows, cols / 32));
  if (rows == 0 || cols == 0) return FP4Q_OK;
  if (!q || !sf) return FP4Q_ERR_INVALID_ARG;
  if (!aligned16(q)) return FP4Q_ERR_MISALIGNED;
  Launch L;
  FP4Q_TRY(bind_device(x, stream, &L));
  FP4Q_TRY(check_dev(q, false));
  FP4Q_TRY(check_dev(sf, false));
  return cuda_status(
      launch_mxfp6(x, dtype, rows, cols, ld, fp6_format, e8m0_mode, q, sf, scale_layout, L));
}

namespace fp4q {
namespace {
fp4q_status gemm_checked(const uint8_t *qa, const uint8_t *sfa, const float *tensor_scale_a,
                         const uint8_t *qb, const uint8_t *sfb, const float *tensor_scale_b,
                         int64_t M, int64_t N, int64_t K, void *c, int c_dtype, int64_t ldc,
                         int *status, void *stream, int withhold, bool mx = false);
}  // namespace
}  // namespace fp4q

fp4q_status fp4q_gemm_nvfp4(const uint8_t *qa, const uint8_t *sfa, const float *tensor_scale_a,
                            const uint8_t *qb, const uint8_t *sfb, const float *tensor_scale_b,
                            int64_t M, int64_t N, int64_t K, void *c, int c_dtype, int64_t ldc,
                            int *status, void *stream) {
  DeviceGuard guard;
  return gemm_checked(qa, sfa, tensor_scale_a, qb, sfb, tensor_scale_b, M, N, K, c, c_dtype, ldc,
                      status, stream, 0);
}

size_t fp4q_gemm_if4_workspace_bytes(int64_t M, int64_t K) {
  if (M < 0 || K < 0) return 0;
  return static_cast<size_t>(3 * (M * K / 2) + M * K / 16);
}

fp4q_status fp4q_gemm_if4_nvfp4(const uint8_t *qa, const uint8_t *sfa, const float *tensor_scale_a,
                                const uint8_t *qb, const uint8_t *sfb,
                                const float *tensor_scale_b, int64_t M, int64_t N, int64_t K,
                                float *c, int64_t ldc, void *workspace, size_t ws_bytes,
                                int *status, void *stream) {
  DeviceGuard guard;
  if (M < 0 || N < 0 || K < 0 || ldc < N) return FP4Q_ERR_INVALID_ARG;
  if (M % 128 != 0 || N % 128 != 0 || K % 256 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if (K > (int64_t{1} << 30) || M / 128 > 65535) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return FP4Q_OK;
  if (!c) return FP4Q_ERR_INVALID_ARG;
  if (!aligned16(c) || (ldc * 4) % 16 != 0) return FP4Q_ERR_MISALIGNED;
  if (K > 0) {
    if (!qa || !sfa || !qb || !sfb) return FP4Q_ERR_INVALID_ARG;
    if (!aligned16(qa) || !aligned16(qb) || !aligned16(sfa) || !aligned16(sfb))
      return FP4Q_ERR_MISALIGNED;
    if (!workspace || ws_bytes < fp4q_gemm_if4_workspace_bytes(M, K))
      return FP4Q_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(workspace)) return FP4Q_ERR_MISALIGNED;
  }
  Launch L;
  FP4Q_TRY(bind_device(c, stream, &L));
  if (K == 0)
    return cuda_status(cudaMemset2DAsync(c, static_cast<size_t>(ldc * 4), 0,
                                         static_cast<size_t>(N * 4), static_cast<size_t>(M),
                                         L.stream));
  FP4Q_TRY(check_dev(qa, false));
  FP4Q_TRY(check_dev(sfa, false));
  FP4Q_TRY(check_dev(qb, false));
  FP4Q_TRY(check_dev(sfb, false));
  FP4Q_TRY(check_dev(workspace, false));
  FP4Q_TRY(check_dev(tensor_scale_a, true));
  FP4Q_TRY(check_dev(tensor_scale_b, true));
  FP4Q_TRY(check_dev(status, true));
  uint8_t *w = static_cast<uint8_t *>(workspace);
  const int64_t codes = M * K / 2;
  uint8_t *q_fp = w, *q_k1 = w + codes, *q_k2 = w + 2 * codes, *sf_plain = w + 3 * codes;
  FP4Q_TRY(cuda_status(launch_if4_split(qa, sfa, M, K, FP4Q_SCALE_SWIZZLED_128x4, q_fp, q_k1,
                                        q_k2, sf_plain, L)));
  return cuda_status(launch_gemm_if4_split(q_fp, q_k1, q_k2, sf_plain, tensor_scale_a, qb, sfb,
                                           tensor_scale_b, M, N, K, c, ldc, status, L));
}

fp4q_status fp4q_gemm_mxfp4(const uint8_t *qa, const uint8_t *sfa, const uint8_t *qb,
                            const uint8_t *sfb, int64_t M, int64_t N, int64_t K, void *c,
                            int c_dtype, int64_t ldc, int *status, void *stream) {
  DeviceGuard guard;
  return gemm_checked(qa, sfa, nullptr, qb, sfb, nullptr, M, N, K, c, c_dtype, ldc, status,
                      stream, 0, /*mx=*/true);
}

fp4q_status fp4q_gemm_nvfp4_withhold_loads(const uint8_t *qa, const uint8_t *sfa,
                                           const float *tensor_scale_a, const uint8_t *qb,
                                           const uint8_t *sfb, const float *tensor_scale_b,
                                           int64_t M, int64_t N, int64_t K, void *c, int c_dtype,
                                           int64_t ldc, int *status, void *stream) {
  DeviceGuard guard;
  if (!status || K == 0) return FP4Q_ERR_INVALID_ARG;   // the hook exists to set *status
  return gemm_checked(qa, sfa, tensor_scale_a, qb, sfb, tensor_scale_b, M, N, K, c, c_dtype, ldc,
                      status, stream, 1);
}

}  // extern "C"

namespace fp4q {
namespace {
fp4q_status gemm_checked(const uint8_t *qa, const uint8_t *sfa, const float *tensor_scale_a,
                         const uint8_t *qb, const uint8_t *sfb, const float *tensor_scale_b,
                         int64_t M, int64_t N, int64_t K, void *c, int c_dtype, int64_t ldc,
                         int *status, void *stream, int withhold, bool mx) {
  if (!valid_dtype(c_dtype)) return FP4Q_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0 || ldc < N) return FP4Q_ERR_INVALID_ARG;
  if (M % 128 != 0 || N % 128 != 0 || K % 256 != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if (K > (int64_t{1} << 30) || M / 128 > 65535 || N / 128 > (int64_t{1} << 30))
    return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return FP4Q_OK;
  if (!c) return FP4Q_ERR_INVALID_ARG;
  const int64_t esz = elem_size(c_dtype);
  if (!aligned16(c) || (ldc * esz) % 16 != 0) return FP4Q_ERR_MISALIGNED;
  if (K > 0) {
    if (!qa || !sfa || !qb || !sfb) return FP4Q_ERR_INVALID_ARG;
    if (!aligned16(qa) || !aligned16(qb) || !aligned16(sfa) || !aligned16(sfb))
      return FP4Q_ERR_MISALIGNED;
  }
  Launch L;
  FP4Q_TRY(bind_device(c, stream, &L));
  if (K == 0)   // an empty sum
    return cuda_status(cudaMemset2DAsync(c, static_cast<size_t>(ldc * esz), 0,
                                         static_cast<size_t>(N * esz), static_cast<size_t>(M),
                                         L.stream));
  FP4Q_TRY(check_dev(qa, false));
  FP4Q_TRY(check_dev(sfa, false));
  FP4Q_TRY(check_dev(qb, false));
  FP4Q_TRY(check_dev(sfb, false));
  FP4Q_TRY(check_dev(tensor_scale_a, true));
  FP4Q_TRY(check_dev(tensor_scale_b, true));
  FP4Q_TRY(check_dev(status, true));
  if (mx)
    return cuda_status(
        launch_gemm_mxfp4(qa, sfa, qb, sfb, M, N, K, c, c_dtype, ldc, status, L));
  GemmOptions opt;
  opt.withhold = withhold;
  return cuda_status(launch_gemm_nvfp4(qa, sfa, tensor_scale_a, qb, sfb, tensor_scale_b, M, N, K,
                                       c, c_dtype, ldc, status, opt, L));
}
}  // namespace
}  // namespace fp4q

extern "C" {

fp4q_status fp4q_dequantize(int format, const uint8_t *q, const uint8_t *sf, int scale_layout,
                            int block_rows, int block_cols, const float *tensor_scale,
                            int64_t rows, int64_t cols, void *y, int y_dtype, void *stream) {
  DeviceGuard guard;
  if (format < FP4Q_FMT_NVFP4 || format > FP4Q_FMT_IF3) return FP4Q_ERR_INVALID_ARG;
  const bool fp6 = format == FP4Q_FMT_MXFP6_E2M3 || format == FP4Q_FMT_MXFP6_E3M2;
  const bool pow2 = fp6 || format == FP4Q_FMT_MXFP4;   // E8M0 scales, no tensor scale
  if (!valid_layout(scale_layout) || !valid_dtype(y_dtype)) return FP4Q_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0) return FP4Q_ERR_INVALID_ARG;
  const bool shape_ok =
      (pow2 && block_rows == 1 && block_cols == 32) ||
      ((format == FP4Q_FMT_IF4 || format == FP4Q_FMT_IF6 || format == FP4Q_FMT_IF3) &&
       block_rows == 1 && block_cols == 16) ||
      (format == FP4Q_FMT_NVFP4 && block_cols == 16 && (block_rows == 1 || block_rows == 16));
  if (!shape_ok) return FP4Q_ERR_INVALID_ARG;
  if (cols % block_cols != 0 || rows % block_rows != 0) return FP4Q_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0 || cols == 0) return FP4Q_OK;
  if (!q || !sf || !y) return FP4Q_ERR_INVALID_ARG;
  if (!pow2 && !tensor_scale) return FP4Q_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(y)) return FP4Q_ERR_MISALIGNED;
  if (block_rows == 1) FP4Q_TRY(check_swizzle(scale_layout, rows, cols / block_cols));
  Launch L;
  FP4Q_TRY(bind_device(q, stream, &L));
  FP4Q_TRY(check_dev(sf, false));
  FP4Q_TRY(check_dev(y, false));
  FP4Q_TRY(check_dev(pow2 ? nullptr : tensor_scale, true));
  if (format == FP4Q_FMT_IF6)
    return cuda_status(
        launch_if6_dequant(q, sf, scale_layout, tensor_scale, rows, cols, y, y_dtype, L));
  if (format == FP4Q_FMT_IF3)
    return cuda_status(
        launch_if3_dequant(q, sf, scale_layout, tensor_scale, rows, cols, y, y_dtype, L));
  if (fp6)
    return cuda_status(launch_mxfp6_dequant(
        q, sf, scale_layout, rows, cols,
        format == FP4Q_FMT_MXFP6_E2M3 ? FP4Q_FP6_E2M3 : FP4Q_FP6_E3M2, y, y_dtype, L));
  return cuda_status(launch_dequant(format, q, sf, scale_layout, block_rows, block_cols,
                                    tensor_scale, rows, cols, y, y_dtype, L));
}

}  // extern "C"
