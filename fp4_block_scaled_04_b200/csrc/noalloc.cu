// noalloc.cu -- fp4q_quantize_nvfp4_noalloc: NVFP4 quantization for callers
// that cannot allocate device memory.
//
// fp4q_quantize_nvfp4 needs a small caller-provided workspace when it has to
// compute the tensor amax itself.  Some callers have no way to provide one:
// code running inside another framework's memory pool that forbids extra
// allocations, plugins whose host application owns every device buffer, or
// hosts that must not call cudaMalloc between set-up and shutdown.  This entry
// point takes that workspace from an array that lives in the library itself,
// so the caller passes only inputs and outputs.
//
// The array is file-scope device memory: every GPU that loads the library
// holds its bytes until the process exits.  Host code cannot use the array's
// name as a device address (on the host it is only a stand-in), so the first
// call on each device looks the device address up with cudaGetSymbolAddress
// while that device is current and caches it together with the identity of
// the device's current context; a later call in a new context (after a
// cudaDeviceReset, say) looks it up again.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "fp4q.h"
#include "launch.h"

namespace {

constexpr size_t kScratchBytes = 256;
constexpr int kMaxDevices = 64;

// Holds the tensor amax of the latest call that computed one.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices];
unsigned long long g_scratch_ctx[kMaxDevices];   // context id the address belongs to

// Unique id of the calling thread's current context (never reused within a
// process), or 0 when the driver cannot say.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext *);
  using GetId = CUresult (*)(CUcontext, unsigned long long *);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
    cudaGetLastError();
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx != nullptr &&
      get_id(ctx, &id) == CUDA_SUCCESS)
    return id;
  return 0;
}

// Device address of g_scratch on `dev` (which must be current), looked up
// once per device and context.
fp4q_status scratch_on(int dev, void **out) {
  if (dev < 0 || dev >= kMaxDevices) return FP4Q_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mutex);
  const unsigned long long ctx = current_context_id();
  if (g_scratch_ptr[dev] == nullptr || ctx == 0 || g_scratch_ctx[dev] != ctx) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      g_scratch_ptr[dev] = nullptr;
      return FP4Q_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return FP4Q_OK;
}

}  // namespace

extern "C" fp4q_status fp4q_quantize_nvfp4_noalloc(
    const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld, unsigned layouts, int round,
    uint64_t seed, const float *amax, float *tensor_scale_out, uint8_t *q_row, uint8_t *sf_row,
    uint8_t *q_col, uint8_t *sf_col, int scale_layout, void *stream) {
  fp4q::DeviceGuard guard;
  // everything fp4q_quantize_nvfp4 would reject is rejected first, before
  // any device is touched
  const int checked = fp4q::check_nvfp4_args(x, dtype, rows, cols, ld, layouts, round, q_row,
                                             sf_row, q_col, sf_col, scale_layout);
  if (checked != FP4Q_OK) return static_cast<fp4q_status>(checked);
  if (fp4q_workspace_bytes(rows, cols) > kScratchBytes) return FP4Q_ERR_WORKSPACE_TOO_SMALL;
  void *scratch = nullptr;
  if (amax == nullptr) {
    // The scratch must be the copy on the device that will run the kernels:
    // the device owning x (or, for an empty x, the output scale).
    const void *anchor = x != nullptr ? x : tensor_scale_out;
    if (anchor != nullptr) {
      cudaPointerAttributes attr;
      if (cudaPointerGetAttributes(&attr, anchor) != cudaSuccess) {
        cudaGetLastError();
        return FP4Q_ERR_INVALID_ARG;
      }
      if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
        return FP4Q_ERR_INVALID_ARG;
      if (attr.device < 0 || attr.device >= kMaxDevices) return FP4Q_ERR_INVALID_ARG;
      int cur = -1;
      if (cudaGetDevice(&cur) != cudaSuccess || cur != attr.device) {
        if (cudaSetDevice(attr.device) != cudaSuccess) {
          cudaGetLastError();
          return FP4Q_ERR_CUDA;
        }
      }
      fp4q_status s = scratch_on(attr.device, &scratch);
      if (s != FP4Q_OK) return s;
    }
  }
  // The amax pre-pass clears its float before reducing into it.
  return fp4q_quantize_nvfp4(x, dtype, rows, cols, ld, layouts, round, seed, amax,
                             tensor_scale_out, q_row, sf_row, q_col, sf_col, scale_layout,
                             scratch, scratch ? kScratchBytes : 0, stream);
}
