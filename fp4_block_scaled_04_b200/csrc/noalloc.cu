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
// while that device is current and caches it.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "fp4q.h"

namespace {

constexpr size_t kScratchBytes = 256;
constexpr int kMaxDevices = 64;

// Holds the tensor amax of the latest call that computed one.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices];

// Device address of g_scratch on `dev` (which must be current), looked up
// once per device.
fp4q_status scratch_on(int dev, void **out) {
  if (dev < 0 || dev >= kMaxDevices) return FP4Q_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return FP4Q_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FP4Q_OK;
}

}  // namespace

extern "C" fp4q_status fp4q_quantize_nvfp4_noalloc(
    const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld, unsigned layouts, int round,
    uint64_t seed, const float *amax, float *tensor_scale_out, uint8_t *q_row, uint8_t *sf_row,
    uint8_t *q_col, uint8_t *sf_col, int scale_layout, void *stream) {
  if (fp4q_workspace_bytes() > kScratchBytes) return FP4Q_ERR_WORKSPACE_TOO_SMALL;
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
      int cur = -1;
      if (cudaGetDevice(&cur) != cudaSuccess || cur != attr.device)
        if (cudaSetDevice(attr.device) != cudaSuccess) return FP4Q_ERR_CUDA;
      fp4q_status s = scratch_on(attr.device, &scratch);
      if (s != FP4Q_OK) return s;
    }
  }
  // The amax pre-pass clears its float before reducing into it.
  return fp4q_quantize_nvfp4(x, dtype, rows, cols, ld, layouts, round, seed, amax,
                             tensor_scale_out, q_row, sf_row, q_col, sf_col, scale_layout,
                             scratch, scratch ? kScratchBytes : 0, stream);
}
