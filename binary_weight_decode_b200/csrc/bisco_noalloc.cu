// bisco_gemv_noalloc: the GEMV entry point for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a workspace buffer: a plug-in loaded into a host
// application that owns every device allocation, code that runs while a stream is
// being captured into a CUDA graph (where a fresh allocation would break the capture),
// or a runtime whose device memory is fully reserved at start-up. For them this file
// keeps the scratch space bisco_gemv needs (the device status word and, for layers with
// a binary low-rank correction, the intermediate z of one batch chunk) in a fixed array
// that lives in the library's own device image. Every GPU that loads the library holds
// this array until the process exits.

#include <cuda_runtime.h>

#include <mutex>

#include "bisco_internal.h"

namespace {

// 256 bytes for the status word, then z for one chunk of 8 batch rows at the largest
// supported correction rank.
constexpr size_t kScratchBytes = bisco::kStatusBytes + static_cast<size_t>(bisco::kMaxBatchChunk) * BISCO_NOALLOC_MAX_RANK * 4;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on each device. The symbol's name is only a
// host-side handle, so the address is looked up once per device, with that device
// current, and cached.
void* scratch_address(int dev, cudaError_t* err) {
  static std::once_flag once[kMaxDevices];
  static void* addr[kMaxDevices];
  static cudaError_t status[kMaxDevices];
  std::call_once(once[dev], [dev] {
    void* p = nullptr;
    status[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    addr[dev] = status[dev] == cudaSuccess ? p : nullptr;
  });
  *err = status[dev];
  return addr[dev];
}

}  // namespace

extern "C" bisco_status bisco_gemv_noalloc(const bisco_layer* layer, const void* X, int32_t x_dtype, int32_t M,
                                           void* Y, int32_t y_dtype, void* stream) {
  if (!layer) return BISCO_ERR_INVALID_ARG;
  if (layer->rank > BISCO_NOALLOC_MAX_RANK) return BISCO_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BISCO_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BISCO_ERR_UNSUPPORTED;
  cudaError_t err = cudaSuccess;
  void* ws = scratch_address(dev, &err);
  if (err != cudaSuccess || ws == nullptr) return BISCO_ERR_CUDA;
  // z is written in full by the correction's first pass before the second pass reads
  // it, and the status word is only ever set, so nothing here has to start at zero.
  return bisco_gemv(layer, X, x_dtype, M, Y, y_dtype, ws, kScratchBytes, stream);
}
