// bisco_gemv_noalloc: the GEMV entry point for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a workspace buffer: a plug-in loaded into a host
// application that owns every device allocation and hands the plug-in only its
// operands, or a runtime whose device memory is fully reserved at start-up. For them
// this file keeps the scratch space bisco_gemv needs (the device status word and, for
// layers with a binary low-rank correction, the intermediate z of one batch chunk) in a
// fixed array that lives in the library's own device image. Every GPU that loads the
// library holds this array until the process exits.

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
// host-side handle, so the address is looked up with that device current and cached.
// Only a successful lookup is cached: a failed one (e.g. a transient error) is retried
// on the next call. A device reset (cudaDeviceReset) invalidates the cached address;
// callers that reset a device must not call this entry point on it afterwards.
void* scratch_address(int dev, cudaError_t* err) {
  static std::mutex mu[kMaxDevices];
  static void* addr[kMaxDevices];
  std::lock_guard<std::mutex> g(mu[dev]);
  if (addr[dev] != nullptr) {
    *err = cudaSuccess;
    return addr[dev];
  }
  void* p = nullptr;
  *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (*err != cudaSuccess) {
    cudaGetLastError();  // clear the (non-sticky) error so that a retry starts clean
    return nullptr;
  }
  addr[dev] = p;
  return p;
}

}  // namespace

extern "C" bisco_status bisco_gemv_noalloc(const bisco_layer* layer, const void* X, int32_t x_dtype, int32_t M,
                                           void* Y, int32_t y_dtype, void* stream) {
  if (!layer) return BISCO_ERR_INVALID_ARG;
  if (layer->rank > BISCO_NOALLOC_MAX_RANK || layer->ref_bases > 0) return BISCO_ERR_UNSUPPORTED;
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
