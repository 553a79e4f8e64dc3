// Device helpers shared by the integer tensor-core GEMV kernel: shared-memory
// addresses, mbarriers with bounded waits, bulk global->shared copies and the
// 8-element loads of scales and activations.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "bisco_internal.h"

namespace bisco {
namespace dev {

__device__ __forceinline__ unsigned saddr(const void* a) { return static_cast<unsigned>(__cvta_generic_to_shared(a)); }

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* b, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, unsigned parity) {
  unsigned done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(saddr(b)), "r"(parity)
      : "memory");
  return done != 0;
}
// Waits at most limit_ns for the phase with the given parity; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, unsigned parity, unsigned long long limit_ns) {
  if (mbar_try(b, parity)) return true;
  const unsigned long long end = global_ns() + limit_ns;
  while (!mbar_try(b, parity))
    if (global_ns() > end) return false;
  return true;
}
// Global -> shared bulk copy (no multicast) whose completion is counted on mbarrier b.
__device__ __forceinline__ void bulk_copy(void* dst, const void* src, unsigned bytes, uint64_t* b) {
  asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(saddr(dst)),
               "l"(src), "r"(bytes), "r"(saddr(b))
               : "memory");
}

// Eight consecutive values v[j] = a[off + j] (bf16 or fp32) as fp32, zero where
// j >= valid. One 16-byte load (two for fp32) when `vec` says the run is aligned.
// Read-only data (weights and scales): non-coherent loads.
__device__ __forceinline__ void load8_ro(const void* a, long long off, int dt, int valid, bool vec, float v[8]) {
  if (dt == BISCO_BF16) {
    const unsigned short* h = reinterpret_cast<const unsigned short*>(a) + off;
    if (vec && valid >= 8) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(h));
      const unsigned w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = j < valid ? __uint_as_float(static_cast<unsigned>(__ldg(h + j)) << 16) : 0.f;
    }
  } else {
    const float* f = reinterpret_cast<const float*>(a) + off;
    if (vec && valid >= 8) {
      const float4 q0 = __ldg(reinterpret_cast<const float4*>(f));
      const float4 q1 = __ldg(reinterpret_cast<const float4*>(f) + 1);
      v[0] = q0.x; v[1] = q0.y; v[2] = q0.z; v[3] = q0.w;
      v[4] = q1.x; v[5] = q1.y; v[6] = q1.z; v[7] = q1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = j < valid ? __ldg(f + j) : 0.f;
    }
  }
}

// The same for activations, which the previous kernel on the stream may have written:
// coherent loads through L2.
__device__ __forceinline__ void load8_act(const void* a, long long off, int dt, int valid, bool vec, float v[8]) {
  if (dt == BISCO_BF16) {
    const unsigned short* h = reinterpret_cast<const unsigned short*>(a) + off;
    if (vec && valid >= 8) {
      const uint4 q = __ldcg(reinterpret_cast<const uint4*>(h));
      const unsigned w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = j < valid ? __uint_as_float(static_cast<unsigned>(__ldcg(h + j)) << 16) : 0.f;
    }
  } else {
    const float* f = reinterpret_cast<const float*>(a) + off;
    if (vec && valid >= 8) {
      const float4 q0 = __ldcg(reinterpret_cast<const float4*>(f));
      const float4 q1 = __ldcg(reinterpret_cast<const float4*>(f) + 1);
      v[0] = q0.x; v[1] = q0.y; v[2] = q0.z; v[3] = q0.w;
      v[4] = q1.x; v[5] = q1.y; v[6] = q1.z; v[7] = q1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = j < valid ? __ldcg(f + j) : 0.f;
    }
  }
}

}  // namespace dev
}  // namespace bisco
