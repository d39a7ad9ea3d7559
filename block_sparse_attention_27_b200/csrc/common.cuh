// common.cuh -- device helpers shared by the libdsa kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

// Bits of the device status word (first 4 bytes of every workspace).
enum : uint32_t {
  kStatusTimeout = 1u,
  kStatusBadIndex = 2u,
  kStatusNonfinite = 4u,
};

// Bytes reserved at the head of every workspace: status word + counters.
constexpr size_t kWorkspaceHeader = 4096;

// Opts kernel K into `bytes` of dynamic shared memory once per device.  The
// attribute belongs to one function on one device, so the flag is kept per
// kernel (a template parameter, not the kernel's type, which all
// instantiations of a kernel template share) and per device.  Doing it once also
// keeps the call out of later graph captures.
template <auto K>
inline cudaError_t set_smem_once(size_t bytes) {
  static unsigned long long done = 0;  // bit per device ordinal < 64
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (__atomic_load_n(&done, __ATOMIC_ACQUIRE) & bit)) return cudaSuccess;
  err = cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (err == cudaSuccess && bit) __atomic_fetch_or(&done, bit, __ATOMIC_ACQ_REL);
  return err;
}

__device__ __forceinline__ void raise_status(uint32_t *status, uint32_t bit) {
  atomicOr(status, bit);
}

// Prefix length of a sequence, clamped to what the page table can address; an
// out-of-range n_ctx is reported as a bad index instead of being followed.
__device__ __forceinline__ int clamp_prefix(int n, int max_pages, int page, uint32_t *status,
                                            bool report) {
  const int cap = max_pages * page;
  if (n < 0 || n > cap) {
    if (report) raise_status(status, kStatusBadIndex);
    n = n < 0 ? 0 : cap;
  }
  return n;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for two halves at once (MUFU ex2 on an f16x2 pair: one instruction for two
// values); inputs and results in half precision.
__device__ __forceinline__ uint32_t fast_exp2_h2(uint32_t x) {
  uint32_t y;
  asm("ex2.approx.f16x2 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace dsa
