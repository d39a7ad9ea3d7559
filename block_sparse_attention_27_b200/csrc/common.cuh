// common.cuh -- device helpers shared by the libdsa kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

constexpr float kLog2e = 1.4426950408889634f;

// Bits of the device status word (first 4 bytes of every workspace).
enum : uint32_t {
  kStatusTimeout = 1u,
  kStatusBadIndex = 2u,
  kStatusNonfinite = 4u,
};

// Bytes reserved at the head of every workspace: status word + counters.
constexpr size_t kWorkspaceHeader = 4096;

// Opts a kernel into `bytes` of dynamic shared memory once per device (the
// attribute is per function and device; setting it on every launch would also
// be a non-stream call inside graph capture).
template <class Kernel>
inline cudaError_t set_smem_once(Kernel kern, size_t bytes) {
  static unsigned long long done = 0;  // bit per device ordinal < 64
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (__atomic_load_n(&done, __ATOMIC_ACQUIRE) & bit)) return cudaSuccess;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
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

// ---- Ampere-style async copies (16-byte granules, zero fill when invalid) ----
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  const int bytes = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// ---- ldmatrix / mma.sync (bf16 in, fp32 accumulate) ----
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
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

// Row-major bf16 tile with rows of D elements, 16-byte chunks XOR-swizzled by
// (row & 7) so that ldmatrix over 8 consecutive rows hits 8 distinct bank groups.
template <int D>
struct SwizzledTile {
  static constexpr int kChunks = D / 8;  // 16-byte chunks per row
  __device__ __forceinline__ static uint32_t offset(int row, int chunk) {
    return static_cast<uint32_t>(row * (D * 2) + ((chunk ^ (row & 7)) << 4));
  }
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace dsa
