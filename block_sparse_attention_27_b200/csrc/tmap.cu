// tmap.cu -- TMA tensor maps for the paged K/V caches.  cuTensorMapEncodeTiled
// is fetched through the runtime's driver entry point, so the library needs no
// link-time dependency on libcuda.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "launch.h"

namespace dsa {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

// A paged cache [n_phys, Hkv, P, D] bf16 seen as a 2-D matrix of n_phys*Hkv*P
// rows of D elements; one box is `box_rows` rows x 64 elements (128 bytes),
// written to shared memory with the 128-byte swizzle.
cudaError_t make_kv_tensor_map(CUtensorMap *out, const void *base, long long rows, int D,
                               int box_rows) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (rows <= 0 || rows >= (1LL << 31)) return cudaErrorInvalidValue;  // int32 box coordinates
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t elem_strides[2] = {1u, 1u};
  CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                  box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The same cache seen as 4-D (D, P, Hkv, n_phys): one box is 64 elements x P
// tokens x 1 head x `pages` consecutive physical pages, i.e. `pages` whole pages
// of one KV head in one load, landing as pages*P rows of 128 bytes.
cudaError_t make_kv_pages_tensor_map(CUtensorMap *out, const void *base, long long n_phys, int Hkv,
                                     int P, int D, int pages) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)P, (cuuint64_t)Hkv, (cuuint64_t)n_phys};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)P * D * 2, (cuuint64_t)Hkv * P * D * 2};
  cuuint32_t box[4] = {64u, (cuuint32_t)P, 1u, (cuuint32_t)pages};
  cuuint32_t elem_strides[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                  box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The block's own keys or values [S*B, Hkv, D] bf16 as a 3-D tensor (D, Hkv,
// S*B); one box is 64 elements x 1 head x `box_tokens` tokens (64 by default), so
// one load brings up to that many consecutive tokens of one KV head (rows past
// S*B read as zeros).
cudaError_t make_blk_tensor_map(CUtensorMap *out, const void *base, long long tokens, int Hkv,
                                int D, int box_tokens) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (box_tokens < 1 || box_tokens > 256) return cudaErrorInvalidValue;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)tokens};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
  cuuint32_t box[3] = {64u, 1u, (cuuint32_t)box_tokens};
  cuuint32_t elem_strides[3] = {1u, 1u, 1u};
  CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                  box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The block's queries [S*B, Hq, D] bf16 as a 3-D tensor (D, Hq, S*B); one box is
// 64 elements x G heads x `tokens` tokens: the rows (b, g) of one KV head's group
// for `tokens` consecutive tokens, landing as tokens*G rows of 128 bytes in the
// order b*G + g (rows past S*B read as zeros).
cudaError_t make_q_tensor_map(CUtensorMap *out, const void *base, long long tokens, int Hq, int D,
                              int G, int box_tokens) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (G < 1 || G > 256 || box_tokens < 1 || box_tokens > 256) return cudaErrorInvalidValue;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)tokens};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
  cuuint32_t box[3] = {64u, (cuuint32_t)G, (cuuint32_t)box_tokens};
  cuuint32_t elem_strides[3] = {1u, 1u, 1u};
  CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                  box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace dsa
