// merge.cu -- dsa_merge_attn: two softmax-attention results over disjoint key
// sets, each with its rows' log-sum-exp, combined into the result over the union
// (the exact step-1 output from the selection pass's prefix-only output and the
// block-only sparse pass; see include/dsa.h).  One row per warp, 8 columns per
// lane and step: an HBM-bound elementwise pass.
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace dsa {
namespace {

constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads)
    merge_attn(const __nv_bfloat16 *__restrict__ o_a, const float *__restrict__ lse_a,
               const __nv_bfloat16 *__restrict__ o_b, const float *__restrict__ lse_b,
               __nv_bfloat16 *o_out, float *lse_out, long long rows, int d) {
  sm100::grid_dep_wait();  // the two results come from the kernels ahead
  sm100::grid_dep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (kMergeThreads / 32);
  for (long long row = (long long)blockIdx.x * (kMergeThreads / 32) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const float la = lse_a[row], lb = lse_b[row];
    const float mx = fmaxf(la, lb);
    float wa = 0.f, wb = 0.f, lse = -INFINITY;
    if (mx > -INFINITY) {
      const float ea = expf(la - mx), eb = expf(lb - mx);
      const float sum = ea + eb;
      wa = ea / sum;
      wb = eb / sum;
      lse = mx + logf(sum);
    }
    const uint4 *pa = reinterpret_cast<const uint4 *>(o_a + row * d);
    const uint4 *pb = reinterpret_cast<const uint4 *>(o_b + row * d);
    uint4 *po = reinterpret_cast<uint4 *>(o_out + row * d);
    for (int c = lane; c < d / 8; c += 32) {
      const uint4 va = pa[c], vb = pb[c];
      const __nv_bfloat162 *ha = reinterpret_cast<const __nv_bfloat162 *>(&va);
      const __nv_bfloat162 *hb = reinterpret_cast<const __nv_bfloat162 *>(&vb);
      uint4 out;
      uint32_t *w = reinterpret_cast<uint32_t *>(&out);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(ha[e]), fb = __bfloat1622float2(hb[e]);
        // a zero weight keeps the other side's values out entirely
        const float x = (wa > 0.f ? wa * fa.x : 0.f) + (wb > 0.f ? wb * fb.x : 0.f);
        const float y = (wa > 0.f ? wa * fa.y : 0.f) + (wb > 0.f ? wb * fb.y : 0.f);
        __nv_bfloat162 r = __floats2bfloat162_rn(x, y);
        w[e] = *reinterpret_cast<uint32_t *>(&r);
      }
      po[c] = out;
    }
    if (lse_out && lane == 0) lse_out[row] = lse;
  }
}

}  // namespace

cudaError_t launch_merge(const __nv_bfloat16 *o_a, const float *lse_a, const __nv_bfloat16 *o_b,
                         const float *lse_b, __nv_bfloat16 *o_out, float *lse_out, long long rows,
                         int d, cudaStream_t stream) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long need = (rows + kMergeThreads / 32 - 1) / (kMergeThreads / 32);
  const int grid = (int)std::min<long long>(need, 8LL * sms);
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kMergeThreads, 1, 1);
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, merge_attn, o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace dsa
