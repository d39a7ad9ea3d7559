// sparse.cu -- sparse pass for denoising steps 2..T ("MAGE: All-[MASK] Block
// Already Knows Where to Look in Block Diffusion LLM", Approach: the step-1
// indices are reused for every later step).  Each query row of the block attends
// to the tokens of the selected pages of its KV head plus the block's own B
// tokens, with no mask inside the block.
//
// One launch per step.  A thread-block cluster of C CTAs serves one (sequence,
// KV head, 128-row tile): CTA c runs the tcgen05 engine (tc_attn.cuh) over its
// slice [c*ppc, (c+1)*ppc) of the selected pages, gathered page by page with TMA
// through the page table; the last CTA also takes the block's own tokens
// (a 3-D TMA box over blk_k / blk_v).  The C partial results (unnormalised O in
// shared memory, row max m and sum l) are merged through distributed shared
// memory: after a cluster barrier CTA c reads every CTA's (m, l, O) for its
// share of the rows and writes those rows of o_out in bf16.
#include <algorithm>

#include "launch.h"
#include "sm100.cuh"
#include "tc_attn.cuh"

namespace dsa {
namespace {

constexpr int kSpStages = 2;
constexpr int kRowsPerCta = 128;

struct SparseParams {
  Shape sh;
  SparsePlan plan;
  SparseArgs a;
};

template <int D, int PAGE>
struct SparsePolicy {
  static constexpr int kPagesPerTile = tc::kBN / PAGE;
  const Shape *sh;
  const SparseArgs *a;
  const CUtensorMap *kmap, *vmap, *bkmap, *bvmap;
  int s, h, n, np, e_begin, e_end, sel_tiles, row_base;
  size_t sh_idx;
  float sl2;

  // physical page of selected entry e, or -1 if the entry is not usable
  __device__ __forceinline__ long long phys_of(int e, int &lp) const {
    lp = -1;
    if (e >= e_end) return -1;
    lp = a->idx[sh_idx * sh->kmax + e];
    if (lp < 0 || lp >= np) return -1;
    const long long p = sh->page_table ? (long long)sh->page_table[(size_t)s * sh->max_pages + lp]
                                       : (long long)s * sh->max_pages + lp;
    return (p >= 0 && p < sh->n_phys) ? p : -1;
  }
  __device__ __forceinline__ void prefetch() const {
    sm100::tma_prefetch_map(kmap);
    sm100::tma_prefetch_map(vmap);
    sm100::tma_prefetch_map(bkmap);
    sm100::tma_prefetch_map(bvmap);
  }
  __device__ __forceinline__ void load_tile(int k, uint32_t sk, uint32_t sv, uint32_t half_bytes,
                                            uint32_t bar) const {
    if (k < sel_tiles) {
      const int e0 = e_begin + k * kPagesPerTile;
      long long phys[kPagesPerTile];
      uint32_t nvalid = 0;
#pragma unroll
      for (int pi = 0; pi < kPagesPerTile; ++pi) {
        int lp;
        phys[pi] = phys_of(e0 + pi, lp);
        if (phys[pi] >= 0) ++nvalid;
        else if (e0 + pi < e_end) raise_status(a->status, kStatusBadIndex);
      }
      sm100::mbar_arrive_expect_tx(bar, nvalid * PAGE * 128u * (D / 64) * 2u);
#pragma unroll
      for (int pi = 0; pi < kPagesPerTile; ++pi) {
        if (phys[pi] < 0) continue;
        const int y = (int)((phys[pi] * sh->Hkv + h) * PAGE);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          sm100::tma_load_2d(sk + hf * half_bytes + pi * PAGE * 128, kmap, bar, hf * 64, y);
          sm100::tma_load_2d(sv + hf * half_bytes + pi * PAGE * 128, vmap, bar, hf * 64, y);
        }
      }
    } else {  // the block's own tokens u = 64j .. 64j+63 of this sequence
      const int j = k - sel_tiles;
      sm100::mbar_arrive_expect_tx(bar, 64u * 128u * (D / 64) * 2u);
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf) {
        sm100::tma_load_3d(sk + hf * half_bytes, bkmap, bar, hf * 64, h, s * sh->B + j * 64);
        sm100::tma_load_3d(sv + hf * half_bytes, bvmap, bar, hf * 64, h, s * sh->B + j * 64);
      }
    }
  }
  __device__ __forceinline__ const __nv_bfloat16 *q_row(int r) const {
    const int row = row_base + r;
    if (row >= sh->BG) return nullptr;
    const int b = row / sh->G, g = row % sh->G;
    return a->q + (((size_t)s * sh->B + b) * sh->Hq + (size_t)h * sh->G + g) * D;
  }
  __device__ __forceinline__ uint64_t key_mask(int k) const {
    uint64_t m = 0;
    if (k < sel_tiles) {
      const int e0 = e_begin + k * kPagesPerTile;
#pragma unroll
      for (int pi = 0; pi < kPagesPerTile; ++pi) {
        int lp;
        if (phys_of(e0 + pi, lp) < 0) continue;
        const int cnt = min(PAGE, n - lp * PAGE);
        if (cnt > 0) m |= ((cnt >= 64) ? ~0ull : ((1ull << cnt) - 1ull)) << (pi * PAGE);
      }
    } else {
      const int cnt = min(64, sh->B - (k - sel_tiles) * 64);
      if (cnt > 0) m = (cnt >= 64) ? ~0ull : ((1ull << cnt) - 1ull);
    }
    return m;
  }
  __device__ __forceinline__ void after_tile(int, int, float, const float *) const {}
};

template <int D, int PAGE>
__global__ void __launch_bounds__(tc::kThreads, 1)
    sparse_attn(const SparseParams prm, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap bkmap,
                const __grid_constant__ CUtensorMap bvmap) {
  using L = tc::Layout<D, kSpStages>;
  extern __shared__ unsigned char smem_raw[];
  const Shape &sh = prm.sh;
  const SparsePlan &plan = prm.plan;
  const SparseArgs &a = prm.a;
  const int C = plan.cluster;   // cluster size == gridDim.x
  const int c = blockIdx.x;     // rank in the cluster
  const int h = blockIdx.y;
  const int s = blockIdx.z / plan.rowtiles, rt = blockIdx.z % plan.rowtiles;
  const size_t sh_idx = (size_t)s * sh.Hkv + h;
  const bool reporter = threadIdx.x == 0 && c == 0 && rt == 0;
  const int n = clamp_prefix(a.n_ctx[s], sh.max_pages, PAGE, a.status, reporter && h == 0);
  int cnt = a.idx_cnt[sh_idx];
  if (cnt < 0 || cnt > sh.kmax) {
    if (reporter) raise_status(a.status, kStatusBadIndex);
    cnt = max(0, min(cnt, sh.kmax));
  }
  const int e_begin = min(cnt, c * plan.ppc), e_end = min(cnt, (c + 1) * plan.ppc);
  constexpr int kPagesPerTile = tc::kBN / PAGE;
  const int sel_tiles = (e_end - e_begin + kPagesPerTile - 1) / kPagesPerTile;
  const int num_tiles = sel_tiles + (c == C - 1 ? plan.blk_tiles : 0);
  const int row_base = rt * kRowsPerCta;

  tc::Engine<D, kSpStages> eng;
  eng.init(smem_raw, a.status);
  SparsePolicy<D, PAGE> pol{&sh, &a, &kmap, &vmap, &bkmap, &bvmap, s, h, n,
                            (n + PAGE - 1) / PAGE, e_begin, e_end, sel_tiles, row_base,
                            sh_idx, sh.sl2};
  float m, l;
  const bool alive = eng.template run<PAGE>(pol, num_tiles, m, l);

  // ---- this CTA's partial into its shared memory (the K/V/P area is free now)
  constexpr int kOStride = D + 4;  // floats per row, padded against bank conflicts
  float *obuf = reinterpret_cast<float *>(eng.smem + L::kOffKV);
  float2 *ml = reinterpret_cast<float2 *>(eng.smem + L::kOffKV + 128 * kOStride * 4);
  float2 *gml = ml + 128;                                   // [rows][C] gathered (m, l)
  float *wts = reinterpret_cast<float *>(gml + 128 + 16);   // [rows][C] merge weights
  static_assert(L::kOffKV + 128 * kOStride * 4 + (128 + 128 + 16) * 8 + (128 + 16) * 4 <= L::kOffBar,
                "merge buffers must fit in the K/V/P area");
  if (eng.warp >= 2) {
    const int r = eng.row_in_tile();
    if (alive) {
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        eng.load_o(c0, o);
        float4 *dst = reinterpret_cast<float4 *>(obuf + r * kOStride + c0);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                               __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
      }
    }
    ml[r] = alive ? make_float2(m, l) : make_float2(-INFINITY, 0.f);
  }
  sm100::cluster_sync();

  // ---- merge: CTA c owns rows [c*rpc, (c+1)*rpc) of the tile
  const int rows_here = min(kRowsPerCta, sh.BG - row_base);
  const int rpc = (kRowsPerCta + C - 1) / C;
  const int r0 = c * rpc;
  const int r1 = min(rows_here, r0 + rpc);
  const int nrows = max(0, r1 - r0);
  const uint32_t ml_addr = smem_addr(ml), o_addr = smem_addr(obuf);
  for (int t = threadIdx.x; t < nrows * C; t += blockDim.x) {
    const int rl = t / C, j = t % C;
    gml[t] = sm100::ld_cluster_f2(sm100::cluster_map(ml_addr + (r0 + rl) * 8, j));
  }
  __syncthreads();
  for (int rl = threadIdx.x; rl < nrows; rl += blockDim.x) {
    float M = -INFINITY;
    for (int j = 0; j < C; ++j)
      if (gml[rl * C + j].y > 0.f) M = fmaxf(M, gml[rl * C + j].x);
    float Lsum = 0.f;
    for (int j = 0; j < C; ++j) {
      const float2 v = gml[rl * C + j];
      const float w = v.y > 0.f ? exp2f(v.x - M) : 0.f;
      wts[rl * C + j] = w;
      Lsum += w * v.y;
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    for (int j = 0; j < C; ++j) wts[rl * C + j] *= inv;
  }
  __syncthreads();
  constexpr int kQuads = D / 4;
  for (int t = threadIdx.x; t < nrows * kQuads; t += blockDim.x) {
    const int rl = t / kQuads, q4 = t % kQuads;
    const int row = r0 + rl;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < C; ++j) {
      const float w = wts[rl * C + j];
      if (w == 0.f) continue;  // an empty partial: its buffer holds no data
      const float4 v =
          sm100::ld_cluster_f4(sm100::cluster_map(o_addr + (row * kOStride + 4 * q4) * 4, j));
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
    const int grow = row_base + row;
    const int b = grow / sh.G, g = grow % sh.G;
    __nv_bfloat16 *dst =
        a.o_out + (((size_t)s * sh.B + b) * sh.Hq + (size_t)h * sh.G + g) * D + 4 * q4;
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t *>(&lo);
    packed.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(dst) = packed;
  }
  sm100::cluster_sync();  // no CTA leaves while another may still read its shared memory
  eng.teardown();
}

// Largest cluster size (16, 8, 4, 2) that the device can schedule with this
// kernel's shared memory, queried once per device; 1 if none.
template <auto K>
int max_cluster(size_t smem) {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int best = 1;
    for (int cs = 16; cs >= 2; cs >>= 1) {
      if (cs > 8 &&
          cudaFuncSetAttribute(K, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        continue;
      }
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(cs, 1, 1);
      cfg.blockDim = dim3(tc::kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cs;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int nclusters = 0;
      if (cudaOccupancyMaxActiveClusters(&nclusters, K, &cfg) == cudaSuccess && nclusters >= 1) {
        best = cs;
        break;
      }
      cudaGetLastError();
    }
    cached[dev] = best;
  }
  return cached[dev];
}

template <int D, int PAGE>
cudaError_t launch_typed(const Shape &sh, const SparsePlan &plan_in, const SparseArgs &a,
                         cudaStream_t stream) {
  constexpr auto kern = sparse_attn<D, PAGE>;
  constexpr size_t smem = tc::Layout<D, kSpStages>::kAlloc;
  cudaError_t err = set_smem_once<kern>(smem);
  if (err != cudaSuccess) return err;
  SparsePlan plan = plan_in;
  const int cap = max_cluster<kern>(smem);
  if (plan.cluster > cap) {
    plan.cluster = cap;
    plan.ppc = (sh.kmax + cap - 1) / cap;
  }
  CUtensorMap kmap, vmap, bkmap, bvmap;
  const long long rows = sh.n_phys * sh.Hkv * PAGE;
  if ((err = make_kv_tensor_map(&kmap, a.k, rows, D, PAGE)) != cudaSuccess) return err;
  if ((err = make_kv_tensor_map(&vmap, a.v, rows, D, PAGE)) != cudaSuccess) return err;
  if ((err = make_blk_tensor_map(&bkmap, a.blk_k, (long long)sh.S * sh.B, sh.Hkv, D)) != cudaSuccess)
    return err;
  if ((err = make_blk_tensor_map(&bvmap, a.blk_v, (long long)sh.S * sh.B, sh.Hkv, D)) != cudaSuccess)
    return err;
  SparseParams prm{sh, plan, a};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.cluster, sh.Hkv, sh.S * plan.rowtiles);
  cfg.blockDim = dim3(tc::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = plan.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, kern, prm, kmap, vmap, bkmap, bvmap);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

SparsePlan plan_sparse(const Shape &sh, int /*num_sms*/) {
  SparsePlan p{};
  p.rowtiles = (sh.BG + kRowsPerCta - 1) / kRowsPerCta;
  int cs = std::min(16, std::max(1, sh.kmax));
  while (cs & (cs - 1)) cs &= cs - 1;  // power of two
  p.cluster = cs;
  p.ppc = (sh.kmax + cs - 1) / cs;
  p.blk_tiles = (sh.B + tc::kBN - 1) / tc::kBN;
  p.total = 4096;  // status word only: partials never leave the cluster
  return p;
}

cudaError_t launch_sparse(const Shape &sh, const SparsePlan &plan, const SparseArgs &a,
                          cudaStream_t stream) {
  if (sh.d == 128) {
    if (sh.P == 16) return launch_typed<128, 16>(sh, plan, a, stream);
    if (sh.P == 32) return launch_typed<128, 32>(sh, plan, a, stream);
    if (sh.P == 64) return launch_typed<128, 64>(sh, plan, a, stream);
  } else if (sh.d == 64) {
    if (sh.P == 16) return launch_typed<64, 16>(sh, plan, a, stream);
    if (sh.P == 32) return launch_typed<64, 32>(sh, plan, a, stream);
    if (sh.P == 64) return launch_typed<64, 64>(sh, plan, a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dsa
