// sparse.cu -- sparse pass for denoising steps 2..T ("MAGE: All-[MASK] Block
// Already Knows Where to Look in Block Diffusion LLM", Approach: the step-1
// indices are reused for every later step).  Each query row of the block attends
// to the tokens of the selected pages of its KV head plus the block's own B
// tokens, with no mask inside the block.
//
// Two launches on the caller's stream:
//   1. sparse_partial: CTA = (64-key tile, row tile) x KV head x sequence.  The
//      key list of a (seq, KV head) is its selected pages in idx order followed by
//      the block's own tokens; tile t covers keys [64t, 64t+64).  The CTA gathers
//      its keys/values (page table lookup, bounds-checked), runs 8 warps x 16 rows
//      of attention and writes an unnormalised partial (O, m, l).
//   2. sparse_merge: one warp per query row merges the tiles' partials into o_out.
#include <algorithm>

#include "attn_core.cuh"
#include "launch.h"

namespace dsa {
namespace {

constexpr int kSpThreads = 256;
constexpr int kRowsPerCta = 128;

struct SparseParams {
  Shape sh;
  SparsePlan plan;
  SparseArgs a;
};

template <int D, int PAGE>
__global__ void __launch_bounds__(kSpThreads, 2) sparse_partial(const SparseParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ unsigned char key_ok[kKeyTile];
  const Shape &sh = prm.sh;
  const SparsePlan &plan = prm.plan;
  const SparseArgs &a = prm.a;
  constexpr int kTileBytes = kKeyTile * D * 2;
  constexpr int kPagesPerTile = kKeyTile / PAGE;
  unsigned char *sQ = smem;
  unsigned char *sK = smem + kRowsPerCta * D * 2;
  unsigned char *sV = sK + kTileBytes;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.z, h = blockIdx.y;
  const int tile = blockIdx.x / plan.rowtiles, rt = blockIdx.x % plan.rowtiles;
  const size_t sh_idx = (size_t)s * sh.Hkv + h;
  const int n = clamp_prefix(a.n_ctx[s], sh.max_pages, PAGE, a.status,
                             tid == 0 && blockIdx.x == 0 && h == 0);
  const int np = (n + PAGE - 1) / PAGE;
  int cnt = a.idx_cnt[sh_idx];
  if (cnt < 0 || cnt > sh.kmax) {
    if (tid == 0 && tile == 0 && rt == 0) raise_status(a.status, kStatusBadIndex);
    cnt = max(0, min(cnt, sh.kmax));
  }
  const int sel_tiles = (cnt * PAGE + kKeyTile - 1) / kKeyTile;
  const int row_base = rt * kRowsPerCta;
  const int warp_row0 = row_base + warp * 16;
  const bool active = warp_row0 < sh.BG;
  const size_t base = (sh_idx * plan.ntiles + tile) * sh.BG;

  const bool is_sel = tile < sel_tiles;
  const int btile = tile - sel_tiles;
  const bool is_blk = !is_sel && btile < plan.blk_tiles;
  if (!is_sel && !is_blk) {  // past this head's keys: an empty partial
    for (int row = row_base + tid; row < min(sh.BG, row_base + kRowsPerCta); row += kSpThreads)
      *reinterpret_cast<float2 *>(a.part_ml + (base + row) * 2) = make_float2(-INFINITY, 0.f);
    return;
  }

  for (int id = tid; id < kRowsPerCta * (D / 8); id += kSpThreads) {
    const int r = id / (D / 8), c = id % (D / 8);
    const int row = row_base + r;
    const bool ok = row < sh.BG;
    const __nv_bfloat16 *src = a.q;
    if (ok) {
      const int b = row / sh.G, g = row % sh.G;
      src = a.q + (((size_t)s * sh.B + b) * sh.Hq + (size_t)h * sh.G + g) * D + c * 8;
    }
    cp_async16(smem_addr(sQ) + SwizzledTile<D>::offset(r, c), src, ok);
  }
  for (int id = tid; id < kKeyTile * (D / 8); id += kSpThreads) {
    const int r = id / (D / 8), c = id % (D / 8);
    bool ok;
    const __nv_bfloat16 *ks = a.k, *vs = a.v;
    if (is_sel) {
      const int e = tile * kPagesPerTile + r / PAGE, slot = r % PAGE;
      ok = e < cnt;
      if (ok) {
        const int lp = a.idx[sh_idx * sh.kmax + e];
        const bool lp_ok = lp >= 0 && lp < np;
        long long phys = -1;
        if (lp_ok)
          phys = sh.page_table ? (long long)sh.page_table[(size_t)s * sh.max_pages + lp]
                               : (long long)s * sh.max_pages + lp;
        if (!lp_ok || phys < 0 || phys >= sh.n_phys) {
          ok = false;
          if (c == 0 && slot == 0) raise_status(a.status, kStatusBadIndex);
        } else {
          ok = lp * PAGE + slot < n;
          const size_t off = (((size_t)phys * sh.Hkv + h) * PAGE + slot) * D + c * 8;
          ks = a.k + off;
          vs = a.v + off;
        }
      }
    } else {
      const int u = btile * kKeyTile + r;
      ok = u < sh.B;
      if (ok) {
        const size_t off = (((size_t)s * sh.B + u) * sh.Hkv + h) * D + c * 8;
        ks = a.blk_k + off;
        vs = a.blk_v + off;
      }
    }
    if (c == 0) key_ok[r] = ok;
    cp_async16(smem_addr(sK) + SwizzledTile<D>::offset(r, c), ks, ok);
    cp_async16(smem_addr(sV) + SwizzledTile<D>::offset(r, c), vs, ok);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  if (!active) return;

  WarpAttn<D> wa;
  wa.init();
  wa.load_q(smem_addr(sQ), warp * 16, lane);
  float acc[WarpAttn<D>::kSNTiles][4];
  wa.scores(smem_addr(sK), acc, lane);
  float m_new[2];
  wa.template softmax_update<0>(acc, sh.sl2, [&](int col) { return key_ok[col] != 0; }, lane,
                                nullptr, m_new);
  wa.pv(smem_addr(sV), acc, lane);
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = warp_row0 + (lane >> 2) + 8 * r;
    if (row >= sh.BG) continue;
    float *dst = a.part_o + (base + row) * D;
#pragma unroll
    for (int i = 0; i < WarpAttn<D>::kONTiles; ++i) {
      const int col = i * 8 + 2 * (lane & 3);
      *reinterpret_cast<float2 *>(dst + col) = make_float2(wa.o[i][2 * r], wa.o[i][2 * r + 1]);
    }
    if ((lane & 3) == 0)
      *reinterpret_cast<float2 *>(a.part_ml + (base + row) * 2) = make_float2(wa.m[r], wa.l[r]);
  }
}

constexpr int kMergeThreads = 256;

template <int D>
__global__ void __launch_bounds__(kMergeThreads) sparse_merge(const SparseParams prm) {
  const Shape &sh = prm.sh;
  const SparsePlan &plan = prm.plan;
  const SparseArgs &a = prm.a;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int s = blockIdx.z, h = blockIdx.y;
  const int row = blockIdx.x * (kMergeThreads / 32) + warp;
  if (row >= sh.BG) return;
  const size_t sh_idx = (size_t)s * sh.Hkv + h;
  float M = -INFINITY;
  for (int t = lane; t < plan.ntiles; t += 32) {
    const float2 ml = *reinterpret_cast<const float2 *>(a.part_ml + ((sh_idx * plan.ntiles + t) * sh.BG + row) * 2);
    if (ml.y > 0.f) M = fmaxf(M, ml.x);
  }
  M = warp_max(M);
  constexpr int kPer = D / 32;
  float acc[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
  float L = 0.f;
  for (int t = 0; t < plan.ntiles; ++t) {
    const size_t r = (sh_idx * plan.ntiles + t) * sh.BG + row;
    const float2 ml = *reinterpret_cast<const float2 *>(a.part_ml + r * 2);
    if (!(ml.y > 0.f)) continue;
    const float w = exp2f(ml.x - M);
    L += w * ml.y;
    const float *src = a.part_o + r * D + lane * kPer;
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] += w * src[i];
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const int b = row / sh.G, g = row % sh.G;
  __nv_bfloat16 *dst = a.o_out + (((size_t)s * sh.B + b) * sh.Hq + (size_t)h * sh.G + g) * D + lane * kPer;
#pragma unroll
  for (int i = 0; i < kPer; i += 2)
    *reinterpret_cast<__nv_bfloat162 *>(dst + i) = __floats2bfloat162_rn(acc[i] * inv, acc[i + 1] * inv);
}

template <int D, int PAGE>
cudaError_t launch_typed(const Shape &sh, const SparsePlan &plan, const SparseArgs &a,
                         cudaStream_t stream) {
  SparseParams prm{sh, plan, a};
  const size_t smem = (size_t)kRowsPerCta * D * 2 + 2 * (size_t)kKeyTile * D * 2;
  auto kern = sparse_partial<D, PAGE>;
  cudaError_t err = set_smem_once(kern, smem);
  if (err != cudaSuccess) return err;
  kern<<<dim3(plan.ntiles * plan.rowtiles, sh.Hkv, sh.S), kSpThreads, smem, stream>>>(prm);
  const int rows_per_cta = kMergeThreads / 32;
  sparse_merge<D><<<dim3((sh.BG + rows_per_cta - 1) / rows_per_cta, sh.Hkv, sh.S), kMergeThreads, 0,
                    stream>>>(prm);
  return cudaGetLastError();
}

}  // namespace

SparsePlan plan_sparse(const Shape &sh, int /*num_sms*/) {
  SparsePlan p{};
  p.rowtiles = (sh.BG + kRowsPerCta - 1) / kRowsPerCta;
  p.sel_tiles = (int)(((long long)sh.kmax * sh.P + kKeyTile - 1) / kKeyTile);
  p.blk_tiles = (sh.B + kKeyTile - 1) / kKeyTile;
  p.ntiles = p.sel_tiles + p.blk_tiles;
  auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = 4096;
  const size_t shn = (size_t)sh.S * sh.Hkv;
  p.off_part_o = off;  off = align(off + shn * p.ntiles * sh.BG * sh.d * 4);
  p.off_part_ml = off; off = align(off + shn * p.ntiles * sh.BG * 2 * 4);
  p.total = off;
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
