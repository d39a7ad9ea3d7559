// select.cu -- selection pass: exact attention of the block's step-1 queries
// over the whole prefix, reduced to page scores and cut to a top-k page set per
// KV head ("MAGE: All-[MASK] Block Already Knows Where to Look in Block
// Diffusion LLM", Approach).
//
// Three launches on the caller's stream:
//   1. select_partial: split-KV attention.  CTA = (split, row tile) x KV head x
//      sequence; 8 warps x 16 rows = 128 query rows (b, g) of one KV head against
//      the split's 64-token tiles, double-buffered with cp.async.  Per split it
//      writes the unnormalised output O_j with its row max m_j and sum l_j, and
//      per (page, row) the partial probability mass of the page relative to the
//      running max at that tile (pagepart), together with that max (mtile).
//   2. select_finalize: merges the splits into o_out and turns the partial
//      masses into page scores  S_h[q] = (1/BG) sum_rows pagepart * 2^(mtile-M) / L.
//   3. select_topk: radix select of the kp-th largest score per (seq, KV head),
//      ties broken towards the lower page index, emitted in ascending order.
#include <algorithm>

#include "attn_core.cuh"
#include "launch.h"

namespace dsa {
namespace {

constexpr int kSelThreads = 256;  // 8 warps
constexpr int kRowsPerCta = 128;

struct PartialParams {
  Shape sh;
  SelectPlan plan;
  SelectArgs a;
};

template <int D, int PAGE>
__global__ void __launch_bounds__(kSelThreads, 2) select_partial(const PartialParams pp) {
  extern __shared__ __align__(128) unsigned char smem[];
  const Shape &sh = pp.sh;
  const SelectPlan &plan = pp.plan;
  const SelectArgs &a = pp.a;
  constexpr int kTileBytes = kKeyTile * D * 2;
  unsigned char *sQ = smem;
  unsigned char *sKV = smem + kRowsPerCta * D * 2;  // [stage][K|V] tiles

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.z, h = blockIdx.y;
  const int split = blockIdx.x / plan.rowtiles, rt = blockIdx.x % plan.rowtiles;
  const int n = clamp_prefix(a.n_ctx[s], sh.max_pages, PAGE, a.status,
                             tid == 0 && blockIdx.x == 0);
  const int np = (n + PAGE - 1) / PAGE;
  const int ntiles = (n + kKeyTile - 1) / kKeyTile;
  const int t_begin = split * plan.tiles_per_split;
  const int t_end = min(ntiles, t_begin + plan.tiles_per_split);
  const int row_base = rt * kRowsPerCta;
  const int warp_row0 = row_base + warp * 16;
  const bool active = warp_row0 < sh.BG;
  const size_t sh_idx = (size_t)s * sh.Hkv + h;

  // queries of this row tile: row r -> (b = r / G, g = r % G), head h*G + g
  for (int id = tid; id < kRowsPerCta * (D / 8); id += kSelThreads) {
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
  cp_async_commit();

  auto load_tile = [&](int tile, int stage) {
    unsigned char *sK = sKV + stage * 2 * kTileBytes;
    unsigned char *sV = sK + kTileBytes;
    for (int id = tid; id < kKeyTile * (D / 8); id += kSelThreads) {
      const int r = id / (D / 8), c = id % (D / 8);
      const int t = tile * kKeyTile + r;
      bool ok = t < n;
      const __nv_bfloat16 *ks = a.k, *vs = a.v;
      if (ok) {
        const int lp = t / PAGE, slot = t % PAGE;
        const long long phys = sh.page_table ? (long long)sh.page_table[(size_t)s * sh.max_pages + lp]
                                             : (long long)s * sh.max_pages + lp;
        if (phys < 0 || phys >= sh.n_phys) {
          ok = false;
          if (c == 0 && slot == 0) raise_status(a.status, kStatusBadIndex);
        } else {
          const size_t off = (((size_t)phys * sh.Hkv + h) * PAGE + slot) * D + c * 8;
          ks = a.k + off;
          vs = a.v + off;
        }
      }
      cp_async16(smem_addr(sK) + SwizzledTile<D>::offset(r, c), ks, ok);
      cp_async16(smem_addr(sV) + SwizzledTile<D>::offset(r, c), vs, ok);
    }
    cp_async_commit();
  };

  WarpAttn<D> wa;
  wa.init();
  if (t_begin < t_end) load_tile(t_begin, 0);
  for (int tile = t_begin; tile < t_end; ++tile) {
    const int stage = (tile - t_begin) & 1;
    if (tile + 1 < t_end) {
      load_tile(tile + 1, stage ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (tile == t_begin && active) wa.load_q(smem_addr(sQ), warp * 16, lane);
    if (active) {
      const uint32_t sK = smem_addr(sKV + stage * 2 * kTileBytes);
      const uint32_t sV = sK + kTileBytes;
      float acc[WarpAttn<D>::kSNTiles][4];
      wa.scores(sK, acc, lane);
      const int t0 = tile * kKeyTile;
      float page_sum[kKeyTile / PAGE][2];
      float m_new[2];
      wa.template softmax_update<PAGE>(acc, sh.sl2, [&](int col) { return t0 + col < n; }, lane,
                                       page_sum, m_new);
      if ((lane & 3) == 0) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int row = warp_row0 + (lane >> 2) + 8 * r;
          if (row < sh.BG) {
            a.mtile[(sh_idx * plan.max_tiles + tile) * sh.BG + row] = m_new[r];
#pragma unroll
            for (int pi = 0; pi < kKeyTile / PAGE; ++pi) {
              const int lp = t0 / PAGE + pi;
              if (lp < np) a.pagepart[(sh_idx * sh.max_pages + lp) * sh.BG + row] = page_sum[pi][r];
            }
          }
        }
      }
      wa.pv(sV, acc, lane);
    }
    __syncthreads();
  }
  if (t_begin >= t_end) cp_async_wait<0>();

  // split partials (unnormalised O, m, l) of the warp's rows
  if (active) {
    const size_t base = (sh_idx * plan.splits + split) * sh.BG;
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
}

constexpr int kFinThreads = 256;
constexpr int kPagesPerFinCta = 64;
constexpr int kRowsPerFinCta = 8;

// Row max M and 1/L over the splits, into shared memory.
__device__ void merged_row_stats(const Shape &sh, const SelectPlan &plan, const float *part_ml,
                                 size_t sh_idx, float *sM, float *sLinv) {
  for (int row = threadIdx.x; row < sh.BG; row += blockDim.x) {
    float M = -INFINITY;
    for (int j = 0; j < plan.splits; ++j) {
      const float2 ml = *reinterpret_cast<const float2 *>(
          part_ml + ((sh_idx * plan.splits + j) * sh.BG + row) * 2);
      if (ml.y > 0.f) M = fmaxf(M, ml.x);
    }
    float L = 0.f;
    for (int j = 0; j < plan.splits; ++j) {
      const float2 ml = *reinterpret_cast<const float2 *>(
          part_ml + ((sh_idx * plan.splits + j) * sh.BG + row) * 2);
      if (ml.y > 0.f) L += ml.y * exp2f(ml.x - M);
    }
    sM[row] = M;
    sLinv[row] = L > 0.f ? 1.f / L : 0.f;
  }
}

template <int D, int PAGE>
__global__ void __launch_bounds__(kFinThreads) select_finalize(const PartialParams pp) {
  __shared__ float sM[256], sLinv[256];
  const Shape &sh = pp.sh;
  const SelectPlan &plan = pp.plan;
  const SelectArgs &a = pp.a;
  const int s = blockIdx.z, h = blockIdx.y;
  const size_t sh_idx = (size_t)s * sh.Hkv + h;
  const int n = clamp_prefix(a.n_ctx[s], sh.max_pages, PAGE, a.status, false);
  const int np = (n + PAGE - 1) / PAGE;
  merged_row_stats(sh, plan, a.part_ml, sh_idx, sM, sLinv);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int score_ctas = (sh.max_pages + kPagesPerFinCta - 1) / kPagesPerFinCta;
  if ((int)blockIdx.x < score_ctas) {
    const float inv_bg = 1.f / (float)sh.BG;
    for (int k = warp; k < kPagesPerFinCta; k += kFinThreads / 32) {
      const int lp = blockIdx.x * kPagesPerFinCta + k;
      if (lp >= sh.max_pages) break;
      float acc = 0.f;
      if (lp < np) {
        const int tile = lp * PAGE / kKeyTile;
        const float *part = a.pagepart + (sh_idx * sh.max_pages + lp) * sh.BG;
        const float *mt = a.mtile + (sh_idx * plan.max_tiles + tile) * sh.BG;
        for (int row = lane; row < sh.BG; row += 32)
          acc += part[row] * exp2f(mt[row] - sM[row]) * sLinv[row];
        acc = warp_sum(acc) * inv_bg;
      }
      if (lane == 0) a.scores[sh_idx * sh.max_pages + lp] = acc;
    }
  } else {
    const int row = (blockIdx.x - score_ctas) * kRowsPerFinCta + warp;
    if (row >= sh.BG) return;
    const int b = row / sh.G, g = row % sh.G;
    constexpr int kPer = D / 32;
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
    for (int j = 0; j < plan.splits; ++j) {
      const size_t r = (sh_idx * plan.splits + j) * sh.BG + row;
      const float2 ml = *reinterpret_cast<const float2 *>(a.part_ml + r * 2);
      if (!(ml.y > 0.f)) continue;
      const float w = exp2f(ml.x - sM[row]);
      const float *src = a.part_o + r * D + lane * kPer;
#pragma unroll
      for (int i = 0; i < kPer; ++i) acc[i] += w * src[i];
    }
    __nv_bfloat16 *dst = a.o_out + (((size_t)s * sh.B + b) * sh.Hq + (size_t)h * sh.G + g) * D + lane * kPer;
#pragma unroll
    for (int i = 0; i < kPer; i += 2)
      *reinterpret_cast<__nv_bfloat162 *>(dst + i) =
          __floats2bfloat162_rn(acc[i] * sLinv[row], acc[i + 1] * sLinv[row]);
  }
}

constexpr int kTopkThreads = 1024;

// Order-preserving key of a non-negative score (-0 folded onto +0).
__device__ __forceinline__ uint32_t score_key(float v) {
  return v > 0.f ? __float_as_uint(v) : 0u;
}

__global__ void __launch_bounds__(kTopkThreads) select_topk(const PartialParams pp) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_digit, s_remaining;
  __shared__ uint32_t scan_eq[kTopkThreads / 32], scan_sel[kTopkThreads / 32];
  __shared__ int s_bad;
  const Shape &sh = pp.sh;
  const SelectArgs &a = pp.a;
  const int s = blockIdx.y, h = blockIdx.x;
  const size_t sh_idx = (size_t)s * sh.Hkv + h;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = clamp_prefix(a.n_ctx[s], sh.max_pages, sh.P, a.status, false);
  const int np = (n + sh.P - 1) / sh.P;
  int kp = a.topk[s] / sh.P;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  if (kp > sh.kmax || kp < 0 || a.topk[s] % sh.P != 0) {
    if (tid == 0) raise_status(a.status, kStatusBadIndex);
    kp = max(0, min(kp, sh.kmax));
  }
  const float *sc = a.scores + sh_idx * sh.max_pages;
  int32_t *out = a.idx_out + sh_idx * sh.kmax;
  const int take = min(kp, np);

  // non-finite scores are reported (they come from non-finite inputs)
  for (int i = tid; i < np; i += kTopkThreads)
    if (!isfinite(sc[i])) s_bad = 1;
  __syncthreads();
  if (s_bad && tid == 0) raise_status(a.status, kStatusNonfinite);

  if (take >= np) {  // the budget covers the prefix: every page
    for (int i = tid; i < sh.kmax; i += kTopkThreads) out[i] = i < np ? i : -1;
    if (tid == 0) a.cnt_out[sh_idx] = np;
    return;
  }
  // radix select of the take-th largest key, 8 bits at a time from the top
  uint32_t prefix = 0, mask = 0;
  if (tid == 0) s_remaining = (uint32_t)take;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < np; i += kTopkThreads) {
      const uint32_t key = score_key(sc[i]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t cum = 0, rem = s_remaining;
      int dgt = 255;
      for (; dgt > 0; --dgt) {
        if (cum + hist[dgt] >= rem) break;
        cum += hist[dgt];
      }
      s_digit = (uint32_t)dgt;
      s_remaining = rem - cum;
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t thr = prefix;           // value of the take-th largest key
  const uint32_t need_eq = s_remaining;  // keys equal to thr to keep, lowest pages first

  // ordered compaction: contiguous chunk per thread, block-wide exclusive scans
  const int chunk = (np + kTopkThreads - 1) / kTopkThreads;
  const int i0 = min(np, tid * chunk), i1 = min(np, i0 + chunk);
  uint32_t n_eq = 0, n_gt = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = score_key(sc[i]);
    n_gt += key > thr;
    n_eq += key == thr;
  }
  // warp-inclusive scans of (n_eq, n_gt)
  uint32_t e = n_eq, g = n_gt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t e2 = __shfl_up_sync(0xffffffffu, e, o), g2 = __shfl_up_sync(0xffffffffu, g, o);
    if (lane >= o) { e += e2; g += g2; }
  }
  if (lane == 31) { scan_eq[warp] = e; scan_sel[warp] = g; }
  __syncthreads();
  if (warp == 0) {
    uint32_t we = scan_eq[lane], wg = scan_sel[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t e2 = __shfl_up_sync(0xffffffffu, we, o), g2 = __shfl_up_sync(0xffffffffu, wg, o);
      if (lane >= o) { we += e2; wg += g2; }
    }
    scan_eq[lane] = we;
    scan_sel[lane] = wg;
  }
  __syncthreads();
  uint32_t eq_before = e - n_eq + (warp > 0 ? scan_eq[warp - 1] : 0u);
  uint32_t gt_before = g - n_gt + (warp > 0 ? scan_sel[warp - 1] : 0u);
  // position = selected pages before i = (greater before) + min(equal before, need_eq)
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = score_key(sc[i]);
    if (key > thr) {
      out[gt_before + min(eq_before, need_eq)] = i;
      ++gt_before;
    } else if (key == thr) {
      if (eq_before < need_eq) out[gt_before + eq_before] = i;
      ++eq_before;
    }
  }
  for (int i = take + tid; i < sh.kmax; i += kTopkThreads) out[i] = -1;
  if (tid == 0) a.cnt_out[sh_idx] = take;
}

template <int D, int PAGE>
cudaError_t launch_typed(const Shape &sh, const SelectPlan &plan, const SelectArgs &a,
                         cudaStream_t stream) {
  PartialParams pp{sh, plan, a};
  const size_t smem = (size_t)kRowsPerCta * D * 2 + 2 * 2 * (size_t)kKeyTile * D * 2;
  auto kern = select_partial<D, PAGE>;
  cudaError_t err = set_smem_once(kern, smem);
  if (err != cudaSuccess) return err;
  dim3 grid(plan.splits * plan.rowtiles, sh.Hkv, sh.S);
  kern<<<grid, kSelThreads, smem, stream>>>(pp);
  const int score_ctas = (sh.max_pages + kPagesPerFinCta - 1) / kPagesPerFinCta;
  const int o_ctas = (sh.BG + kRowsPerFinCta - 1) / kRowsPerFinCta;
  select_finalize<D, PAGE><<<dim3(score_ctas + o_ctas, sh.Hkv, sh.S), kFinThreads, 0, stream>>>(pp);
  select_topk<<<dim3(sh.Hkv, sh.S), kTopkThreads, 0, stream>>>(pp);
  return cudaGetLastError();
}

}  // namespace

SelectPlan plan_select(const Shape &sh, int num_sms) {
  SelectPlan p{};
  p.rowtiles = (sh.BG + kRowsPerCta - 1) / kRowsPerCta;
  p.max_tiles = (int)(((long long)sh.max_pages * sh.P + kKeyTile - 1) / kKeyTile);
  const long long base = (long long)sh.S * sh.Hkv * p.rowtiles;
  const long long target = 2LL * num_sms;  // two resident CTAs per SM
  int splits = (int)std::max(1LL, (target + base - 1) / base);
  splits = std::min(splits, p.max_tiles);
  p.tiles_per_split = (p.max_tiles + splits - 1) / splits;
  p.splits = (p.max_tiles + p.tiles_per_split - 1) / p.tiles_per_split;
  auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = 4096;  // status word and counters
  const size_t shn = (size_t)sh.S * sh.Hkv;
  p.off_part_o = off;   off = align(off + shn * p.splits * sh.BG * sh.d * 4);
  p.off_part_ml = off;  off = align(off + shn * p.splits * sh.BG * 2 * 4);
  p.off_pagepart = off; off = align(off + shn * sh.max_pages * sh.BG * 4);
  p.off_mtile = off;    off = align(off + shn * p.max_tiles * sh.BG * 4);
  p.off_scores = off;   off = align(off + shn * sh.max_pages * 4);
  p.total = off;
  return p;
}

cudaError_t launch_select(const Shape &sh, const SelectPlan &plan, const SelectArgs &a,
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
