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

#include "launch.h"
#include "sm100.cuh"
#include "tc_attn.cuh"

namespace dsa {
namespace {

constexpr int kRowsPerCta = 128;  // query rows per CTA (one M=128 MMA tile)

struct PartialParams {
  Shape sh;
  SelectPlan plan;
  SelectArgs a;
};

// ---------------------------------------------------------------------------
// select_partial: tcgen05 split-KV attention (tc_attn.cuh engine) over the
// split's contiguous 64-token tiles of the prefix, loaded page by page through
// the page table.  After each tile the softmax threads record, per (page, row),
// the tile's probability mass relative to the row's reference max (pagepart)
// and that max (mtile); the split's unnormalised O row, m and l go to part_o /
// part_ml.
// ---------------------------------------------------------------------------
constexpr int kSelStages = 4;

template <int D, int PAGE>
struct SelectPolicy {
  const Shape *sh;
  const SelectPlan *plan;
  const SelectArgs *a;
  const CUtensorMap *kmap, *vmap;
  int s, h, n, np, t_begin, row_base;
  size_t sh_idx;
  float sl2;

  __device__ __forceinline__ long long phys_of(int lp) const {
    if (lp >= np) return -1;
    const long long p = sh->page_table ? (long long)sh->page_table[(size_t)s * sh->max_pages + lp]
                                       : (long long)s * sh->max_pages + lp;
    return (p >= 0 && p < sh->n_phys) ? p : -1;
  }
  __device__ __forceinline__ void prefetch() const {
    sm100::tma_prefetch_map(kmap);
    sm100::tma_prefetch_map(vmap);
  }
  __device__ __forceinline__ void load_tile(int k, uint32_t sk, uint32_t sv, uint32_t half_bytes,
                                            uint32_t bar) const {
    constexpr int kPages = tc::kBN / PAGE;
    const int lp0 = (t_begin + k) * tc::kBN / PAGE;
    long long phys[kPages];
    uint32_t nvalid = 0;
#pragma unroll
    for (int pi = 0; pi < kPages; ++pi) {
      phys[pi] = phys_of(lp0 + pi);
      if (phys[pi] >= 0) ++nvalid;
      else if (lp0 + pi < np && blockIdx.x == 0) raise_status(a->status, kStatusBadIndex);
    }
    sm100::mbar_arrive_expect_tx(bar, nvalid * PAGE * 128u * (D / 64) * 2u);
#pragma unroll
    for (int pi = 0; pi < kPages; ++pi) {
      if (phys[pi] < 0) continue;
      const int y = (int)((phys[pi] * sh->Hkv + h) * PAGE);
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf) {
        sm100::tma_load_2d(sk + hf * half_bytes + pi * PAGE * 128, kmap, bar, hf * 64, y);
        sm100::tma_load_2d(sv + hf * half_bytes + pi * PAGE * 128, vmap, bar, hf * 64, y);
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
    const int t0 = (t_begin + k) * tc::kBN;
    uint64_t m = 0;
#pragma unroll
    for (int pi = 0; pi < tc::kBN / PAGE; ++pi) {
      if (phys_of(t0 / PAGE + pi) < 0) continue;
      const int lo = t0 + pi * PAGE;
      const int cnt = min(PAGE, n - lo);
      if (cnt > 0) m |= ((cnt >= 64) ? ~0ull : ((1ull << cnt) - 1ull)) << (pi * PAGE);
    }
    return m;
  }
  __device__ __forceinline__ void after_tile(int k, int r, float m_used, const float *psum) const {
    const int row = row_base + r;
    if (row >= sh->BG) return;
    const int tile = t_begin + k;
    a->mtile[(sh_idx * plan->max_tiles + tile) * sh->BG + row] = m_used;
#pragma unroll
    for (int pi = 0; pi < tc::kBN / PAGE; ++pi) {
      const int lp = tile * tc::kBN / PAGE + pi;
      if (lp < np) a->pagepart[(sh_idx * sh->max_pages + lp) * sh->BG + row] = psum[pi];
    }
  }
};

template <int D, int PAGE>
__global__ void __launch_bounds__(tc::kThreads, 1)
    select_partial(const PartialParams pp, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap) {
  extern __shared__ unsigned char smem_raw[];
  const Shape &sh = pp.sh;
  const SelectPlan &plan = pp.plan;
  const SelectArgs &a = pp.a;
  const int s = blockIdx.z, h = blockIdx.y;
  const int split = blockIdx.x / plan.rowtiles, rt = blockIdx.x % plan.rowtiles;
  const int n = clamp_prefix(a.n_ctx[s], sh.max_pages, PAGE, a.status,
                             threadIdx.x == 0 && blockIdx.x == 0);
  const int ntiles = (n + tc::kBN - 1) / tc::kBN;
  const int t_begin = split * plan.tiles_per_split;
  const int num_tiles = max(0, min(ntiles, t_begin + plan.tiles_per_split) - t_begin);

  tc::Engine<D, kSelStages> eng;
  eng.init(smem_raw, a.status);
  SelectPolicy<D, PAGE> pol{&sh, &plan, &a, &kmap, &vmap, s, h, n, (n + PAGE - 1) / PAGE,
                            t_begin, rt * kRowsPerCta, (size_t)s * sh.Hkv + h, sh.sl2};
  float m, l;
  const bool alive = eng.template run<PAGE>(pol, num_tiles, m, l);
  if (eng.warp >= 2) {
    const int row = rt * kRowsPerCta + eng.row_in_tile();
    const bool row_ok = row < sh.BG;
    const size_t prow = ((pol.sh_idx * plan.splits + split) * sh.BG + row);
    if (alive) {
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        eng.load_o(c0, o);
        if (row_ok) {
          float4 *dst = reinterpret_cast<float4 *>(a.part_o + prow * D + c0);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                 __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
        }
      }
    }
    if (row_ok)
      *reinterpret_cast<float2 *>(a.part_ml + prow * 2) =
          alive ? make_float2(m, l) : make_float2(-INFINITY, 0.f);
  }
  eng.teardown();
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
        const int tile = lp * PAGE / tc::kBN;
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
  CUtensorMap kmap, vmap;
  const long long rows = sh.n_phys * sh.Hkv * PAGE;
  cudaError_t err = make_kv_tensor_map(&kmap, a.k, rows, D, PAGE);
  if (err != cudaSuccess) return err;
  err = make_kv_tensor_map(&vmap, a.v, rows, D, PAGE);
  if (err != cudaSuccess) return err;
  constexpr auto kern = select_partial<D, PAGE>;
  constexpr size_t smem = tc::Layout<D, kSelStages>::kAlloc;
  err = set_smem_once<kern>(smem);
  if (err != cudaSuccess) return err;
  dim3 grid(plan.splits * plan.rowtiles, sh.Hkv, sh.S);
  kern<<<grid, tc::kThreads, smem, stream>>>(pp, kmap, vmap);
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
  p.max_tiles = (int)(((long long)sh.max_pages * sh.P + tc::kBN - 1) / tc::kBN);
  const long long base = (long long)sh.S * sh.Hkv * p.rowtiles;
  const long long target = num_sms;  // one resident CTA per SM
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
