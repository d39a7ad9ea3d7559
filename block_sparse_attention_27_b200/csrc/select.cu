// select.cu -- selection pass: exact attention of the block's step-1 queries
// over the whole prefix, reduced to page scores and cut to a top-k page set per
// KV head ("MAGE: All-[MASK] Block Already Knows Where to Look in Block
// Diffusion LLM", Approach).
//
// Three launches on the caller's stream, each a programmatic dependent of the
// one before it:
//   1. select_partial: split-KV attention on the tcgen05 engine (tc_attn.cuh).
//      CTA = (split, 128-row tile) x KV head x sequence, one wave over the SMs;
//      the split's 64-token tiles stream through a TMA ring.  Per split it
//      writes the unnormalised output O_j with its row max m_j and sum l_j, and
//      per (tile, row) the partial probability mass of each unit of the tile
//      (min(page, 32) keys of one page) relative to the row's reference max at
//      that tile (pagepart, [tile][row][unit]), together with that max (mtile).
//   2. select_finalize: merges the splits into o_out and turns the partial
//      masses into page scores  S_h[q] = (1/BG) sum_rows pagepart * 2^(mtile-M) / L.
//   3. select_topk: radix select of the kp-th largest score per (seq, KV head),
//      ties broken towards the lower page index, emitted in ascending order.
#include <algorithm>
#include <cstring>
#include <type_traits>

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
constexpr int kSelStages = 5;

template <int D, int PAGE>
struct SelectPolicy {
  // everything the hot loops touch is held by value (registers), with base
  // pointers already offset to this (sequence, KV head)
  static constexpr bool kIssueBeforeSync = true;  // tile addresses need no table
  const CUtensorMap *kmap, *vmap;    // one page per box
  const CUtensorMap *kmap4, *vmap4;  // 64/PAGE consecutive pages per box
  const int32_t *page_row;          // page-table row of the sequence, or null (identity)
  const __nv_bfloat16 *q_head;      // q[s, 0, h*G, 0]
  float *mtile_head;                // mtile[s, h, 0, 0]
  float *pagepart_head;             // pagepart[s, h, 0, 0, 0]
  uint32_t *status;
  long long n_phys, phys0;          // phys0 = s*max_pages (identity map)
  int Hkv, h, G, Hq, BG, n, np, t_begin, row_base;
  float sl2;

  __device__ __forceinline__ long long phys_of(int lp) const {
    if (lp >= np) return -1;
    const long long p = page_row ? (long long)page_row[lp] : phys0 + lp;
    return (p >= 0 && p < n_phys) ? p : -1;
  }
  __device__ __forceinline__ void prepare(unsigned char *) const {}
  __device__ __forceinline__ void ready() const {}
  __device__ __forceinline__ void prefetch() const {
    sm100::tma_prefetch_map(kmap);
    sm100::tma_prefetch_map(vmap);
    sm100::tma_prefetch_map(kmap4);
    sm100::tma_prefetch_map(vmap4);
  }
  // Run by all 32 lanes of warp 0: lanes 0..kPages-1 resolve one page each,
  // lane 0 arms the barrier, then each box of the tile is issued by a lane of
  // its own (one warp instruction for the tile).
  __device__ __forceinline__ void load_tile(int k, uint32_t sk, uint32_t sv, uint32_t half_bytes,
                                            uint32_t bar, int lane) const {
    constexpr int kPages = tc::kBN / PAGE;
    constexpr int kHalves = D / 64;
    const int lp0 = (t_begin + k) * tc::kBN / PAGE;
    const long long my = phys_of(lp0 + (lane < kPages ? lane : 0));
    const bool valid = lane < kPages && my >= 0;
    if (lane < kPages && my < 0 && lp0 + lane < np && blockIdx.x == 0)
      raise_status(status, kStatusBadIndex);
    const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
    const long long p0 = __shfl_sync(0xffffffffu, my, 0);
    const bool consec = lane >= kPages || (valid && my == p0 + lane);
    const bool run = kPages > 1 && __all_sync(0xffffffffu, consec);
    if (lane == 0)
      sm100::mbar_arrive_expect_tx(bar, (uint32_t)__popc(vmask) * PAGE * 128u * kHalves * 2u);
    if (run) {  // the whole tile in one box per half and tensor
      if (lane < 2 * kHalves) {
        const int hf = lane % kHalves;
        const bool isv = lane >= kHalves;
        sm100::tma_load_4d((isv ? sv : sk) + hf * half_bytes, isv ? vmap4 : kmap4, bar, hf * 64, 0, h,
                           (int)p0);
      }
      return;
    }
    const int pi = lane / (2 * kHalves), rem = lane % (2 * kHalves);
    const long long ph = __shfl_sync(0xffffffffu, my, pi < kPages ? pi : 0);
    if (pi < kPages && ((vmask >> pi) & 1u)) {
      const int hf = rem % kHalves;
      const bool isv = rem >= kHalves;
      const int y = (int)((ph * Hkv + h) * PAGE);
      sm100::tma_load_2d((isv ? sv : sk) + hf * half_bytes + pi * PAGE * 128, isv ? vmap : kmap, bar,
                         hf * 64, y);
    }
  }
  __device__ __forceinline__ const __nv_bfloat16 *q_row(int r) const {
    const int row = row_base + r;
    if (row >= BG) return nullptr;
    const int b = row / G, g = row % G;
    return q_head + ((size_t)b * Hq + g) * D;
  }
  __device__ __forceinline__ uint64_t key_mask(int k) const {
    const int t0 = (t_begin + k) * tc::kBN;
    if (t0 + tc::kBN <= n && !page_row && phys0 + (t0 + tc::kBN - 1) / PAGE < n_phys)
      return ~0ull;  // a full tile of pages that are all in the cache
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
  // per-unit masses of tile k (a unit is min(PAGE, 32) keys of one page),
  // relative to the row's reference max m_used of the group that ran the tile
  __device__ __forceinline__ void after_tile(int k, int r, float m_used, const float *usum) const {
    using U = tc::Units<PAGE>;
    const int row = row_base + r;
    if (row >= BG) return;
    const int tile = t_begin + k;
    mtile_head[(size_t)tile * BG + row] = m_used;
    // the row's unit masses of the tile, one vector store (units past the prefix hold 0)
    float *dst = pagepart_head + ((size_t)tile * BG + row) * U::kPerTile;
    if constexpr (U::kPerTile == 4)
      *reinterpret_cast<float4 *>(dst) = make_float4(usum[0], usum[1], usum[2], usum[3]);
    else
      *reinterpret_cast<float2 *>(dst) = make_float2(usum[0], usum[1]);
  }
};

template <int D, int PAGE>
__global__ void __launch_bounds__(tc::kThreads, 1)
    select_partial(const __grid_constant__ PartialParams pp, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap kmap4,
                   const __grid_constant__ CUtensorMap vmap4) {
  extern __shared__ unsigned char smem_raw[];
  const Shape &sh = pp.sh;
  const SelectPlan &plan = pp.plan;
  const SelectArgs &a = pp.a;
  const int s = blockIdx.z, h = blockIdx.y;
  const int split = blockIdx.x / plan.rowtiles, rt = blockIdx.x % plan.rowtiles;
  if (threadIdx.x == 0) DSA_TRACE_EVENT(0);
  SelectPolicy<D, PAGE> pol;
  pol.kmap = &kmap;
  pol.vmap = &vmap;
  pol.kmap4 = &kmap4;
  pol.vmap4 = &vmap4;
  tc::Engine<D, kSelStages> eng;
  eng.setup(smem_raw, pol);
  // everything below may read what the kernel ahead of this one wrote
  sm100::grid_dep_wait();
  sm100::grid_dep_launch_dependents();

  const int n = clamp_prefix(a.n_ctx[s], sh.max_pages, PAGE, a.status,
                             threadIdx.x == 0 && blockIdx.x == 0);
  const int ntiles = (n + tc::kBN - 1) / tc::kBN;
  const int t_begin = split * plan.tiles_per_split;
  const int num_tiles = max(0, min(ntiles, t_begin + plan.tiles_per_split) - t_begin);
  const size_t sh_idx = (size_t)s * sh.Hkv + h;
  pol.page_row = sh.page_table ? sh.page_table + (size_t)s * sh.max_pages : nullptr;
  pol.q_head = a.q + ((size_t)s * sh.B * sh.Hq + (size_t)h * sh.G) * D;
  pol.mtile_head = a.mtile + sh_idx * plan.max_tiles * sh.BG;
  pol.pagepart_head = a.pagepart + sh_idx * plan.max_tiles * sh.BG * tc::Units<PAGE>::kPerTile;
  pol.status = a.status;
  pol.n_phys = sh.n_phys;
  pol.phys0 = (long long)s * sh.max_pages;
  pol.Hkv = sh.Hkv;
  pol.h = h;
  pol.G = sh.G;
  pol.Hq = sh.Hq;
  pol.BG = sh.BG;
  pol.n = n;
  pol.np = (n + PAGE - 1) / PAGE;
  pol.t_begin = t_begin;
  pol.row_base = rt * kRowsPerCta;
  pol.sl2 = sh.sl2;
  eng.init(a.status, pol, num_tiles);
  float m, l;
  eng.template run<PAGE>(pol, num_tiles, m, l);
  float m_row, l_row, wa, wb;
  eng.finish(m, l, m_row, l_row, wa, wb);
  if (eng.warp >= 2) {
    // O = wa * O_0 + wb * O_1 relative to m_row; this thread writes its half of the columns
    const int g = eng.group();
    const int row = rt * kRowsPerCta + eng.row_in_tile();
    const bool row_ok = row < sh.BG;
    const size_t prow = ((sh_idx * plan.splits + split) * sh.BG + row);
#pragma unroll
    for (int c0 = g * (D / 2); c0 < (g + 1) * (D / 2); c0 += 32) {
      uint32_t oa[32], ob[32];
      eng.load_o(0, c0, oa);
      eng.load_o(1, c0, ob);
      if (row_ok && l_row > 0.f) {
        float4 *dst = reinterpret_cast<float4 *>(a.part_o + prow * D + c0);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float v[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = wa > 0.f ? wa * __uint_as_float(oa[4 * i + e]) : 0.f;
            const float x1 = wb > 0.f ? wb * __uint_as_float(ob[4 * i + e]) : 0.f;
            v[e] = x0 + x1;
          }
          dst[i] = make_float4(v[0], v[1], v[2], v[3]);
        }
      }
    }
    if (row_ok && g == 0)
      *reinterpret_cast<float2 *>(a.part_ml + prow * 2) =
          l_row > 0.f ? make_float2(m_row, l_row) : make_float2(-INFINITY, 0.f);
    if (row == rt * kRowsPerCta) DSA_TRACE_EVENT(7);
  }
  eng.teardown();
  if (threadIdx.x == 0) DSA_TRACE_EVENT(11);
}

// ---------------------------------------------------------------------------
// select_finalize: merges the splits.  Every CTA first forms, for each query
// row, the global reference M = max_j m_j and 1/L with L = sum_j l_j 2^(m_j - M)
// (one online pass over the splits).  Score CTAs then turn the partial masses of
// their pages into  S_h[q] = (1/BG) sum_rows pagepart * 2^(mtile - M) / L;
// output CTAs write o_out = sum_j 2^(m_j - M) O_j / L in bf16.
// ---------------------------------------------------------------------------
constexpr int kFinThreads = 256;
constexpr int kRowsPerFinCta = 8;   // output CTAs: one query row per warp
constexpr int kFinBatch = 16;       // output CTAs: split partials a lane loads at once

// Folds a partial (m, l) into the running (M, L) of a row (log2 domain); an
// empty partial (l = 0) leaves it unchanged.
__device__ __forceinline__ void merge_ml(float &M, float &L, float m, float l) {
  if (!(l > 0.f)) return;
  if (m > M) {
    L = L * exp2f(M - m) + l;
    M = m;
  } else {
    L += l * exp2f(m - M);
  }
}

// sM[row] = M and sLinv[row] = 1/L over all splits.  Each row gets tpr = the
// largest power of two <= blockDim.x / BG (at most 32) threads of one warp; each
// of them loads its splits 8 at a time (all in flight together), then the tpr
// partial results are combined with shuffles.
__device__ __forceinline__ void merged_row_stats(const Shape &sh, const SelectPlan &plan,
                                                 const float *part_ml, size_t sh_idx, float *sM,
                                                 float *sLinv) {
  int tpr = 1;
  while (tpr < 32 && 2 * tpr * sh.BG <= (int)blockDim.x) tpr *= 2;
  const int sub = threadIdx.x % tpr;
  const int per_pass = (int)blockDim.x / tpr;
  const float2 *ml = reinterpret_cast<const float2 *>(part_ml) + sh_idx * plan.splits * sh.BG;
  // every thread runs the same passes (the shuffles need whole warps)
  for (int row0 = 0; row0 < sh.BG; row0 += per_pass) {
    const int row = row0 + (int)threadIdx.x / tpr;
    const bool valid = row < sh.BG;
    float M = -INFINITY, L = 0.f;
    for (int j0 = sub; j0 < plan.splits; j0 += 8 * tpr) {
      float2 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * tpr;
        v[u] = (valid && j < plan.splits) ? ml[(size_t)j * sh.BG + row] : make_float2(-INFINITY, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) merge_ml(M, L, v[u].x, v[u].y);
    }
    for (int o = tpr / 2; o > 0; o >>= 1) {
      const float M2 = __shfl_xor_sync(0xffffffffu, M, o);
      const float L2 = __shfl_xor_sync(0xffffffffu, L, o);
      merge_ml(M, L, M2, L2);
    }
    if (valid && sub == 0) {
      sM[row] = M;
      sLinv[row] = L > 0.f ? 1.f / L : 0.f;
    }
  }
}

// Sum over the 32 lanes of a warp of the kP values v[0..kP) (kP = 1, 2 or 4)
// with log2(32) + kP - 1 shuffles: the first rounds halve the set of values a
// lane carries.  Value p ends in lane p * (32 / kP).
template <int kP>
__device__ __forceinline__ float warp_sum_multi(const float (&v)[kP], int lane) {
  if constexpr (kP == 4) {
    const bool hi = lane & 16;
    const float s0 = hi ? v[0] : v[2], s1 = hi ? v[1] : v[3];
    const float b0 = (hi ? v[2] : v[0]) + __shfl_xor_sync(0xffffffffu, s0, 16);
    const float b1 = (hi ? v[3] : v[1]) + __shfl_xor_sync(0xffffffffu, s1, 16);
    const bool h8 = lane & 8;
    float c = (h8 ? b1 : b0) + __shfl_xor_sync(0xffffffffu, h8 ? b0 : b1, 8);
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    return c;
  } else if constexpr (kP == 2) {
    const bool hi = lane & 16;
    float c = (hi ? v[1] : v[0]) + __shfl_xor_sync(0xffffffffu, hi ? v[0] : v[1], 16);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    return c;
  } else {
    return warp_sum(v[0]);
  }
}

// Page scores of the pages [p0, p1) (tile-aligned) of one (sequence, KV head).
// Lane i of a warp handles the rows VEC*i + 32*VEC*c + e (c < kChunks, e < VEC):
// their M and 1/L stay in registers, and for kFinTiles tiles at a time the
// tile maxima and each row's vector of unit masses are loaded before any of
// them is used.
template <int PAGE, int VEC, int kChunks, int kFinTiles>
__device__ __forceinline__ void page_scores(const Shape &sh, const SelectPlan &plan,
                                            const SelectArgs &a, size_t sh_idx, int np, int p0,
                                            int p1, float *sM, float *sLinv) {
  using U = tc::Units<PAGE>;
  using V = typename std::conditional<VEC == 4, float4, float>::type;
  constexpr int kPagesPerTile = tc::kBN / PAGE;
  constexpr int kUnits = U::kPerTile;  // 4 or 2
  using W = typename std::conditional<kUnits == 4, float4, float2>::type;
  static_assert(kUnits == 4 || kUnits == 2, "units per tile");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int BG = sh.BG;
  auto lanes = [](const V &v, int e) -> float { return reinterpret_cast<const float *>(&v)[e]; };
  auto units = [](const W &w, int u) -> float { return reinterpret_cast<const float *>(&w)[u]; };
  const float inv_bg = 1.f / (float)BG;
  const int warps = (int)blockDim.x / 32;
  const int stride = warps * kPagesPerTile * kFinTiles;
  const float *mt_head = a.mtile + sh_idx * plan.max_tiles * BG;
  const float *pp_head = a.pagepart + sh_idx * plan.max_tiles * BG * kUnits;
  V mt[kFinTiles][kChunks];
  W part[kFinTiles][kChunks][VEC];
  // every load of the kFinTiles tiles from lp0 on, issued together
  auto load = [&](int lp0) {
#pragma unroll
    for (int t = 0; t < kFinTiles; ++t) {
      const int lpt = lp0 + t * kPagesPerTile;
      const bool live = lpt < min(np, p1);  // tiles past the prefix were never written
      const int tile = lpt * PAGE / tc::kBN;
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        const int row0 = VEC * lane + 32 * VEC * c;
        if (live && row0 < BG) {
          mt[t][c] = *reinterpret_cast<const V *>(mt_head + (size_t)tile * BG + row0);
        } else {
          memset(&mt[t][c], 0, sizeof(V));
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          if (live && row0 + e < BG) {
            part[t][c][e] = *reinterpret_cast<const W *>(pp_head + ((size_t)tile * BG + row0 + e) * kUnits);
          } else {
            memset(&part[t][c][e], 0, sizeof(W));
          }
        }
      }
    }
  };
  int lp0 = p0 + warp * kPagesPerTile * kFinTiles;
  if (lp0 < p1) load(lp0);  // in flight while the row statistics are formed
  merged_row_stats(sh, plan, a.part_ml, sh_idx, sM, sLinv);
  __syncthreads();
  float rm[kChunks][VEC], rl[kChunks][VEC];
#pragma unroll
  for (int c = 0; c < kChunks; ++c)
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const int row = VEC * lane + 32 * VEC * c + e;
      rm[c][e] = row < BG ? sM[row] : 0.f;
      rl[c][e] = row < BG ? sLinv[row] : 0.f;  // 0: the row does not exist
    }
  for (; lp0 < p1; lp0 += stride) {
#pragma unroll
    for (int t = 0; t < kFinTiles; ++t) {
      const int lpt = lp0 + t * kPagesPerTile;
      float acc[kUnits];
#pragma unroll
      for (int u = 0; u < kUnits; ++u) acc[u] = 0.f;
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float f = rl[c][e] > 0.f ? exp2f(lanes(mt[t][c], e) - rm[c][e]) * rl[c][e] : 0.f;
#pragma unroll
          for (int u = 0; u < kUnits; ++u) acc[u] = fmaf(units(part[t][c][e], u), f, acc[u]);
        }
      float pv[kPagesPerTile];
#pragma unroll
      for (int pi = 0; pi < kPagesPerTile; ++pi) {
        pv[pi] = 0.f;
#pragma unroll
        for (int u = pi * U::kPerPage; u < (pi + 1) * U::kPerPage; ++u) pv[pi] += acc[u];
      }
      const float v = warp_sum_multi<kPagesPerTile>(pv, lane) * inv_bg;
      const int pi = lane / (32 / kPagesPerTile);
      if (lane % (32 / kPagesPerTile) == 0 && lpt + pi < p1) a.scores[sh_idx * sh.max_pages + lpt + pi] = v;
    }
    if (lp0 + stride < p1) load(lp0 + stride);
  }
}

template <int D, int PAGE>
__global__ void __launch_bounds__(kFinThreads, 2) select_finalize(const __grid_constant__ PartialParams pp) {
  __shared__ float sM[256], sLinv[256];
  const Shape &sh = pp.sh;
  const SelectPlan &plan = pp.plan;
  const SelectArgs &a = pp.a;
  sm100::grid_dep_wait();  // the partials of select_partial
  sm100::grid_dep_launch_dependents();
  const int s = blockIdx.z, h = blockIdx.y;
  const size_t sh_idx = (size_t)s * sh.Hkv + h;
  const int n = clamp_prefix(a.n_ctx[s], sh.max_pages, PAGE, a.status, false);
  const int np = (n + PAGE - 1) / PAGE;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int score_ctas = (sh.max_pages + plan.fin_pages - 1) / plan.fin_pages;
  if ((int)blockIdx.x < score_ctas) {  // (page_scores forms the row statistics itself)
    const int p0 = blockIdx.x * plan.fin_pages;  // a multiple of 64 tokens
    const int p1 = min(sh.max_pages, p0 + plan.fin_pages);
    // (kFinTiles: 64-token tiles whose loads a warp has in flight at once)
    if (sh.BG % 4 == 0) {
      if (sh.BG <= 128) page_scores<PAGE, 4, 1, 4>(sh, plan, a, sh_idx, np, p0, p1, sM, sLinv);
      else page_scores<PAGE, 4, 2, 2>(sh, plan, a, sh_idx, np, p0, p1, sM, sLinv);
    } else {
      if (sh.BG <= 32) page_scores<PAGE, 1, 1, 4>(sh, plan, a, sh_idx, np, p0, p1, sM, sLinv);
      else page_scores<PAGE, 1, 8, 1>(sh, plan, a, sh_idx, np, p0, p1, sM, sLinv);
    }
  } else {
    merged_row_stats(sh, plan, a.part_ml, sh_idx, sM, sLinv);
    __syncthreads();
    // o_out row: lane j holds the weight 2^(m_j - M) of split j (0 for an empty
    // split, whose O was never written); kFinBatch splits' O loads are in flight
    // together
    const int row = (blockIdx.x - score_ctas) * kRowsPerFinCta + warp;
    if (row >= sh.BG) return;
    const int b = row / sh.G, g = row % sh.G;
    static_assert(D / 32 == 4 || D / 32 == 2, "columns per lane");
    constexpr int kPer = D / 32;
    using V = typename std::conditional<kPer == 4, float4, float2>::type;
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
    const float Mrow = sM[row];
    for (int j0 = 0; j0 < plan.splits; j0 += 32) {
      float w_lane = 0.f;
      if (j0 + lane < plan.splits) {
        const size_t r = (sh_idx * plan.splits + j0 + lane) * sh.BG + row;
        const float2 ml = *reinterpret_cast<const float2 *>(a.part_ml + r * 2);
        w_lane = ml.y > 0.f ? exp2f(ml.x - Mrow) : 0.f;
      }
      const int nj = min(32, plan.splits - j0);
      for (int jb = 0; jb < nj; jb += kFinBatch) {
        V o[kFinBatch];
        float w[kFinBatch];
#pragma unroll
        for (int u = 0; u < kFinBatch; ++u) {
          w[u] = __shfl_sync(0xffffffffu, w_lane, (jb + u) & 31);
          const bool use = jb + u < nj && w[u] > 0.f;
          if (use) {
            const size_t r = (sh_idx * plan.splits + j0 + jb + u) * sh.BG + row;
            o[u] = *reinterpret_cast<const V *>(a.part_o + r * D + lane * kPer);
          } else {
            memset(&o[u], 0, sizeof(V));
            w[u] = 0.f;
          }
        }
#pragma unroll
        for (int u = 0; u < kFinBatch; ++u) {
          const float *ov = reinterpret_cast<const float *>(&o[u]);
#pragma unroll
          for (int i = 0; i < kPer; ++i) acc[i] += w[u] * ov[i];
        }
      }
    }
    const size_t orow = ((size_t)s * sh.B + b) * sh.Hq + (size_t)h * sh.G + g;
    __nv_bfloat16 *dst = a.o_out + orow * D + lane * kPer;
#pragma unroll
    for (int i = 0; i < kPer; i += 2)
      *reinterpret_cast<__nv_bfloat162 *>(dst + i) =
          __floats2bfloat162_rn(acc[i] * sLinv[row], acc[i + 1] * sLinv[row]);
    // log-sum-exp of the row's scaled logits over the prefix: (M + log2 L) ln 2
    if (sh.lse_out && lane == 0)
      sh.lse_out[orow] = sLinv[row] > 0.f ? (Mrow - log2f(sLinv[row])) * 0.6931471805599453f : -INFINITY;
  }
}

// ---------------------------------------------------------------------------
// select_topk: one CTA per (sequence, KV head).  Page scores are >= 0, so their
// fp32 bit patterns order like the values; a 4-pass radix select (8 bits per
// pass, histogram in shared memory, bin search by one warp) finds the kp-th
// largest key T.  Pages with key > T are kept, and among keys == T the lowest
// page indices, so ties go to the lower index; an ordered compaction writes the
// kept pages in ascending order.
// ---------------------------------------------------------------------------
constexpr int kTopkThreads = 1024;
constexpr int kTopkSmemKeys = 11264;  // keys staged in shared memory up to this many pages (44 KB)

__device__ __forceinline__ uint32_t score_key(float v) {
  return v > 0.f ? __float_as_uint(v) : 0u;  // -0 folds onto +0
}

__global__ void __launch_bounds__(kTopkThreads) select_topk(const __grid_constant__ PartialParams pp) {
  __shared__ uint32_t keys[kTopkSmemKeys];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_digit, s_remaining;
  __shared__ uint32_t scan_eq[kTopkThreads / 32], scan_gt[kTopkThreads / 32];
  __shared__ int s_bad;
  const Shape &sh = pp.sh;
  const SelectArgs &a = pp.a;
  sm100::grid_dep_wait();  // the page scores of select_finalize
  sm100::grid_dep_launch_dependents();
  const int s = blockIdx.y, h = blockIdx.x;
  const size_t sh_idx = (size_t)s * sh.Hkv + h;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = clamp_prefix(a.n_ctx[s], sh.max_pages, sh.P, a.status, false);
  const int np = (n + sh.P - 1) / sh.P;
  const int topk_tokens = a.topk[s];
  int kp = topk_tokens / sh.P;
  if (kp > sh.kmax || kp < 0 || topk_tokens % sh.P != 0) {
    if (tid == 0) raise_status(a.status, kStatusBadIndex);
    kp = max(0, min(kp, sh.kmax));
  }
  const float *sc = a.scores + sh_idx * sh.max_pages;
  int32_t *out = a.idx_out + sh_idx * sh.kmax;
  const int take = min(kp, np);
  const bool staged = np <= kTopkSmemKeys;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  int bad = 0;
  for (int i = tid; i < np; i += kTopkThreads) {
    const float v = sc[i];
    bad |= !isfinite(v);
    if (staged) keys[i] = score_key(v);
  }
  if (bad) s_bad = 1;
  __syncthreads();
  if (s_bad && tid == 0) raise_status(a.status, kStatusNonfinite);
  auto key_at = [&](int i) -> uint32_t { return staged ? keys[i] : score_key(sc[i]); };

  if (take >= np) {  // the budget covers the prefix: every page
    for (int i = tid; i < sh.kmax; i += kTopkThreads) out[i] = i < np ? i : -1;
    if (tid == 0) a.cnt_out[sh_idx] = np;
    return;
  }
  uint32_t prefix = 0, mask = 0;
  if (tid == 0) s_remaining = (uint32_t)take;
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0;
    __syncthreads();
    for (int i = tid; i < np; i += kTopkThreads) {
      const uint32_t key = key_at(i);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane L owns bins 255-8L down to 248-8L; counts above a lane's bins are
      // the exclusive prefix over the lanes before it
      const uint32_t rem = s_remaining;
      uint32_t cnt[8], local = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnt[q] = hist[255 - 8 * lane - q];
        local += cnt[q];
      }
      uint32_t incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t above = incl - local;
      if (above < rem && rem <= incl) {
        uint32_t cum = above;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (cum + cnt[q] >= rem) {
            s_digit = (uint32_t)(255 - 8 * lane - q);
            s_remaining = rem - cum;
            break;
          }
          cum += cnt[q];
        }
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
  }
  const uint32_t thr = prefix;           // the take-th largest key
  const uint32_t need_eq = s_remaining;  // keys equal to thr to keep, lowest pages first

  // ordered compaction: a contiguous chunk per thread, block-wide exclusive scans
  const int chunk = (np + kTopkThreads - 1) / kTopkThreads;
  const int i0 = min(np, tid * chunk), i1 = min(np, i0 + chunk);
  uint32_t n_eq = 0, n_gt = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
    n_gt += key > thr;
    n_eq += key == thr;
  }
  uint32_t e = n_eq, g = n_gt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t e2 = __shfl_up_sync(0xffffffffu, e, o), g2 = __shfl_up_sync(0xffffffffu, g, o);
    if (lane >= o) {
      e += e2;
      g += g2;
    }
  }
  if (lane == 31) {
    scan_eq[warp] = e;
    scan_gt[warp] = g;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t we = scan_eq[lane], wg = scan_gt[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t e2 = __shfl_up_sync(0xffffffffu, we, o), g2 = __shfl_up_sync(0xffffffffu, wg, o);
      if (lane >= o) {
        we += e2;
        wg += g2;
      }
    }
    scan_eq[lane] = we;
    scan_gt[lane] = wg;
  }
  __syncthreads();
  uint32_t eq_before = e - n_eq + (warp > 0 ? scan_eq[warp - 1] : 0u);
  uint32_t gt_before = g - n_gt + (warp > 0 ? scan_gt[warp - 1] : 0u);
  // position of a kept page = kept pages before it = (greater before) + min(equal before, need_eq)
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
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
  CUtensorMap kmap4, vmap4;
  err = make_kv_pages_tensor_map(&kmap4, a.k, sh.n_phys, sh.Hkv, PAGE, D, tc::kBN / PAGE);
  if (err != cudaSuccess) return err;
  err = make_kv_pages_tensor_map(&vmap4, a.v, sh.n_phys, sh.Hkv, PAGE, D, tc::kBN / PAGE);
  if (err != cudaSuccess) return err;
  constexpr auto kern = select_partial<D, PAGE>;
  constexpr size_t smem = tc::Layout<D, kSelStages>::kAlloc;
  err = set_smem_once<kern>(smem);
  if (err != cudaSuccess) return err;
  // all three kernels are programmatic dependents of the kernel ahead of them:
  // each one's set-up overlaps the tail of the previous one
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(plan.splits * plan.rowtiles, sh.Hkv, sh.S);
  cfg.blockDim = dim3(tc::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  err = cudaLaunchKernelEx(&cfg, kern, pp, kmap, vmap, kmap4, vmap4);
  if (err != cudaSuccess) return err;
  const int score_ctas = (sh.max_pages + plan.fin_pages - 1) / plan.fin_pages;
  const int o_ctas = (sh.BG + kRowsPerFinCta - 1) / kRowsPerFinCta;
  cfg.gridDim = dim3(score_ctas + o_ctas, sh.Hkv, sh.S);
  cfg.blockDim = dim3(kFinThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  err = cudaLaunchKernelEx(&cfg, select_finalize<D, PAGE>, pp);
  if (err != cudaSuccess) return err;
  cfg.gridDim = dim3(sh.Hkv, sh.S, 1);
  cfg.blockDim = dim3(kTopkThreads, 1, 1);
  err = cudaLaunchKernelEx(&cfg, select_topk, pp);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

DSA_TRACE_EXPORT(dsa_trace_select)

SelectPlan plan_select(const Shape &sh, int num_sms) {
  SelectPlan p{};
  p.rowtiles = (sh.BG + kRowsPerCta - 1) / kRowsPerCta;
  p.max_tiles = (int)(((long long)sh.max_pages * sh.P + tc::kBN - 1) / tc::kBN);
  const long long base = (long long)sh.S * sh.Hkv * p.rowtiles;
  // one resident CTA per SM and a single wave: a second, partial wave would
  // double the makespan
  int splits = (int)std::max(1LL, (long long)num_sms / base);
  splits = std::min(splits, p.max_tiles);
  p.tiles_per_split = (p.max_tiles + splits - 1) / splits;
  p.splits = (p.max_tiles + p.tiles_per_split - 1) / p.tiles_per_split;
  auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = 4096;  // status word and counters
  const size_t shn = (size_t)sh.S * sh.Hkv;
  // finalize: two resident CTAs per SM and a single wave; the output CTAs take
  // their share, the score CTAs the rest, each a multiple of 8 tiles (one per warp)
  const long long all_pages = (long long)sh.S * sh.Hkv * sh.max_pages;
  const long long o_ctas = (long long)sh.S * sh.Hkv * ((sh.BG + kRowsPerFinCta - 1) / kRowsPerFinCta);
  const long long score_target = std::max<long long>(num_sms, 2LL * num_sms - o_ctas);
  const long long fp = (all_pages + score_target - 1) / score_target;
  const long long tile_pages = tc::kBN / sh.P;  // score CTAs start on tile boundaries
  p.fin_pages = (int)std::max(tile_pages * 8, (fp + tile_pages * 8 - 1) / (tile_pages * 8) * (tile_pages * 8));
  p.off_part_o = off;   off = align(off + shn * p.splits * sh.BG * sh.d * 4);
  p.off_part_ml = off;  off = align(off + shn * p.splits * sh.BG * 2 * 4);
  const size_t units_per_tile = (size_t)tc::kBN / std::min(sh.P, tc::kHalfBN);
  p.off_pagepart = off; off = align(off + shn * p.max_tiles * sh.BG * units_per_tile * 4);
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
