// select.cu -- selection pass: exact attention of the block's step-1 queries
// over the whole prefix, reduced to page scores and cut to a top-k page set per
// KV head ("MAGE: All-[MASK] Block Already Knows Where to Look in Block
// Diffusion LLM", Approach).
//
// select_fused, launched so that the CTAs of a group are co-resident (as one
// thread-block cluster when a group has at most 16 CTAs, else cooperatively).  A group is
// one (sequence, KV head); its CTAs are the (split, 128-row tile) pairs.
//   1. Split-KV attention on the tcgen05 engine (tc_attn.cuh).  Per split: the
//      unnormalised O_j with row max m_j and sum l_j; per (tile, row): the mass
//      of each unit of the tile (min(page, 32) keys of one page) relative to the
//      row's reference max (pagepart), and that max (mtile).
//   2. Group barrier: a counter in the workspace header, bounded wait.
//   3. Every CTA forms each row's M = max_j m_j and L = sum_j l_j 2^(m_j - M),
//      scores the pages of its own tiles from partials bulk-copied into shared
//      memory,  S_h[q] = (1/BG) sum_rows pagepart * 2^(mtile - M) / L,  and
//      keeps its local top-kp as candidates (warp bitonic lists of (score,
//      page) keys for kp <= 128, a radix select beyond).
//   4. The group's last CTA to hand in its candidates selects the kp largest
//      (the head's top-kp is among them: each of its pages is in the local
//      top-kp of its own CTA) and writes them ascending.
//   5. Every CTA merges rows of o_out = sum_j 2^(m_j - M) O_j / L, taken from
//      a counter.
// Under the head-adaptive budget steps 3-4 keep kh = min(Hkv kp, np) pages per
// head instead, into a workspace list, and select_global_topk then selects over
// all KV heads of each sequence from those lists.
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
  int group0;  // first (sequence, KV head) group of this launch: s * Hkv + h
};

// ---------------------------------------------------------------------------
// Step 1, the engine policy: tcgen05 split-KV attention (tc_attn.cuh) over the
// split's contiguous 64-token tiles of the prefix, loaded page by page through
// the page table.  After each tile the softmax threads record, per (page, row),
// the tile's probability mass relative to the row's reference max (pagepart)
// and that max (mtile); the split's unnormalised O row, m and l go to part_o /
// part_ml.
// ---------------------------------------------------------------------------
constexpr int kSelStages = 6;  // three pairs of stages (the engine's PAIR mode)

// K/V tiles are read once: loaded with an evict-first L2 policy, so that the
// partials the tail reads back (written during the loop) stay in L2.
#ifndef DSA_KV_EVICT_FIRST
#define DSA_KV_EVICT_FIRST 1
#endif
// The partials (written once, read back by the tail) are stored evict-last.
#ifndef DSA_PART_EVICT_LAST
#define DSA_PART_EVICT_LAST 1
#endif

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
  int Hkv, h, G, Hq, BG, BGp, n, np, t_begin, row_base;  // BGp: row stride of mtile / pagepart
  bool report;                      // this CTA reports bad page-table entries (row tile 0)
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
    if (lane < kPages && my < 0 && lp0 + lane < np && report)
      raise_status(status, kStatusBadIndex);
    const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
    const long long p0 = __shfl_sync(0xffffffffu, my, 0);
    const bool consec = lane >= kPages || (valid && my == p0 + lane);
    const bool run = kPages > 1 && __all_sync(0xffffffffu, consec);
    if (lane == 0)
      sm100::mbar_arrive_expect_tx(bar, (uint32_t)__popc(vmask) * PAGE * 128u * kHalves * 2u);
#if DSA_KV_EVICT_FIRST
    const uint64_t l2pol = sm100::l2_policy_evict_first();
#endif
    if (run) {  // the whole tile in one box per half and tensor
      if (lane < 2 * kHalves) {
        const int hf = lane % kHalves;
        const bool isv = lane >= kHalves;
#if DSA_KV_EVICT_FIRST
        sm100::tma_load_4d_hint((isv ? sv : sk) + hf * half_bytes, isv ? vmap4 : kmap4, bar, hf * 64, 0,
                                h, (int)p0, l2pol);
#else
        sm100::tma_load_4d((isv ? sv : sk) + hf * half_bytes, isv ? vmap4 : kmap4, bar, hf * 64, 0, h,
                           (int)p0);
#endif
      }
      return;
    }
    const int pi = lane / (2 * kHalves), rem = lane % (2 * kHalves);
    const long long ph = __shfl_sync(0xffffffffu, my, pi < kPages ? pi : 0);
    if (pi < kPages && ((vmask >> pi) & 1u)) {
      const int hf = rem % kHalves;
      const bool isv = rem >= kHalves;
      const int y = (int)((ph * Hkv + h) * PAGE);
#if DSA_KV_EVICT_FIRST
      sm100::tma_load_2d_hint((isv ? sv : sk) + hf * half_bytes + pi * PAGE * 128, isv ? vmap : kmap,
                              bar, hf * 64, y, l2pol);
#else
      sm100::tma_load_2d((isv ? sv : sk) + hf * half_bytes + pi * PAGE * 128, isv ? vmap : kmap, bar,
                         hf * 64, y);
#endif
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
    // the row's tile max and unit masses of the tile, one vector store (units
    // past the prefix hold 0)
    float *dst = pagepart_head + ((size_t)tile * BGp + row) * U::kPerTile;
#if DSA_PART_EVICT_LAST
    const uint64_t pol = sm100::l2_policy_evict_last();
    sm100::st_hint(mtile_head + (size_t)tile * BGp + row, m_used, pol);
    if constexpr (U::kPerTile == 4)
      sm100::st_hint(reinterpret_cast<float4 *>(dst), make_float4(usum[0], usum[1], usum[2], usum[3]), pol);
    else
      sm100::st_hint(reinterpret_cast<float2 *>(dst), make_float2(usum[0], usum[1]), pol);
#else
    mtile_head[(size_t)tile * BGp + row] = m_used;
    if constexpr (U::kPerTile == 4)
      *reinterpret_cast<float4 *>(dst) = make_float4(usum[0], usum[1], usum[2], usum[3]);
    else
      *reinterpret_cast<float2 *>(dst) = make_float2(usum[0], usum[1]);
#endif
  }
};

// ---------------------------------------------------------------------------
// Steps 3 and 5 of the tail: the splits' row statistics and the output rows.
// ---------------------------------------------------------------------------
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
// of them loads its splits 16 at a time (all in flight together), then the tpr
// partial results are combined with shuffles.  after_issue() runs once, right
// after the first loads are issued (so that they go ahead of whatever it issues).
template <class AfterIssue>
__device__ __forceinline__ void merged_row_stats(const Shape &sh, const SelectPlan &plan,
                                                 const float *part_ml, size_t sh_idx, float *sM,
                                                 float *sLinv, AfterIssue after_issue) {
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
    for (int j0 = sub; j0 < plan.splits; j0 += 16 * tpr) {
      float2 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int j = j0 + u * tpr;
        v[u] = (valid && j < plan.splits) ? __ldcg(&ml[(size_t)j * sh.BG + row]) : make_float2(-INFINITY, 0.f);
      }
      if (row0 == 0 && j0 == sub) after_issue();  // (the loads above are already issued)
#pragma unroll
      for (int u = 0; u < 16; ++u) merge_ml(M, L, v[u].x, v[u].y);
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

// One row of o_out (0 <= row < BG of the group), merged by one warp:
//   o_out = sum_j 2^(m_j - M) O_j / L  (bf16),  lse = (M + log2 L) ln 2.
// Lane j of the warp loads the (m, l) of split j while kFinBatch splits' O rows
// are loaded together; an empty split (l = 0, O never written) gets weight 0.
constexpr int kFinBatch = 20;

template <int D>
__device__ __forceinline__ void merge_output_row(const Shape &sh, const SelectPlan &plan,
                                                 const SelectArgs &a, size_t sh_idx, int s, int h,
                                                 int row, const float *sM, const float *sLinv) {
  static_assert(D / 32 == 4 || D / 32 == 2, "columns per lane");
  constexpr int kPer = D / 32;
  using V = typename std::conditional<kPer == 4, float4, float2>::type;
  const int lane = threadIdx.x & 31;
  {
    const int b = row / sh.G, g = row % sh.G;
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
    const float Mrow = sM[row];
    for (int j0 = 0; j0 < plan.splits; j0 += 32) {
      // lane j: the (m, l) of split j0 + j; its O rows are loaded alongside, and
      // weighted once the (m, l) are in
      float2 ml_lane = make_float2(-INFINITY, 0.f);
      if (j0 + lane < plan.splits) {
        const size_t r = (sh_idx * plan.splits + j0 + lane) * sh.BG + row;
        ml_lane = __ldcg(reinterpret_cast<const float2 *>(a.part_ml + r * 2));
      }
      const int nj = min(32, plan.splits - j0);
      for (int jb = 0; jb < nj; jb += kFinBatch) {
        V o[kFinBatch];
#pragma unroll
        for (int u = 0; u < kFinBatch; ++u) {
          if (jb + u < nj) {
            const size_t r = (sh_idx * plan.splits + j0 + jb + u) * sh.BG + row;
            o[u] = __ldcg(reinterpret_cast<const V *>(a.part_o + r * D + lane * kPer));
          } else {
            memset(&o[u], 0, sizeof(V));
          }
        }
        const float w_lane = ml_lane.y > 0.f ? exp2f(ml_lane.x - Mrow) : 0.f;
#pragma unroll
        for (int u = 0; u < kFinBatch; ++u) {
          // an empty split (weight 0) never wrote its O: its loaded values are not used
          const float w = __shfl_sync(0xffffffffu, w_lane, (jb + u) & 31);
          if (jb + u < nj && w > 0.f) {
            const float *ov = reinterpret_cast<const float *>(&o[u]);
#pragma unroll
            for (int i = 0; i < kPer; ++i) acc[i] += w * ov[i];
          }
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
// Block-wide top-k by radix select.  Page scores are >= 0, so their fp32 bit
// patterns order like the values.  A 4-pass radix select (8 bits per pass,
// histogram in shared memory, bin search by one warp) finds the take-th largest
// key T; the keys > T are kept, and among the keys == T the lowest positions.
// An ordered compaction then emits the kept positions in ascending order, so a
// list sorted by page keeps ties towards the lower page.
// ---------------------------------------------------------------------------
struct TopkScratch {
  uint32_t hist[256];
  uint32_t scan_eq[32], scan_gt[32];
  uint32_t digit, remaining, flag, bad;
};

__device__ __forceinline__ uint32_t score_key(float v) {
  return v > 0.f ? __float_as_uint(v) : 0u;  // -0 (and NaN, reported separately) fold onto +0
}

// Threshold key T and the number of keys == T to keep, for 0 < take < n.  Every
// thread of the CTA calls it.
template <class KeyAt>
__device__ __forceinline__ void radix_threshold(int n, int take, KeyAt key_at, TopkScratch &sc,
                                                uint32_t &thr, uint32_t &need_eq) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = (int)blockDim.x;
  uint32_t prefix = 0, mask = 0;
  if (tid == 0) sc.remaining = (uint32_t)take;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += nt) sc.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += nt) {
      const uint32_t key = key_at(i);
      if ((key & mask) == prefix) atomicAdd(&sc.hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane L owns bins 255-8L down to 248-8L; counts above a lane's bins are
      // the exclusive prefix over the lanes before it
      const uint32_t rem = sc.remaining;
      uint32_t cnt[8], local = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnt[q] = sc.hist[255 - 8 * lane - q];
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
            sc.digit = (uint32_t)(255 - 8 * lane - q);
            sc.remaining = rem - cum;
            break;
          }
          cum += cnt[q];
        }
      }
    }
    __syncthreads();
    prefix |= sc.digit << shift;
    mask |= 255u << shift;
  }
  thr = prefix;
  need_eq = sc.remaining;
  __syncthreads();  // sc is reused by the caller
}

// Visits the positions 0..n-1 in ascending order, each thread a contiguous
// chunk, as visit(i, before, kept): kept tells whether key i is kept (key > T, or
// key == T among the first need_eq such positions) and before counts the kept
// positions below i.  The counts come from block-wide exclusive scans of each
// chunk's numbers of keys > T and == T.
template <class KeyAt, class Visit>
__device__ __forceinline__ void ordered_visit(int n, uint32_t thr, uint32_t need_eq, KeyAt key_at,
                                              Visit visit, TopkScratch &sc) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = (int)blockDim.x;
  const int warps = nt >> 5;
  const int chunk = (n + nt - 1) / nt;
  const int i0 = min(n, tid * chunk), i1 = min(n, i0 + chunk);
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
    sc.scan_eq[warp] = e;
    sc.scan_gt[warp] = g;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t we = lane < warps ? sc.scan_eq[lane] : 0u, wg = lane < warps ? sc.scan_gt[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t e2 = __shfl_up_sync(0xffffffffu, we, o), g2 = __shfl_up_sync(0xffffffffu, wg, o);
      if (lane >= o) {
        we += e2;
        wg += g2;
      }
    }
    sc.scan_eq[lane] = we;
    sc.scan_gt[lane] = wg;
  }
  __syncthreads();
  uint32_t eq_before = e - n_eq + (warp > 0 ? sc.scan_eq[warp - 1] : 0u);
  uint32_t gt_before = g - n_gt + (warp > 0 ? sc.scan_gt[warp - 1] : 0u);
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
    const bool gt = key > thr, eq = key == thr;
    visit(i, (int)(gt_before + min(eq_before, need_eq)), gt || (eq && eq_before < need_eq));
    gt_before += gt;
    eq_before += eq;
  }
  __syncthreads();  // sc is reused by the caller
}

// Emits (position, output slot) of the kept keys in ascending position; the slot
// of a kept key is the number of kept keys before it.
template <class KeyAt, class Emit>
__device__ __forceinline__ void ordered_emit(int n, uint32_t thr, uint32_t need_eq, KeyAt key_at,
                                             Emit emit, TopkScratch &sc) {
  ordered_visit(n, thr, need_eq, key_at, [&](int i, int before, bool kept) {
    if (kept) emit(i, before);
  }, sc);
}

// The take largest of n keys (ties to the lower position), emitted in ascending
// position; every key when take >= n.
template <class KeyAt, class Emit>
__device__ __forceinline__ void block_topk(int n, int take, KeyAt key_at, Emit emit, TopkScratch &sc) {
  if (take <= 0 || n <= 0) return;
  if (take >= n) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) emit(i, i);
    return;
  }
  uint32_t thr, need_eq;
  radix_threshold(n, take, key_at, sc, thr, need_eq);
  ordered_emit(n, thr, need_eq, key_at, emit, sc);
}

// ---------------------------------------------------------------------------
// Warp-level top-k for kp <= 128 (the fast path).  A candidate is a 64-bit key
// (score bits << 32) | ~page: keys order by score, then by lower page, and are
// all distinct; 0 pads (below every real key).  A warp holds a list of
// P = 32 E keys, key i = lane + 32 j in register j, and sorts or merges it with
// bitonic networks of shuffles.
// ---------------------------------------------------------------------------
constexpr int kFastTopk = 128;  // largest kp of the fast path

__device__ __forceinline__ uint64_t cand_key(float score, int page) {
  return ((uint64_t)score_key(score) << 32) | (uint32_t)~(uint32_t)page;
}
__device__ __forceinline__ int cand_page(uint64_t key) { return (int)~(uint32_t)key; }

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((uint64_t)hi << 32) | lo;
}
__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int src) {
  const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)v, src);
  const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(v >> 32), src);
  return ((uint64_t)hi << 32) | lo;
}

// One compare-exchange stage (distance d) of a bitonic network over the warp's
// list, in sub-sequences of length k: a pair (i, i + d) ends larger-first where
// (i & k) == 0 and smaller-first elsewhere.
template <int E>
__device__ __forceinline__ void bitonic_stage(uint64_t (&x)[E], int k, int d, int lane) {
  if (d >= 32) {
    const int dj = d >> 5;
#pragma unroll
    for (int j = 0; j < E; ++j) {
      if (j & dj) continue;
      const int jp = j | dj;
      const bool desc = ((lane + 32 * j) & k) == 0;
      const uint64_t a = x[j], b = x[jp];
      const bool swap = desc ? (a < b) : (a > b);
      x[j] = swap ? b : a;
      x[jp] = swap ? a : b;
    }
  } else {
#pragma unroll
    for (int j = 0; j < E; ++j) {
      const int i = lane + 32 * j;
      const uint64_t y = shfl_xor_u64(x[j], d);
      const bool keep_max = ((i & d) == 0) == ((i & k) == 0);
      x[j] = keep_max ? (x[j] > y ? x[j] : y) : (x[j] < y ? x[j] : y);
    }
  }
}

// Sorts the warp's list in descending order.
template <int E>
__device__ __forceinline__ void warp_sort_desc(uint64_t (&x)[E], int lane) {
#pragma unroll
  for (int k = 2; k <= 32 * E; k <<= 1)
#pragma unroll
    for (int d = k >> 1; d > 0; d >>= 1) bitonic_stage<E>(x, k, d, lane);
}

// x, y sorted descending: x becomes the P largest of x and y, sorted descending
// (max(x_i, y_{P-1-i}) is a bitonic sequence holding them; a bitonic merge sorts it).
template <int E>
__device__ __forceinline__ void warp_merge_top(uint64_t (&x)[E], const uint64_t (&y)[E], int lane) {
#pragma unroll
  for (int j = 0; j < E; ++j) {
    const uint64_t r = shfl_u64(y[E - 1 - j], 31 - lane);
    x[j] = x[j] > r ? x[j] : r;
  }
#pragma unroll
  for (int d = 16 * E; d > 0; d >>= 1) bitonic_stage<E>(x, 64 * E, d, lane);
}

// Every warp holds a sorted list; afterwards warp 0 holds the P largest of all
// of them, sorted descending.  wl: shared memory for (warps) lists.  Every
// thread of the CTA calls it.
template <int E>
__device__ __forceinline__ void block_merge_lists(uint64_t (&x)[E], uint64_t *wl) {
  constexpr int P = 32 * E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, warps = (int)blockDim.x >> 5;
#pragma unroll
  for (int j = 0; j < E; ++j) wl[warp * P + lane + 32 * j] = x[j];
  __syncthreads();
  for (int st = 1; st < warps; st <<= 1) {
    if (warp % (2 * st) == 0 && warp + st < warps) {
      uint64_t y[E];
#pragma unroll
      for (int j = 0; j < E; ++j) y[j] = wl[(warp + st) * P + lane + 32 * j];
      warp_merge_top<E>(x, y, lane);
#pragma unroll
      for (int j = 0; j < E; ++j) wl[warp * P + lane + 32 * j] = x[j];
    }
    __syncthreads();
  }
}

// Final selection (fast path), one CTA: the take largest keys over the G
// candidate lists (each P keys, sorted descending, in global memory), written
// to out[0..take) as ascending pages, out[take..kmax) = -1.
template <int E>
__device__ __forceinline__ void final_topk_fast(const uint64_t *lists, size_t list_stride, int G, int take,
                                                int32_t *out, int kmax, uint64_t *wl) {
  constexpr int P = 32 * E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, warps = (int)blockDim.x >> 5;
  uint64_t x[E];
#pragma unroll
  for (int j = 0; j < E; ++j) x[j] = 0;
  // one list ahead in flight
  uint64_t nx[E];
  if (warp < G) {
#pragma unroll
    for (int j = 0; j < E; ++j) nx[j] = __ldcg(lists + (size_t)warp * list_stride + lane + 32 * j);
  }
  for (int c = warp; c < G; c += warps) {
    uint64_t y[E];
#pragma unroll
    for (int j = 0; j < E; ++j) y[j] = nx[j];
    if (c + warps < G) {
#pragma unroll
      for (int j = 0; j < E; ++j) nx[j] = __ldcg(lists + (size_t)(c + warps) * list_stride + lane + 32 * j);
    }
    if (c == warp) {
#pragma unroll
      for (int j = 0; j < E; ++j) x[j] = y[j];
    } else {
      warp_merge_top<E>(x, y, lane);
    }
  }
  block_merge_lists<E>(x, wl);
  if (warp == 0) {
    // the take largest, re-sorted by ascending page: descending order of ~page
#pragma unroll
    for (int j = 0; j < E; ++j) x[j] = (lane + 32 * j < take) ? (x[j] & 0xffffffffull) : 0ull;
    warp_sort_desc<E>(x, lane);
#pragma unroll
    for (int j = 0; j < E; ++j) {
      const int i = lane + 32 * j;
      if (i < kmax) out[i] = i < take ? cand_page(x[j]) : -1;
    }
  }
  for (int i = P + (int)threadIdx.x; i < kmax; i += blockDim.x) out[i] = -1;
}

// Candidate list of one warp, built while the warp scores its tiles (fast path,
// E > 0): x holds the warp's P = 32 E largest keys so far, sorted descending;
// keys of newly scored pages collect in the warp's pend[0..P) and are sorted
// and merged into x whenever P of them are pending.
template <int E>
struct WarpCands {
  uint64_t x[E > 0 ? E : 1];
  uint64_t *pend;
  int npend;  // warp-uniform
  __device__ __forceinline__ void init(uint64_t *p) {
#pragma unroll
    for (int j = 0; j < (E > 0 ? E : 1); ++j) x[j] = 0;
    pend = p;
    npend = 0;
  }
  __device__ __forceinline__ void flush(int lane) {
    if constexpr (E > 0) {
      __syncwarp();
      uint64_t y[E];
#pragma unroll
      for (int j = 0; j < E; ++j) y[j] = lane + 32 * j < npend ? pend[lane + 32 * j] : 0ull;
      __syncwarp();
      warp_sort_desc<E>(y, lane);
      warp_merge_top<E>(x, y, lane);
      npend = 0;
    }
  }
};

// Stage-and-score loop of one CTA: tiles [tl0, tl1) of its (sequence, KV head),
// in batches of cap_t tiles through kStageBufs shared buffers (bulk copies of
// the tile maxima and unit masses; while one batch is scored the next
// kStageBufs - 1 are in flight).  start() issues the first kStageBufs batches;
// thread 0 issues each later one as its buffer is freed.
constexpr int kStageBufs = 4;
struct ScoreStager {
  const float *mt_head, *pp_head;  // [max_tiles][BGp], [max_tiles][BGp][units] of the head
  unsigned char *buf0;             // shared buffers, buf_bytes apart
  uint32_t bar0;                   // their mbarriers, 8 bytes apart (shared addresses)
  int tl0, tl1, cap_t, BGp, units, buf_bytes;

  __device__ __forceinline__ int batches() const { return tl1 > tl0 ? (tl1 - tl0 + cap_t - 1) / cap_t : 0; }
  __device__ __forceinline__ unsigned char *buf(int b) const { return buf0 + (size_t)(b % kStageBufs) * buf_bytes; }
  __device__ __forceinline__ uint32_t bar(int b) const { return bar0 + 8u * (uint32_t)(b % kStageBufs); }
  __device__ __forceinline__ uint32_t parity(int b) const { return (uint32_t)((b / kStageBufs) & 1); }
  __device__ __forceinline__ const float *mt_buf(int b) const { return reinterpret_cast<const float *>(buf(b)); }
  __device__ __forceinline__ const float *pp_buf(int b) const {
    return reinterpret_cast<const float *>(buf(b) + (size_t)cap_t * BGp * 4);
  }
  // thread 0 only
  __device__ __forceinline__ void issue(int b) const {
    const int t0 = tl0 + b * cap_t, nt = min(cap_t, tl1 - t0);
    const uint32_t mt_bytes = (uint32_t)nt * BGp * 4, pp_bytes = mt_bytes * units;
    sm100::mbar_arrive_expect_tx(bar(b), mt_bytes + pp_bytes);
    sm100::bulk_load(smem_addr(buf(b)), mt_head + (size_t)t0 * BGp, mt_bytes, bar(b));
    sm100::bulk_load(smem_addr(buf(b) + (size_t)cap_t * BGp * 4), pp_head + (size_t)t0 * BGp * units, pp_bytes,
                     bar(b));
  }
  // thread 0 only: barrier set-up and the first batches
  __device__ __forceinline__ void start() const {
#pragma unroll
    for (int i = 0; i < kStageBufs; ++i) sm100::mbar_init(bar0 + 8u * i, 1);
    sm100::fence_mbar_init();
    const int nb = batches();
    for (int b = 0; b < kStageBufs && b < nb; ++b) issue(b);
  }
};

// Page scores of nt tiles staged in shared memory, tile t being tile0 + t of the
// (sequence, KV head): mt [nt][BGp] tile maxima, pp [nt][BGp][units] unit
// masses.  One warp per tile; lane l takes the rows l + 32 c < BG, whose M and
// 1/L (rm, rl) it holds in registers.  Scores of pages below p_hi go to
// gout[page] and sout[page - p_lo] and, with E > 0, into the warp's candidates;
// a non-finite score (a non-finite input row) is reported in the status word.
template <int PAGE, int kRowChunks, int E>
__device__ __forceinline__ void scores_from_smem(const float *mt, const float *pp, int nt, int tile0,
                                                 int BG, int BGp, const float (&rm)[kRowChunks],
                                                 const float (&rl)[kRowChunks], float inv_bg, int p_lo,
                                                 int p_hi, float *gout, float *sout, uint32_t *status,
                                                 WarpCands<E> &wc) {
  using U = tc::Units<PAGE>;
  constexpr int kUnits = U::kPerTile;
  constexpr int kPagesPerTile = tc::kBN / PAGE;
  using W = typename std::conditional<kUnits == 4, float4, float2>::type;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, warps = (int)blockDim.x >> 5;
  constexpr int kT = 2;  // tiles a warp scores at once (independent chains)
  for (int t0 = warp; t0 < nt; t0 += kT * warps) {
    float acc[kT][kUnits];
#pragma unroll
    for (int tt = 0; tt < kT; ++tt)
#pragma unroll
      for (int u = 0; u < kUnits; ++u) acc[tt][u] = 0.f;
#pragma unroll
    for (int c = 0; c < kRowChunks; ++c) {
      const int row = lane + 32 * c;
      if (row < BG) {  // (rows past BG hold no data; a non-finite row makes the scores non-finite)
#pragma unroll
        for (int tt = 0; tt < kT; ++tt) {
          const int t = t0 + tt * warps;
          if (t < nt) {
            const float f = exp2f(mt[t * BGp + row] - rm[c]) * rl[c];
            const W w = reinterpret_cast<const W *>(pp)[t * BGp + row];
            const float *wu = reinterpret_cast<const float *>(&w);
#pragma unroll
            for (int u = 0; u < kUnits; ++u) acc[tt][u] = fmaf(wu[u], f, acc[tt][u]);
          }
        }
      }
    }
#pragma unroll
    for (int tt = 0; tt < kT; ++tt) {
      const int t = t0 + tt * warps;
      if (t >= nt) break;  // (warp-uniform)
      float pv[kPagesPerTile];
#pragma unroll
      for (int pi = 0; pi < kPagesPerTile; ++pi) {
        pv[pi] = 0.f;
#pragma unroll
        for (int u = pi * U::kPerPage; u < (pi + 1) * U::kPerPage; ++u) pv[pi] += acc[tt][u];
      }
      const float v = warp_sum_multi<kPagesPerTile>(pv, lane) * inv_bg;
      const int pi = lane / (32 / kPagesPerTile);
      const int page = (tile0 + t) * kPagesPerTile + pi;
      const bool owner = lane % (32 / kPagesPerTile) == 0, live = page < p_hi;
      if (owner && live) {
        gout[page] = v;
        if (sout) sout[page - p_lo] = v;
        if (!isfinite(v)) raise_status(status, kStatusNonfinite);
      }
      if constexpr (E > 0) {
        if (owner) wc.pend[wc.npend + pi] = live ? cand_key(v, page) : 0ull;
        wc.npend += kPagesPerTile;
        if (wc.npend == 32 * E) wc.flush(lane);
      }
    }
  }
}

// Scores every staged batch of a ScoreStager (all threads of the CTA); with
// E > 0 each warp also builds its candidate list and the CTA's P largest keys
// end in `slot` (sorted descending, 0-padded), through the warp lists in wl.
template <int PAGE, int kRC, int E>
__device__ __forceinline__ void score_batches(const ScoreStager &st, const float *sM, const float *sLinv,
                                              int BG, float inv_bg, int p_lo, int p_hi, float *gout,
                                              float *sout, uint32_t *status, const sm100::WaitCtx &ctx,
                                              uint64_t *wl, uint64_t *slot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float rm[kRC], rl[kRC];
#pragma unroll
  for (int c = 0; c < kRC; ++c) {
    const int row = lane + 32 * c;
    rm[c] = row < BG ? sM[row] : 0.f;
    rl[c] = row < BG ? sLinv[row] : 0.f;
  }
  WarpCands<E> wc;
  wc.init(wl + (size_t)warp * 32 * (E > 0 ? E : 1));
  const int nb = st.batches();
  for (int b = 0; b < nb; ++b) {
    sm100::mbar_wait(st.bar(b), st.parity(b), ctx);
    const int t0 = st.tl0 + b * st.cap_t;
    scores_from_smem<PAGE, kRC, E>(st.mt_buf(b), st.pp_buf(b), min(st.cap_t, st.tl1 - t0), t0, BG, st.BGp,
                                   rm, rl, inv_bg, p_lo, p_hi, gout, sout, status, wc);
    __syncthreads();  // every read of this buffer is done before it is refilled
    if (threadIdx.x == 0 && b + kStageBufs < nb) {
      sm100::fence_proxy_async_smem();
      st.issue(b + kStageBufs);
    }
  }
  if constexpr (E > 0) {
    if (wc.npend > 0) wc.flush(lane);
  }
  if (threadIdx.x == 0) DSA_TRACE_EVENT(39);
  if constexpr (E > 0) {
    block_merge_lists<E>(wc.x, wl);
    if (warp == 0) {
#pragma unroll
      for (int j = 0; j < E; ++j) slot[lane + 32 * j] = wc.x[j];
    }
  }
  __syncthreads();
}

// Shared memory of the tail (steps 2-4): the engine's whole layout is free once
// it has been torn down.  [0, 1K) sM, [1K, 2K) sLinv, [2K, ..) TopkScratch,
// kOffTailBars: the staging buffers' mbarriers; kTailHead: the warps' candidate
// lists (fast path); kOffSf: the CTA's page scores, then the staging buffers.
constexpr int kOffTailBars = 3584;
// A CTA that arrives at the group barrier with more than this many CTAs of the
// group still to come starts its staging copies before it waits.
constexpr int kPrefetchMargin = 3;
constexpr int kTailHead = 4096;
constexpr int kOffSf = kTailHead + (tc::kThreads / 32) * kFastTopk * 8;
template <int D>
constexpr int tail_bytes() { return (int)tc::Layout<D, kSelStages>::kOffBar; }
// the page scores take at most a quarter of what follows kOffSf; the rest holds
// the staging buffers, each at least one tile
static_assert((tail_bytes<64>() - kOffSf) * 3 / 4 / 4 >= 256 * 4 * 5, "staging buffer");

template <int D, int PAGE>
__global__ void __launch_bounds__(tc::kThreads, 1)
    select_fused(const __grid_constant__ PartialParams pp, const __grid_constant__ CUtensorMap kmap,
                 const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap kmap4,
                 const __grid_constant__ CUtensorMap vmap4) {
  extern __shared__ unsigned char smem_raw[];
  const Shape &sh = pp.sh;
  const SelectPlan &plan = pp.plan;
  const SelectArgs &a = pp.a;
  const int G = plan.group_ctas;
  const int gl = blockIdx.x / G, c = blockIdx.x % G;  // group of this launch, CTA in the group
  const int group = pp.group0 + gl;
  const int s = group / sh.Hkv, h = group % sh.Hkv;
  const int split = c / plan.rowtiles, rt = c % plan.rowtiles;
  if (threadIdx.x == 0) DSA_TRACE_EVENT(0);
  SelectPolicy<D, PAGE> pol;
  pol.kmap = &kmap;
  pol.vmap = &vmap;
  pol.kmap4 = &kmap4;
  pol.vmap4 = &vmap4;
  tc::Engine<D, kSelStages, true> eng;
  eng.setup(smem_raw, pol);
  // everything below may read what the kernel ahead of this one wrote
  sm100::grid_dep_wait();
  sm100::grid_dep_launch_dependents();

  // ---- 1. split-KV attention ----
  const int n = clamp_prefix(a.n_ctx[s], sh.max_pages, PAGE, a.status, threadIdx.x == 0 && c == 0);
  const int ntiles = (n + tc::kBN - 1) / tc::kBN;
  const int t_begin = split * plan.tiles_per_split;
  const int num_tiles = max(0, min(ntiles, t_begin + plan.tiles_per_split) - t_begin);
  const size_t sh_idx = (size_t)s * sh.Hkv + h;
  pol.page_row = sh.page_table ? sh.page_table + (size_t)s * sh.max_pages : nullptr;
  pol.q_head = a.q + ((size_t)s * sh.B * sh.Hq + (size_t)h * sh.G) * D;
  pol.mtile_head = a.mtile + sh_idx * plan.max_tiles * plan.bgp;
  pol.pagepart_head = a.pagepart + sh_idx * plan.max_tiles * plan.bgp * tc::Units<PAGE>::kPerTile;
  pol.status = a.status;
  pol.n_phys = sh.n_phys;
  pol.phys0 = (long long)s * sh.max_pages;
  pol.Hkv = sh.Hkv;
  pol.h = h;
  pol.G = sh.G;
  pol.Hq = sh.Hq;
  pol.BG = sh.BG;
  pol.BGp = plan.bgp;
  pol.n = n;
  pol.np = (n + PAGE - 1) / PAGE;
  pol.t_begin = t_begin;
  pol.row_base = rt * kRowsPerCta;
  pol.report = rt == 0;
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
#if DSA_PART_EVICT_LAST
          sm100::st_hint(dst + i, make_float4(v[0], v[1], v[2], v[3]), sm100::l2_policy_evict_last());
#else
          dst[i] = make_float4(v[0], v[1], v[2], v[3]);
#endif
        }
      }
    }
    if (row_ok && g == 0)
      *reinterpret_cast<float2 *>(a.part_ml + prow * 2) =
          l_row > 0.f ? make_float2(m_row, l_row) : make_float2(-INFINITY, 0.f);
    if (row == rt * kRowsPerCta) DSA_TRACE_EVENT(7);
  }
  eng.teardown();  // ends with a __syncthreads: every partial of this CTA is written

  // ---- staging of this CTA's page partials (tile maxima, unit masses) ----
  constexpr int kPagesPerTile = tc::kBN / PAGE;
  constexpr int kUnits = tc::Units<PAGE>::kPerTile;
  unsigned char *tail = eng.smem;
  float *sM = reinterpret_cast<float *>(tail);
  float *sLinv = sM + 256;
  TopkScratch &sc = *reinterpret_cast<TopkScratch *>(tail + 2048);
  static_assert(2048 + sizeof(TopkScratch) <= kOffTailBars, "tail header");
  const int np = (n + PAGE - 1) / PAGE;
  const int per_rt = (num_tiles + plan.rowtiles - 1) / plan.rowtiles;
  const int tl0 = t_begin + min(num_tiles, rt * per_rt);
  const int tl1 = t_begin + min(num_tiles, (rt + 1) * per_rt);
  const int p0 = tl0 * kPagesPerTile;
  const int p1 = max(p0, min(np, tl1 * kPagesPerTile));
  const int n_loc = p1 - p0;
  const int BGp = plan.bgp;
  const bool aborted = *eng.abort_flag() != 0;
  uint64_t *wl = reinterpret_cast<uint64_t *>(tail + kTailHead);
  const int sf_bytes = (n_loc * 4 + 15) & ~15;
  const bool staged = sf_bytes <= (tail_bytes<D>() - kOffSf) / 4;
  float *sf = reinterpret_cast<float *>(tail + kOffSf);
  const int off_buf = kOffSf + (staged ? sf_bytes : 0);
  const int tile_bytes = BGp * 4 * (1 + kUnits);
  ScoreStager st;
  st.mt_head = a.mtile + sh_idx * plan.max_tiles * BGp;
  st.pp_head = a.pagepart + sh_idx * plan.max_tiles * BGp * kUnits;
  st.cap_t = (tail_bytes<D>() - off_buf) / (kStageBufs * tile_bytes);  // >= 1 (see kOffSf)
  st.buf_bytes = st.cap_t * tile_bytes;
  st.buf0 = tail + off_buf;
  st.bar0 = smem_addr(tail + kOffTailBars);
  st.tl0 = tl0;
  st.tl1 = aborted ? tl0 : tl1;  // nothing is staged after an abort
  st.BGp = BGp;
  st.units = kUnits;
  // With one row tile the CTA scores only tiles it wrote itself.  A CTA that
  // will wait at the group barrier (several CTAs of the group still to come)
  // starts their copies before waiting; the late ones load the row statistics
  // first, so that those loads are not queued behind the copies.
  const bool own_rows = plan.rowtiles == 1;
  sm100::fence_proxy_async_global();  // this thread's partial stores, before any bulk copy
  __syncthreads();

  // ---- 2. group barrier ----
  uint32_t *arrive = a.counters + 4 * gl, *leave = arrive + 1, *orows = arrive + 2, *odone = arrive + 3;
  const int topk_tokens = a.topk[s];  // (in flight during the wait)
  if (threadIdx.x == 0) {
    DSA_TRACE_EVENT(40);
    const uint32_t prev = sm100::arrive_gpu(arrive);
    sc.flag = own_rows && (int)prev + kPrefetchMargin < G;
  }
  __syncthreads();
  const bool started = sc.flag;
  if (started && threadIdx.x == 0) st.start();
  if (threadIdx.x == 0) {
    // (the test build waits for one arrival more than the group has, so that this
    // wait runs out and reports itself; all G partials are written even then)
    if (!sm100::wait_count_geq(arrive, (uint32_t)G + sm100::kTestExtraArrivals))
      sm100::note_timeout(a.status, 0xffu);
    DSA_TRACE_EVENT(41);
  }
  sm100::fence_proxy_async_global();  // the other CTAs' partials, before the bulk copies
  __syncthreads();

  // ---- 3. row statistics, page scores, local candidates ----
  // Under the head-adaptive budget the final selection is select_global_topk's:
  // this kernel writes the page scores and each head's best kh = min(Hkv kp, np)
  // pages, which hold every page of the head that the shared budget of Hkv kp
  // keeps (within a head the two rankings agree, so a kept page has fewer than
  // Hkv kp pages of its own head above it).
  const bool per_head = sh.head_budget == 0;
  int kp = topk_tokens / PAGE;
  if ((per_head && kp > sh.kmax) || kp < 0 || topk_tokens % PAGE != 0) {
    if (threadIdx.x == 0 && c == 0) raise_status(a.status, kStatusBadIndex);
    kp = max(0, min(kp, sh.kmax));
  }
  const int kh = per_head ? kp : (int)min((long long)sh.Hkv * kp, (long long)np);
  const int take = min(kh, np);
  const bool every_page = take >= np;
  const bool fast = kh <= kFastTopk;
  const int E = every_page ? 0 : (!fast ? 0 : (kh <= 32 ? 1 : (kh <= 64 ? 2 : 4)));
  merged_row_stats(sh, plan, a.part_ml, sh_idx, sM, sLinv, [&]() {
    if (threadIdx.x == 0 && !started) st.start();
  });
  __syncthreads();
  if (threadIdx.x == 0) DSA_TRACE_EVENT(31);
  float *gs = a.scores + sh_idx * sh.max_pages;
  const size_t cslot = sh_idx * G + c;
  uint64_t *slot = a.cand + cslot * plan.slot_len;
  {
    const float inv_bg = 1.f / (float)sh.BG;
    float *sout = staged ? sf : nullptr;
#define DSA_SCORE(KRC, EE)                                                                                   \
  score_batches<PAGE, KRC, EE>(st, sM, sLinv, sh.BG, inv_bg, p0, p1, gs, sout, a.status, eng.ctx, wl, slot)
    if (BGp <= 128) {
      if (E == 0) DSA_SCORE(4, 0); else if (E == 1) DSA_SCORE(4, 1); else if (E == 2) DSA_SCORE(4, 2); else DSA_SCORE(4, 4);
    } else {
      if (E == 0) DSA_SCORE(8, 0); else if (E == 1) DSA_SCORE(8, 1); else if (E == 2) DSA_SCORE(8, 2); else DSA_SCORE(8, 4);
    }
#undef DSA_SCORE
  }
  if (threadIdx.x == 0) DSA_TRACE_EVENT(44);
  // (score_batches ends with a __syncthreads: sf, the slot and this CTA's part of
  // a.scores are complete)
  if (!every_page && !fast) {
    const int take_loc = min(take, n_loc);
    auto score_at = [&](int i) -> float { return staged ? sf[i] : __ldcg(gs + p0 + i); };
    auto key_loc = [&](int i) -> uint32_t { return score_key(score_at(i)); };
    block_topk(n_loc, take_loc, key_loc, [&](int i, int pos) { slot[pos] = cand_key(score_at(i), p0 + i); },
               sc);
    if (threadIdx.x == 0) a.ccnt[cslot] = take_loc;
  }
  if (threadIdx.x == 0) DSA_TRACE_EVENT(46);

  // ---- 4. the group's last CTA selects among the candidates; every CTA then
  //      merges output rows, taken from a counter ----
  __syncthreads();  // every candidate of this CTA is written
  if (threadIdx.x == 0) {
    DSA_TRACE_EVENT(42);
    const uint32_t prev = sm100::arrive_gpu(leave);
    sc.flag = prev == (uint32_t)G - 1u;
    if (sc.flag) __threadfence();  // the other CTAs' candidates are visible from here on
  }
  __syncthreads();
  if (sc.flag) {
    // per head: idx_out, padded with -1 to kmax; head-adaptive budget: the head's
    // list for select_global_topk, take entries
    int32_t *out = per_head ? a.idx_out + sh_idx * sh.kmax : a.hsel + sh_idx * sh.max_pages;
    const int out_len = per_head ? sh.kmax : take;
    const uint64_t *lists = a.cand + sh_idx * G * plan.slot_len;
    if (every_page) {
      for (int i = threadIdx.x; i < out_len; i += blockDim.x) out[i] = i < np ? i : -1;
    } else if (fast) {
      if (E == 1) final_topk_fast<1>(lists, plan.slot_len, G, take, out, out_len, wl);
      else if (E == 2) final_topk_fast<2>(lists, plan.slot_len, G, take, out, out_len, wl);
      else final_topk_fast<4>(lists, plan.slot_len, G, take, out, out_len, wl);
    } else {
      // offsets of the CTAs' candidate lists (CTA order is page order)
      int *offs = reinterpret_cast<int *>(tail + kTailHead);
      const int offs_bytes = ((G + 1) * 4 + 15) & ~15;
      uint64_t *cs = reinterpret_cast<uint64_t *>(tail + kTailHead + offs_bytes);
      const int cap = (tail_bytes<D>() - kTailHead - offs_bytes) / 8;
      const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, warps = (int)blockDim.x >> 5;
      if (warp == 0) {
        int carry = 0;
        for (int j0 = 0; j0 < G; j0 += 32) {
          const int v = j0 + lane < G ? min(max(__ldcg(a.ccnt + sh_idx * G + j0 + lane), 0), plan.slot_len) : 0;
          int incl = v;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
          }
          if (j0 + lane < G) offs[j0 + lane] = carry + incl - v;
          carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) offs[G] = carry;
      }
      __syncthreads();
      const int ncand = offs[G];
      if (ncand <= cap) {
        for (int j = warp; j < G; j += warps) {
          const uint64_t *src = lists + (size_t)j * plan.slot_len;
          const int o = offs[j], cnt = offs[j + 1] - o;
          for (int i = lane; i < cnt; i += 32) cs[o + i] = __ldcg(src + i);
        }
        __syncthreads();
        if (threadIdx.x == 0) DSA_TRACE_EVENT(47);
        block_topk(ncand, take, [&](int i) -> uint32_t { return (uint32_t)(cs[i] >> 32); },
                   [&](int i, int pos) { out[pos] = cand_page(cs[i]); }, sc);
      } else {  // too many candidates to stage: select over every page score of the head
        block_topk(np, take, [&](int i) -> uint32_t { return score_key(__ldcg(gs + i)); },
                   [&](int i, int pos) { out[pos] = i; }, sc);
      }
      for (int i = take + threadIdx.x; i < out_len; i += blockDim.x) out[i] = -1;
    }
    if (threadIdx.x == 0) {
      if (per_head) a.cnt_out[sh_idx] = take;
      else a.hcnt[sh_idx] = take;
      DSA_TRACE_EVENT(43);
    }
  }
  {
    const int warp = threadIdx.x >> 5, warps = (int)blockDim.x >> 5;
    for (;;) {
      __syncthreads();  // the previous row block is taken
      if (threadIdx.x == 0) sc.digit = atomicAdd(orows, (uint32_t)warps);
      __syncthreads();
      const int base = (int)sc.digit;
      if (base >= sh.BG) break;
      if (base + warp < sh.BG) merge_output_row<D>(sh, plan, a, sh_idx, s, h, base + warp, sM, sLinv);
    }
  }
  if (threadIdx.x == 0) {
    // the group's last CTA to find no rows left resets the counters: every CTA
    // of the group has passed them all
    if (atomicAdd(odone, 1u) == (uint32_t)G - 1u) {
      *arrive = 0u;
      *leave = 0u;
      *orows = 0u;
      *odone = 0u;
    }
    DSA_TRACE_EVENT(45);
  }
}

// ---------------------------------------------------------------------------
// Head-adaptive budget ("Step-dLLM: Adaptive Step-aware Sparse Attention for
// Efficient Diffusion LLM Inference", abstract): one CTA per sequence ranks the
// (KV head, page) pairs of the sequence by the page scores select_fused wrote
// and keeps the best Hkv * kp; pair (h, q) is position h * np + q, so ties go to
// the lower head, then the lower page.  Each head's kept pages are written in
// ascending order, a head keeping any number of them (none included).
//
// Fast path (positions <= kGlobalBits, candidates <= kGlobalCand):
//   1. the candidates: the heads' lists of select_fused (each head's best
//      min(Hkv kp, np) pages, which hold every kept pair) when they number at
//      most kGlobalCand; otherwise the range of all keys (one pass, coalesced
//      16-byte loads), then histograms of up to 4096 bins over it give the bin
//      holding the take-th largest key, narrowed while it holds too many keys,
//      and the keys >= its lower edge t0 are compacted;
//   2. with their positions in shared memory, an exact radix select among the
//      candidates gives T and the number of keys == T to keep;
//   3. bitmaps over the positions: keys > T kept, keys == T kept in ascending
//      position until need_eq of them;
//   4. warp h writes head h's kept pages (its stretch of the bitmap) in order.
// Otherwise every pass reads the keys from L2 (radix select and two ordered
// visits).
// ---------------------------------------------------------------------------
// Calls f(key, position) for every (KV head, page) pair of a sequence, position
// h * np + q; rows of the score array are max_pages apart.  16-byte loads, eight
// per thread in flight, when the rows are 16-byte aligned.  A flat index v over
// rows of n items splits as (h, j) = (v / n, v % n) with one division per eight
// items: the next item of the thread is nt further, i.e. nt / n rows and nt % n
// items on.
template <class F>
__device__ __forceinline__ void for_each_pair(const float *scores, int max_pages, int Hkv, int np, F f) {
  const int nt = (int)blockDim.x;
  const bool vec = (max_pages & 3) == 0;
  const int n = vec ? (np + 3) >> 2 : np;  // items per row: 4-page vectors or pages
  const int tot = Hkv * n;
  if (tot <= 0) return;
  const int dq = nt / n, dr = nt - dq * n;
  for (int v0 = threadIdx.x; v0 < tot; v0 += 8 * nt) {
    int hh[8], jj[8];
    {
      int h = v0 / n, j = v0 - h * n;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        hh[u] = h;
        jj[u] = j;
        h += dq;
        j += dr;
        if (j >= n) {
          j -= n;
          ++h;
        }
      }
    }
    if (vec) {
      float4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (hh[u] < Hkv) x[u] = __ldcg(reinterpret_cast<const float4 *>(scores + (size_t)hh[u] * max_pages) + jj[u]);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (hh[u] < Hkv) {
          const float e[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (4 * jj[u] + c < np) f(score_key(e[c]), hh[u] * np + 4 * jj[u] + c);
        }
      }
    } else {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (hh[u] < Hkv) x[u] = __ldcg(scores + (size_t)hh[u] * max_pages + jj[u]);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (hh[u] < Hkv) f(score_key(x[u]), hh[u] * np + jj[u]);
    }
  }
}

constexpr int kGlobalThreads = 1024;
constexpr int kGlobalBits = 1 << 18;       // positions the bitmaps cover (2 x 32 KB)
constexpr int kGlobalCand = 8192;          // candidates held in shared memory (64 KB)
constexpr int kGlobalHistBins = 4096;
constexpr int kGlobalSmem = 2 * (kGlobalBits / 8) + kGlobalCand * 8 + kGlobalHistBins * 4;

__global__ void __launch_bounds__(kGlobalThreads) select_global_topk(const __grid_constant__ PartialParams pp) {
  extern __shared__ __align__(16) unsigned char gsm[];
  __shared__ TopkScratch sc;
  __shared__ int s_base[kMaxHeadsAdaptive + 1];  // kept pairs before head h
  __shared__ uint32_t s_ncand, s_bin, s_above;
  const Shape &sh = pp.sh;
  const SelectArgs &a = pp.a;
  sm100::grid_dep_wait();  // the page scores of select_fused
  sm100::grid_dep_launch_dependents();
  const int s = blockIdx.x, tid = threadIdx.x, nt = (int)blockDim.x;
  const int lane = tid & 31, warp = tid >> 5, warps = nt >> 5;
  const int n = clamp_prefix(a.n_ctx[s], sh.max_pages, sh.P, a.status, false);
  const int np = (n + sh.P - 1) / sh.P;
  const int topk_tokens = a.topk[s];
  int kp = topk_tokens / sh.P;
  if (kp < 0 || topk_tokens % sh.P != 0) {
    if (tid == 0) raise_status(a.status, kStatusBadIndex);
    kp = max(0, kp);
  }
  const int total = sh.Hkv * np;
  const int take = (int)min((long long)sh.Hkv * kp, (long long)total);
  const float *scores = a.scores + (size_t)s * sh.Hkv * sh.max_pages;
  int32_t *out = a.idx_out + (size_t)s * sh.Hkv * sh.kmax;
  auto key_at = [&](int i) -> uint32_t {
    const int h = i / np;
    return score_key(__ldcg(scores + (size_t)h * sh.max_pages + (i - h * np)));
  };
  // per head: count, padding, overflow report (s_base complete)
  auto finish_counts = [&]() {
    for (int h = warp; h < sh.Hkv; h += warps) {
      const int cnt = s_base[h + 1] - s_base[h];
      if (cnt > sh.kmax && lane == 0) raise_status(a.status, kStatusBadIndex);
      const int kept = min(cnt, sh.kmax);
      for (int j = kept + lane; j < sh.kmax; j += 32) out[(size_t)h * sh.kmax + j] = -1;
      if (lane == 0) a.cnt_out[(size_t)s * sh.Hkv + h] = kept;
    }
  };

  uint32_t *keep = reinterpret_cast<uint32_t *>(gsm);                   // [kGlobalBits / 32]
  uint32_t *eqb = keep + kGlobalBits / 32;                               // [kGlobalBits / 32]
  uint2 *cand = reinterpret_cast<uint2 *>(eqb + kGlobalBits / 32);       // [kGlobalCand] (key, position)
  uint32_t *hist = reinterpret_cast<uint32_t *>(cand + kGlobalCand);     // [kGlobalHistBins]
  constexpr int kHist = kGlobalHistBins;
  bool fast = total <= kGlobalBits && take > 0 && take < total;
  uint32_t t0 = 0u;  // candidates: every key >= t0
  // the candidates can be the heads' lists of select_fused (each head's best
  // min(Hkv kp, np) pages, which hold every pair the budget keeps) when they fit
  int ncl = 0;
  for (int h = 0; h < sh.Hkv; ++h) ncl += min(max(a.hcnt[(size_t)s * sh.Hkv + h], 0), np);
  const bool from_lists = fast && ncl <= kGlobalCand;
  if (fast && !from_lists) {
    // 1. the key range holding the take-th largest key: the range of all keys
    //    (one pass), then histograms of up to 4096 bins of 2^shift keys over the
    //    current range, narrowed to the bin that holds it while that bin has
    //    too many keys
    uint32_t kmn = 0xffffffffu, kmx = 0u;
    for_each_pair(scores, sh.max_pages, sh.Hkv, np, [&](uint32_t key, int) {
      kmn = min(kmn, key);
      kmx = max(kmx, key);
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      kmn = min(kmn, __shfl_xor_sync(0xffffffffu, kmn, o));
      kmx = max(kmx, __shfl_xor_sync(0xffffffffu, kmx, o));
    }
    if (lane == 0) {
      sc.scan_eq[warp] = kmn;
      sc.scan_gt[warp] = kmx;
    }
    __syncthreads();
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int w = 0; w < warps; ++w) {
      lo = min(lo, sc.scan_eq[w]);
      hi = max(hi, sc.scan_gt[w]);
    }
    __syncthreads();  // (sc is reused)
    uint32_t above = 0u;  // keys above the current range
    for (int level = 0; level < 4; ++level) {
      uint32_t shift = 0u;  // the smallest with (hi - lo) >> shift < kHist
      while (((hi - lo) >> shift) >= (uint32_t)kHist) ++shift;
      const uint32_t width = 1u << shift;
      for (int i = tid; i < kHist; i += nt) hist[i] = 0u;
      if (tid == 0) {
        s_bin = 0u;
        s_above = 0xffffffffu;  // (set below: some bin always holds the take-th key)
      }
      __syncthreads();
      for_each_pair(scores, sh.max_pages, sh.Hkv, np, [&](uint32_t key, int) {
        if (key >= lo && key <= hi) atomicAdd(&hist[(key - lo) >> shift], 1u);
      });
      __syncthreads();
      // the bin of the take-th largest key: warp 0 scans from the top
      if (warp == 0) {
        constexpr int kPer = kHist / 32;
        uint32_t local = 0;
        for (int j = 0; j < kPer; ++j) local += hist[kHist - 1 - (lane * kPer + j)];
        uint32_t incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const uint32_t before = above + incl - local;
        if (before < (uint32_t)take && (uint32_t)take <= above + incl) {
          uint32_t cum = before;
          for (int j = 0; j < kPer; ++j) {
            const int bin = kHist - 1 - (lane * kPer + j);
            if (cum + hist[bin] >= (uint32_t)take) {
              s_bin = (uint32_t)bin;
              s_above = cum + hist[bin];  // keys >= the bin's lower edge
              break;
            }
            cum += hist[bin];
          }
        }
      }
      __syncthreads();
      const uint32_t b = s_bin;
      t0 = lo + b * width;
      if (s_above <= (uint32_t)kGlobalCand || width == 1u) break;
      above = s_above - hist[b];
      hi = (uint32_t)min((unsigned long long)hi, (unsigned long long)t0 + width - 1u);
      lo = t0;
      __syncthreads();  // (hist is cleared for the next level)
    }
    fast = s_above <= (uint32_t)kGlobalCand;
  }
  if (fast) {
    // 2. candidates with their positions: the heads' lists, or every key >= t0
    if (tid == 0) s_ncand = from_lists ? (uint32_t)ncl : 0u;
    __syncthreads();
    if (from_lists) {
      for (int i = tid; i < ncl; i += nt) {
        int h = 0, base = 0;
        for (;;) {  // the head whose list holds entry i (ncl counts every list)
          const int c = min(max(a.hcnt[(size_t)s * sh.Hkv + h], 0), np);
          if (i < base + c || h == sh.Hkv - 1) break;
          base += c;
          ++h;
        }
        int page = a.hsel[((size_t)s * sh.Hkv + h) * sh.max_pages + (i - base)];
        if (page < 0 || page >= np) {
          raise_status(a.status, kStatusBadIndex);
          page = 0;
        }
        cand[i] = make_uint2(score_key(__ldcg(scores + (size_t)h * sh.max_pages + page)),
                             (uint32_t)(h * np + page));
      }
    } else {
      for_each_pair(scores, sh.max_pages, sh.Hkv, np, [&](uint32_t key, int pos) {
        if (key >= t0) {
          const uint32_t slot = atomicAdd(&s_ncand, 1u);
          if (slot < (uint32_t)kGlobalCand) cand[slot] = make_uint2(key, (uint32_t)pos);
        }
      });
    }
    for (int w = tid; w < (total + 31) / 32; w += nt) {
      keep[w] = 0u;
      eqb[w] = 0u;
    }
    __syncthreads();
    const int nc = (int)min(s_ncand, (uint32_t)kGlobalCand);
    uint32_t thr = 0u, need_eq = 0u;
    if (take < nc) {
      radix_threshold(nc, take, [&](int i) -> uint32_t { return cand[i].x; }, sc, thr, need_eq);
    } else {  // (every candidate is kept)
      thr = 0u;
      need_eq = (uint32_t)nc;
    }
    // 3. bitmaps: keys > T kept; keys == T in ascending position until need_eq
    for (int i = tid; i < nc; i += nt) {
      const uint2 c = cand[i];
      if (c.x > thr) atomicOr(&keep[c.y >> 5], 1u << (c.y & 31));
      else if (c.x == thr) atomicOr(&eqb[c.y >> 5], 1u << (c.y & 31));
    }
    __syncthreads();
    {
      const int words = (total + 31) / 32;
      const int chunk = (words + nt - 1) / nt;
      const int w0 = min(words, tid * chunk), w1 = min(words, w0 + chunk);
      uint32_t mine = 0;
      for (int w = w0; w < w1; ++w) mine += __popc(eqb[w]);
      uint32_t incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (lane == 31) sc.scan_eq[warp] = incl;
      __syncthreads();
      if (warp == 0) {
        uint32_t we = lane < warps ? sc.scan_eq[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t v = __shfl_up_sync(0xffffffffu, we, o);
          if (lane >= o) we += v;
        }
        sc.scan_eq[lane] = we;
      }
      __syncthreads();
      uint32_t before = incl - mine + (warp > 0 ? sc.scan_eq[warp - 1] : 0u);
      for (int w = w0; w < w1; ++w) {
        uint32_t bits = eqb[w];
        while (bits) {
          const int b = __ffs(bits) - 1;
          bits &= bits - 1u;
          if (before < need_eq) keep[w] |= 1u << b;
          ++before;
        }
      }
    }
    __syncthreads();
    // 4. warp h: head h's kept pages in ascending order
    for (int h = warp; h < sh.Hkv; h += warps) {
      const int p0 = h * np, p1 = p0 + np;
      int cnt = 0;
      for (int wb = p0 >> 5; wb <= (p1 - 1) >> 5; wb += 32) {
        const int w = wb + lane;
        uint32_t bits = 0u;
        if (w <= (p1 - 1) >> 5) {
          bits = keep[w];
          const int lo = max(p0 - w * 32, 0), hi = min(p1 - w * 32, 32);  // bits [lo, hi) of this head
          const uint32_t mhi = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
          bits &= mhi & ~((1u << lo) - 1u);
        }
        const int c = __popc(bits);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        int pos = cnt + incl - c;
        while (bits) {
          const int b = __ffs(bits) - 1;
          bits &= bits - 1u;
          if (pos < sh.kmax) out[(size_t)h * sh.kmax + pos] = w * 32 + b - p0;
          ++pos;
        }
        cnt += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) s_base[h + 1] = cnt;  // (a count here; prefix below)
    }
    __syncthreads();
    if (tid == 0) {
      s_base[0] = 0;
      for (int h = 0; h < sh.Hkv; ++h) s_base[h + 1] += s_base[h];
    }
    __syncthreads();
    finish_counts();
    return;
  }

  // general path: every pass reads the keys from L2
  uint32_t thr = 0u, need_eq = (uint32_t)total;  // take == total: every pair (keys >= 0)
  if (take == 0) {
    thr = 0xffffffffu;  // above every key: none kept
    need_eq = 0u;
  } else if (take < total) {
    radix_threshold(total, take, key_at, sc, thr, need_eq);
  }
  if (tid == 0) s_base[sh.Hkv] = take;
  if (np == 0) {
    for (int h = tid; h < sh.Hkv; h += blockDim.x) s_base[h] = 0;
  } else {
    ordered_visit(total, thr, need_eq, key_at, [&](int i, int before, bool) {
      if (i % np == 0) s_base[i / np] = before;
    }, sc);
  }
  __syncthreads();
  if (take > 0) {
    ordered_visit(total, thr, need_eq, key_at, [&](int i, int before, bool kept) {
      if (!kept) return;
      const int h = i / np, pos = before - s_base[h];
      if (pos < sh.kmax) out[(size_t)h * sh.kmax + pos] = i - h * np;
    }, sc);
  }
  finish_counts();
}

template <int D, int PAGE>
cudaError_t launch_typed(const Shape &sh, const SelectPlan &plan, const SelectArgs &a,
                         cudaStream_t stream) {
  PartialParams pp{sh, plan, a, 0};
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
  constexpr auto kern = select_fused<D, PAGE>;
  constexpr size_t smem = tc::Layout<D, kSelStages>::kAlloc;
  err = set_smem_once<kern>(smem);
  if (err != cudaSuccess) return err;
  // The group barrier needs the CTAs of a group co-resident.  A group of at most
  // 16 CTAs is one thread-block cluster (co-scheduled by the hardware; groups do
  // not wait for one another, so kernels of other streams run beside them); a
  // larger group needs a cooperative launch, which holds the device for itself.
  // The cooperative launch is also a programmatic dependent of the kernel ahead
  // on the stream (its set-up overlaps that kernel's tail); the clustered one is
  // not: a dependent's CTAs would take SMs while they wait, the SMs that the
  // kernels of another stream use when the pass is held to part of the device
  // (dsa_dims.sm_limit) to run beside them.
  const bool clustered = plan.group_ctas <= 16;
  if (clustered) {
    static unsigned long long big_done = 0;  // bit per device ordinal < 64
    int dev = 0;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
    if (!bit || !(__atomic_load_n(&big_done, __ATOMIC_ACQUIRE) & bit)) {
      if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) !=
          cudaSuccess)
        return err;
      if (bit) __atomic_fetch_or(&big_done, bit, __ATOMIC_ACQ_REL);
    }
  }
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  if (clustered) {
    attrs[1].id = cudaLaunchAttributeClusterDimension;
    attrs[1].val.clusterDim.x = plan.group_ctas;
    attrs[1].val.clusterDim.y = 1;
    attrs[1].val.clusterDim.z = 1;
  } else {
    attrs[1].id = cudaLaunchAttributeCooperative;
    attrs[1].val.cooperative = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.stream = stream;
  cfg.attrs = clustered ? attrs + 1 : attrs;
  cfg.numAttrs = clustered ? 1 : 2;
  cfg.blockDim = dim3(tc::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  const int groups = sh.S * sh.Hkv;
  for (int g0 = 0; g0 < groups; g0 += plan.groups_per_launch) {
    pp.group0 = g0;
    cfg.gridDim = dim3(std::min(plan.groups_per_launch, groups - g0) * plan.group_ctas, 1, 1);
    err = cudaLaunchKernelEx(&cfg, kern, pp, kmap, vmap, kmap4, vmap4);
    if (err != cudaSuccess) return err;
  }
  if (sh.head_budget) {  // the selection over all KV heads of each sequence
    cfg.attrs = attrs;  // programmatic dependent only
    cfg.numAttrs = 1;
    err = set_smem_once<select_global_topk>(kGlobalSmem);
    if (err != cudaSuccess) return err;
    cfg.gridDim = dim3(sh.S, 1, 1);
    cfg.blockDim = dim3(kGlobalThreads, 1, 1);
    cfg.dynamicSmemBytes = kGlobalSmem;
    err = cudaLaunchKernelEx(&cfg, select_global_topk, pp);
    if (err != cudaSuccess) return err;
  }
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
  // rows of the tile maxima / unit masses padded to 4 (16-byte aligned tile blocks)
  p.bgp = (sh.BG + 3) & ~3;
  // candidate list of a CTA: kp <= 128 keeps a power of two >= 32 of them
  if (sh.kmax <= kFastTopk) {
    p.slot_len = 32;
    while (p.slot_len < sh.kmax) p.slot_len *= 2;
  } else {
    p.slot_len = sh.kmax;
  }
  // head-adaptive budget: a CTA's list holds up to 128 keys (kh <= 128) or up to
  // the pages of its split (kh > 128), whatever kmax is
  if (sh.head_budget)
    p.slot_len = std::max(p.slot_len, std::max(kFastTopk, p.tiles_per_split * (tc::kBN / std::min(sh.P, tc::kBN))));
  // groups of one launch: all of their CTAs resident at once
  p.group_ctas = p.splits * p.rowtiles;
  p.groups_per_launch = (int)std::max(1LL, std::min<long long>(kMaxGroupsPerLaunch, num_sms / p.group_ctas));
  const long long groups = (long long)sh.S * sh.Hkv;
  p.groups_per_launch = (int)std::min<long long>(p.groups_per_launch, groups);
  p.launches = (int)((groups + p.groups_per_launch - 1) / p.groups_per_launch);
  auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
  p.off_counters = 256;  // inside the zeroed header, after the status word
  size_t off = kWorkspaceHeader;
  const size_t shn = (size_t)sh.S * sh.Hkv;
  p.off_part_o = off;   off = align(off + shn * p.splits * sh.BG * sh.d * 4);
  p.off_part_ml = off;  off = align(off + shn * p.splits * sh.BG * 2 * 4);
  const size_t units_per_tile = (size_t)tc::kBN / std::min(sh.P, tc::kHalfBN);
  p.off_pagepart = off; off = align(off + shn * p.max_tiles * p.bgp * units_per_tile * 4);
  p.off_mtile = off;    off = align(off + shn * p.max_tiles * p.bgp * 4);
  p.off_scores = off;   off = align(off + shn * sh.max_pages * 4);
  p.off_cand = off;     off = align(off + shn * p.group_ctas * p.slot_len * 8);
  p.off_ccnt = off;     off = align(off + shn * p.group_ctas * 4);
  p.off_hsel = off;     off = align(off + shn * sh.max_pages * 4);
  p.off_hcnt = off;     off = align(off + shn * 4);
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
