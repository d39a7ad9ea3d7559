// sparse.cu -- sparse pass for denoising steps 2..T ("MAGE: All-[MASK] Block
// Already Knows Where to Look in Block Diffusion LLM", Approach: the step-1
// indices are reused for every later step).  Each query row of the block attends
// to the tokens of the selected pages of its KV head plus the block's own B
// tokens, with no mask inside the block.
//
// One launch per step.  A thread-block cluster of C CTAs serves one (sequence,
// KV head, 128-row tile): CTAs 0..C-2 run the tcgen05 engine (tc_attn.cuh) over
// even slices (whole tiles) of the head's own count of selected pages, gathered
// with TMA through the page table; CTA C-1 takes the block's own tokens (a 3-D
// TMA box over blk_k / blk_v).  The C partial results are then merged: every
// softmax thread writes its row, normalised, in fp16 with the row's (m, l), to
// this cluster's exchange area in the workspace (L2); after one cluster barrier
// (release / acquire) the CTA that owns a row combines its C contributions and
// writes o_out in bf16.  The cluster only provides the co-scheduling and the
// barrier: going through L2 moves the partial rows faster than stores into the
// owners' shared memory.  With dims.active (reuse of the prefix part of stable
// tokens, "LoSA: Locality Aware Sparse Attention for Block-Wise Diffusion
// Language Models", abstract) the page contributions form the prefix part, which
// is taken from or written to the caches and then merged with the block part.
#include <cuda_fp16.h>

#include <algorithm>

#include "launch.h"
#include "sm100.cuh"
#include "tc_attn.cuh"

namespace dsa {
namespace {

constexpr int kRowsPerCta = 128;
constexpr int kMaxCluster = 16;

// Shared memory beyond the engine's layout: the CTA's page table (int2 per
// entry) and a uint64 key mask per page tile.  Exchange area of one cluster in
// the workspace: kMaxCluster slots (one per CTA), each the CTA's 128 partial rows
// as [D/8 column chunks][128 rows][16 bytes] of fp16 (so a warp's stores of one
// chunk are contiguous) followed by [128 rows] of (m, l) in fp32.
template <int D, int STG>
struct SparseLayout {
  static constexpr uint32_t kSlotBytes = 128u * (2u * D + 8u);
  static __host__ __device__ constexpr uint32_t align16(uint32_t x) { return (x + 15u) & ~15u; }
  static __host__ __device__ constexpr uint32_t table_offset() {
    return align16(tc::Layout<D, STG>::kBytes);
  }
  static __host__ __device__ constexpr uint32_t mask_offset(int ppc) {
    return table_offset() + 8u * (uint32_t)ppc;
  }
  static __host__ __device__ constexpr size_t smem(int ppc) {
    return mask_offset(ppc) + 8u * (uint32_t)ppc + 1024u;  // + alignment slack
  }
};

struct SparseParams {
  Shape sh;
  SparsePlan plan;
  SparseArgs a;
};

template <int D, int PAGE>
struct SparsePolicy {
  // warp 0 resolves the CTA's selected pages into a shared-memory table of
  // (logical page, physical page) and a key mask per page tile during set-up,
  // before it issues the first loads; the other warps read both after the
  // CTA-wide barrier
  static constexpr bool kIssueBeforeSync = true;
  static constexpr int kPagesPerTile = tc::kBN / PAGE;
  static constexpr int kHalves = D / 64;
  const CUtensorMap *kmap, *vmap, *kmap4, *vmap4, *bkmap, *bvmap;
  const int32_t *idx_row;       // idx[s, h, :]
  const int32_t *page_row;      // page-table row of the sequence, or null (identity)
  const __nv_bfloat16 *q_head;  // q[s, 0, h*G, 0]
  uint32_t *status;
  const int2 *tab;              // shared: (lp, phys) per entry of this CTA, phys < 0 = unusable
  const uint64_t *masks;        // shared: key mask of each page tile
  uint32_t tab_off, mask_off;   // byte offsets in the aligned shared memory
  int lp_spec;                  // warp 0: idx[s, h, c*ppc + lane], loaded with idx_cnt (-2: not this slice)
  long long n_phys, phys0;
  int Hkv, h, G, Hq, B, BG, s, n, np, e_begin, e_end, sel_tiles, row_base;
  float sl2;

  __device__ __forceinline__ int2 resolve_lp(int lp) const {
    int phys = -1;
    if (lp >= 0 && lp < np) {
      const long long p = page_row ? (long long)page_row[lp] : phys0 + lp;
      if (p >= 0 && p < n_phys) phys = (int)p;
    }
    return make_int2(lp, phys);
  }
  __device__ __forceinline__ void prepare(unsigned char *smem) {
    int2 *t = reinterpret_cast<int2 *>(smem + tab_off);
    uint64_t *mk = reinterpret_cast<uint64_t *>(smem + mask_off);
    tab = t;
    masks = mk;
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    // e_begin == c * ppc whenever the slice is not empty and lp_spec != -2, so
    // entry i = lane of the first pass is then the one loaded speculatively
    for (int i = lane; i < e_end - e_begin; i += 32) {
      const int lp = (i == lane && lp_spec != -2) ? lp_spec : idx_row[e_begin + i];
      const int2 v = resolve_lp(lp);
      if (v.y < 0) raise_status(status, kStatusBadIndex);
      t[i] = v;
    }
    __syncwarp();
    for (int k = lane; k < sel_tiles; k += 32) {
      uint64_t m = 0;
#pragma unroll
      for (int pi = 0; pi < kPagesPerTile; ++pi) {
        const int e = e_begin + k * kPagesPerTile + pi;
        if (e >= e_end) continue;
        const int2 v = t[e - e_begin];
        if (v.y < 0) continue;
        const int cnt = min(PAGE, n - v.x * PAGE);
        if (cnt > 0) m |= ((cnt >= 64) ? ~0ull : ((1ull << cnt) - 1ull)) << (pi * PAGE);
      }
      mk[k] = m;
    }
    __syncwarp();
  }
  __device__ __forceinline__ void ready() const {}
  __device__ __forceinline__ void prefetch() const {
    sm100::tma_prefetch_map(kmap);
    sm100::tma_prefetch_map(vmap);
    sm100::tma_prefetch_map(kmap4);
    sm100::tma_prefetch_map(vmap4);
    sm100::tma_prefetch_map(bkmap);
    sm100::tma_prefetch_map(bvmap);
  }
  __device__ __forceinline__ int2 entry(int e) const {
    if (e >= e_end) return make_int2(-1, -1);
    return tab[e - e_begin];
  }
  // Run by all 32 lanes of warp 0: lane 0 arms the barrier, then each box of the
  // tile is issued by a lane of its own (one warp instruction for the tile).
  __device__ __forceinline__ void load_tile(int k, uint32_t sk, uint32_t sv, uint32_t half_bytes,
                                            uint32_t bar, int lane) const {
    if (k < sel_tiles) {
      const int e0 = e_begin + k * kPagesPerTile;
      const int2 my = entry(e0 + (lane < kPagesPerTile ? lane : 0));
      const bool valid = lane < kPagesPerTile && my.y >= 0;
      const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
      const int p0 = __shfl_sync(0xffffffffu, my.y, 0);
      const bool consec = lane >= kPagesPerTile || (valid && my.y == p0 + lane);
      const bool run = kPagesPerTile > 1 && __all_sync(0xffffffffu, consec);
      if (lane == 0)
        sm100::mbar_arrive_expect_tx(bar, (uint32_t)__popc(vmask) * PAGE * 128u * kHalves * 2u);
      if (run) {  // the whole tile in one box per half and tensor
        if (lane < 2 * kHalves) {
          const int hf = lane % kHalves;
          const bool isv = lane >= kHalves;
          sm100::tma_load_4d((isv ? sv : sk) + hf * half_bytes, isv ? vmap4 : kmap4, bar, hf * 64, 0,
                             h, p0);
        }
        return;
      }
      const int pi = lane / (2 * kHalves), rem = lane % (2 * kHalves);
      const int ph = __shfl_sync(0xffffffffu, my.y, pi < kPagesPerTile ? pi : 0);
      if (pi < kPagesPerTile && ((vmask >> pi) & 1u)) {
        const int hf = rem % kHalves;
        const bool isv = rem >= kHalves;
        const int y = (int)(((long long)ph * Hkv + h) * PAGE);
        sm100::tma_load_2d((isv ? sv : sk) + hf * half_bytes + pi * PAGE * 128, isv ? vmap : kmap, bar,
                           hf * 64, y);
      }
    } else {  // the block's own tokens u = 64j .. 64j+63 of this sequence
      const int j = k - sel_tiles;
      if (lane == 0) sm100::mbar_arrive_expect_tx(bar, 64u * 128u * kHalves * 2u);
      if (lane < 2 * kHalves) {
        const int hf = lane % kHalves;
        const bool isv = lane >= kHalves;
        sm100::tma_load_3d((isv ? sv : sk) + hf * half_bytes, isv ? bvmap : bkmap, bar, hf * 64, h,
                           s * B + j * 64);
      }
    }
  }
  __device__ __forceinline__ const __nv_bfloat16 *q_row(int r) const {
    const int row = row_base + r;
    if (row >= BG) return nullptr;
    const int b = row / G, g = row % G;
    return q_head + ((size_t)b * Hq + g) * D;
  }
  __device__ __forceinline__ uint64_t key_mask(int k) const {
    if (k < sel_tiles) return masks[k];
    const int cnt = min(64, B - (k - sel_tiles) * 64);
    return cnt <= 0 ? 0ull : (cnt >= 64 ? ~0ull : ((1ull << cnt) - 1ull));
  }
  __device__ __forceinline__ void after_tile(int, int, float, const float *) const {}
};

template <int D, int PAGE, int STG>
__global__ void __launch_bounds__(tc::kThreads, 1)
    sparse_attn(const __grid_constant__ SparseParams prm, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap kmap4,
                const __grid_constant__ CUtensorMap vmap4, const __grid_constant__ CUtensorMap bkmap,
                const __grid_constant__ CUtensorMap bvmap) {
  using M = SparseLayout<D, STG>;
  extern __shared__ unsigned char smem_raw[];
  const Shape &sh = prm.sh;
  const SparsePlan &plan = prm.plan;
  const SparseArgs &a = prm.a;
  const int C = plan.cluster;   // cluster size == gridDim.x
  const int c = blockIdx.x;     // rank in the cluster
  const int h = blockIdx.y;
  const int s = blockIdx.z / plan.rowtiles, rt = blockIdx.z % plan.rowtiles;
  const size_t sh_idx = (size_t)s * sh.Hkv + h;
  const int row_base = rt * kRowsPerCta;
  const bool blk_cta = c == C - 1;  // CTAs 0..C-2: pages; CTA C-1: the block's own tokens
  constexpr int kPagesPerTile = tc::kBN / PAGE;
  const bool early = sh.early_gather != 0;

  SparsePolicy<D, PAGE> pol;
  pol.kmap = &kmap;
  pol.vmap = &vmap;
  pol.kmap4 = &kmap4;
  pol.vmap4 = &vmap4;
  pol.bkmap = &bkmap;
  pol.bvmap = &bvmap;
  if (threadIdx.x == 0) DSA_TRACE_EVENT(0);
  tc::Engine<D, STG> eng;
  eng.setup(smem_raw, pol);
  if (threadIdx.x == 0) DSA_TRACE_EVENT(32);

  const int32_t *idx_row = a.idx + sh_idx * sh.kmax;
  pol.idx_row = idx_row;
  pol.page_row = sh.page_table ? sh.page_table + (size_t)s * sh.max_pages : nullptr;
  pol.q_head = a.q + ((size_t)s * sh.B * sh.Hq + (size_t)h * sh.G) * D;
  pol.status = a.status;
  pol.tab = nullptr;
  pol.masks = nullptr;
  pol.tab_off = M::table_offset();
  pol.mask_off = M::mask_offset(plan.ppc);
  pol.n_phys = sh.n_phys;
  pol.phys0 = (long long)s * sh.max_pages;
  pol.Hkv = sh.Hkv;
  pol.h = h;
  pol.G = sh.G;
  pol.Hq = sh.Hq;
  pol.B = sh.B;
  pol.BG = sh.BG;
  pol.s = s;
  pol.row_base = row_base;
  pol.sl2 = sh.sl2;

  // The key side of the step: the prefix length, the count and (warp 0 of a page
  // CTA) this CTA's slice of idx are loaded together (idx entries below kmax are
  // always readable; the ones beyond the count are ignored), then this CTA's
  // share of the pages.  With early gathering this runs before the dependency
  // wait, else after it.
  int num_tiles = 0;
  auto key_side = [&]() {
    const int n_raw = a.n_ctx[s];
    int cnt = a.idx_cnt[sh_idx];
    int lp_spec = -1;
    if (threadIdx.x < 32 && !blk_cta) {
      const int e = c * plan.ppc + (int)threadIdx.x;
      if ((int)threadIdx.x < plan.ppc && e < sh.kmax) lp_spec = idx_row[e];
    }
    const bool reporter = threadIdx.x == 0 && c == 0 && rt == 0;
    const int n = clamp_prefix(n_raw, sh.max_pages, PAGE, a.status, reporter && h == 0);
    if (cnt < 0 || cnt > sh.kmax) {
      if (reporter) raise_status(a.status, kStatusBadIndex);
      cnt = max(0, min(cnt, sh.kmax));
    }
    if (sh.active && !blk_cta) {
      // prefix-part reuse: a row tile whose tokens are all stable needs no page
      // (each warp checks the tile's tokens itself: a warp-uniform answer)
      const int lane = threadIdx.x & 31;
      const int b0 = row_base / sh.G, b1 = min(sh.B, (row_base + kRowsPerCta + sh.G - 1) / sh.G);
      bool any = false;
      for (int b = b0 + lane; b < b1; b += 32) any |= sh.active[(size_t)s * sh.B + b] != 0;
      if (!__any_sync(0xffffffffu, any)) cnt = 0;
    }
    if (threadIdx.x == 0) DSA_TRACE_AFTER(34, cnt + n);
    // the page CTAs split this head's cnt pages evenly, in whole tiles (counts
    // differ per head under the head-adaptive budget); ppc_eff = plan.ppc when
    // cnt = kmax, and then the speculative idx load above is this CTA's slice
    const int ppc_eff =
        min(plan.ppc, ((cnt + C - 2) / (C - 1) + kPagesPerTile - 1) / kPagesPerTile * kPagesPerTile);
    const int e_begin = blk_cta ? cnt : min(cnt, c * ppc_eff);
    const int e_end = blk_cta ? cnt : min(cnt, (c + 1) * ppc_eff);
    if (ppc_eff != plan.ppc) lp_spec = -2;  // not this slice's: prepare() loads it again
    const int sel_tiles = (e_end - e_begin + kPagesPerTile - 1) / kPagesPerTile;
    num_tiles = sel_tiles + (blk_cta ? plan.blk_tiles : 0);
    pol.lp_spec = lp_spec;
    pol.n = n;
    pol.np = (n + PAGE - 1) / PAGE;
    pol.e_begin = e_begin;
    pol.e_end = e_end;
    pol.sel_tiles = sel_tiles;
  };

  if (early) {
    // everything the key side reads is, by the caller's contract, not written by
    // the kernel ahead of this one: a page CTA builds its tables and has its
    // first STG tiles in flight before the wait
    key_side();
    if (!blk_cta) eng.stage(pol, num_tiles);
  }
  // While the kernel ahead of this one may still run: L2 prefetches of what this
  // CTA will read.  Without early gathering the page list is read here without
  // any ordering (through L2 only, so that no stale line stays in L1) and serves
  // only as prefetch addresses, clamped to the cache; everything the computation
  // uses is read again after grid_dep_wait().  Warp 1 (the MMA issuer, idle until
  // the first tiles land) and the softmax warps do this, not the producer.
  if (eng.warp == 1) {
    const int lane = eng.lane;
    if (blk_cta) {
      const __nv_bfloat16 *bk = a.blk_k + ((size_t)s * sh.B * sh.Hkv + h) * D;
      const __nv_bfloat16 *bv = a.blk_v + ((size_t)s * sh.B * sh.Hkv + h) * D;
      for (int u = lane; u < sh.B; u += 32) {
        sm100::prefetch_l2_bulk(bk + (size_t)u * sh.Hkv * D, D * 2);
        sm100::prefetch_l2_bulk(bv + (size_t)u * sh.Hkv * D, D * 2);
      }
    } else if (!early) {
      const int e = c * plan.ppc + lane;
      if (lane < plan.ppc && e < sh.kmax) {
        const int lp = __ldcg(a.idx + sh_idx * sh.kmax + e);
        if (lp >= 0 && lp < sh.max_pages) {
          const long long ph = sh.page_table ? (long long)__ldcg(sh.page_table + (size_t)s * sh.max_pages + lp)
                                             : (long long)s * sh.max_pages + lp;
          if (ph >= 0 && ph < sh.n_phys) {
            const size_t off = ((size_t)ph * sh.Hkv + h) * PAGE * D;
            sm100::prefetch_l2_bulk(a.k + off, PAGE * D * 2);
            sm100::prefetch_l2_bulk(a.v + off, PAGE * D * 2);
          }
        }
      }
    }
  } else if (eng.warp >= 2) {  // this thread's half of its query row
    const int row = row_base + eng.row_in_tile();
    if (row < sh.BG) {
      const int b = row / sh.G, g = row % sh.G;
      sm100::prefetch_l2(a.q + (((size_t)s * sh.B + b) * sh.Hq + (size_t)h * sh.G + g) * D +
                         eng.group() * (D / 2));
    }
  }
  // everything below may read what the kernel ahead of this one wrote
  sm100::grid_dep_wait();
  sm100::grid_dep_launch_dependents();
  if (threadIdx.x == 0) DSA_TRACE_EVENT(33);
  if (!early) key_side();
  eng.init(a.status, pol, num_tiles, early && !blk_cta);
  // rows this CTA owns in the merge
  const int rpc = (kRowsPerCta + C - 1) / C;
  const int r0 = c * rpc;
  const int nrows = max(0, min(kRowsPerCta, r0 + rpc) - r0);

  float m, l;
  eng.template run<PAGE>(pol, num_tiles, m, l);
  float m_row, l_row, wa, wb;
  eng.finish(m, l, m_row, l_row, wa, wb);

  // ---- exchange: each softmax thread writes its half of its row, normalised
  //      (O / l) in fp16, to this CTA's slot of the cluster's exchange area; the
  //      group-0 thread adds the row's (m, l)
  unsigned char *xc = a.xchg + (((size_t)s * sh.Hkv + h) * plan.rowtiles + rt) * kMaxCluster * M::kSlotBytes;
  if (eng.warp >= 2) {
    const int r = eng.row_in_tile();
    const int g = eng.group();
    unsigned char *slot = xc + (size_t)c * M::kSlotBytes;
    const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
    const float ca = wa * inv, cb = wb * inv;
#pragma unroll
    for (int c0 = g * (D / 2); c0 < (g + 1) * (D / 2); c0 += 32) {
      uint32_t oa[32], ob[32];
      eng.load_o2(c0, oa, ob);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v;
        uint32_t *pv = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float f[2];
#pragma unroll
          for (int z = 0; z < 2; ++z) {
            const int i = 8 * q + 2 * e + z;
            // an empty group (weight 0) may hold stale TMEM: never multiply it
            f[z] = (ca > 0.f ? ca * __uint_as_float(oa[i]) : 0.f) +
                   (cb > 0.f ? cb * __uint_as_float(ob[i]) : 0.f);
          }
          __half2 hv = __floats2half2_rn(f[0], f[1]);
          pv[e] = *reinterpret_cast<uint32_t *>(&hv);
        }
        const int ch = c0 / 8 + q;
        *reinterpret_cast<uint4 *>(slot + ((size_t)ch * kRowsPerCta + r) * 16) = v;
      }
    }
    if (g == 0)
      *reinterpret_cast<float2 *>(slot + (size_t)kRowsPerCta * 2 * D + r * 8) = make_float2(m_row, l_row);
    if (r == 0 && g == 0) DSA_TRACE_EVENT(7);
  }
  sm100::cluster_arrive();  // release: this CTA's partial rows are written
  sm100::cluster_wait();    // acquire: so are those of every CTA of the cluster
  if (threadIdx.x == 0) DSA_TRACE_EVENT(9);

  // ---- merge the rows this CTA owns: a work item (row, 8 columns) loads the C
  //      contributions' (m, l) and values at once (L2 only: they come from other
  //      SMs), then weighs them with 2^(m_j - M) l_j / L.  Consecutive threads
  //      take consecutive rows of one column chunk, so that their loads are
  //      contiguous in the chunk-major slots.
  const int rows_here = min(kRowsPerCta, sh.BG - row_base);
  constexpr int kChunks = D / 8;  // 8 values (16 bytes of fp16) per work item
  for (int t = threadIdx.x; t < nrows * kChunks; t += blockDim.x) {
    const int rl = t % nrows, ch = t / nrows;
    const int row = r0 + rl;
    if (row >= rows_here) continue;
    float2 st[kMaxCluster];
    uint4 v[kMaxCluster];
#pragma unroll
    for (int j = 0; j < kMaxCluster; ++j) {
      if (j < C) {
        const unsigned char *slot = xc + (size_t)j * M::kSlotBytes;
        st[j] = __ldcg(reinterpret_cast<const float2 *>(slot + (size_t)kRowsPerCta * 2 * D + row * 8));
        const int4 x = __ldcg(reinterpret_cast<const int4 *>(slot + ((size_t)ch * kRowsPerCta + row) * 16));
        v[j] = make_uint4((uint32_t)x.x, (uint32_t)x.y, (uint32_t)x.z, (uint32_t)x.w);
      } else {
        st[j] = make_float2(-INFINITY, 0.f);
        v[j] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    const int grow = row_base + row;
    const int b = grow / sh.G, g = grow % sh.G;
    const size_t orow = ((size_t)s * sh.B + b) * sh.Hq + (size_t)h * sh.G + g;
    if (sh.active) {
      // prefix-part reuse: the page contributions (all but the last) merge into
      // the prefix part; an active token keeps it and writes it to the cache, a
      // stable one takes the cache's instead; then prefix and block part merge
      float mp = -INFINITY;
#pragma unroll
      for (int j = 0; j < kMaxCluster - 1; ++j)
        if (j < C - 1 && st[j].y > 0.f) mp = fmaxf(mp, st[j].x);
      float lp = 0.f;
      float op[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < kMaxCluster - 1; ++j) {
        if (j >= C - 1 || !(st[j].y > 0.f)) continue;
        const float w = exp2f(st[j].x - mp) * st[j].y;
        lp += w;
        const __half2 *hv = reinterpret_cast<const __half2 *>(&v[j]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(hv[e]);
          op[2 * e] = fmaf(w, f.x, op[2 * e]);
          op[2 * e + 1] = fmaf(w, f.y, op[2 * e + 1]);
        }
      }
      float m1;  // prefix part: log2-domain log-sum-exp (-inf: empty), values normalised
      __nv_bfloat16 *co = sh.prefix_o + orow * D + ch * 8;
      if (sh.active[(size_t)s * sh.B + b] != 0) {
        const float inv = lp > 0.f ? 1.f / lp : 0.f;
        m1 = lp > 0.f ? mp + log2f(lp) : -INFINITY;
        uint4 cv;
        uint32_t *pc = reinterpret_cast<uint32_t *>(&cv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          op[2 * e] *= inv;
          op[2 * e + 1] *= inv;
          __nv_bfloat162 bv = __floats2bfloat162_rn(op[2 * e], op[2 * e + 1]);
          pc[e] = *reinterpret_cast<uint32_t *>(&bv);
        }
        *reinterpret_cast<uint4 *>(co) = cv;
        if (ch == 0) sh.prefix_lse[orow] = m1 * 0.6931471805599453f;
      } else {
        const float lse_c = sh.prefix_lse[orow];
        m1 = lse_c * 1.4426950408889634f;  // (-inf stays -inf)
        const uint4 cv = *reinterpret_cast<const uint4 *>(co);
        const __nv_bfloat162 *pc = reinterpret_cast<const __nv_bfloat162 *>(&cv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(pc[e]);
          op[2 * e] = f.x;
          op[2 * e + 1] = f.y;
        }
      }
      // the block part: the last contribution
      float2 sb = make_float2(-INFINITY, 0.f);
      uint4 vb = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int j = 0; j < kMaxCluster; ++j)
        if (j == C - 1) {
          sb = st[j];
          vb = v[j];
        }
      const bool has_p = m1 > -INFINITY, has_b = sb.y > 0.f;
      const float mm = fmaxf(has_p ? m1 : -INFINITY, has_b ? sb.x : -INFINITY);
      const float wp = has_p ? exp2f(m1 - mm) : 0.f;
      const float wb = has_b ? exp2f(sb.x - mm) * sb.y : 0.f;
      const float tot = wp + wb;
      const float inv = tot > 0.f ? 1.f / tot : 0.f;
      if (sh.lse_out && ch == 0) sh.lse_out[orow] = tot > 0.f ? (mm + log2f(tot)) * 0.6931471805599453f : -INFINITY;
      const __half2 *hb = reinterpret_cast<const __half2 *>(&vb);
      uint4 outv;
      uint32_t *po = reinterpret_cast<uint32_t *>(&outv);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(hb[e]);
        __nv_bfloat162 bv = __floats2bfloat162_rn((wp * op[2 * e] + wb * f.x) * inv,
                                                  (wp * op[2 * e + 1] + wb * f.y) * inv);
        po[e] = *reinterpret_cast<uint32_t *>(&bv);
      }
      *reinterpret_cast<uint4 *>(a.o_out + orow * D + ch * 8) = outv;
      continue;
    }
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < kMaxCluster; ++j)
      if (st[j].y > 0.f) mx = fmaxf(mx, st[j].x);
    float lsum = 0.f;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kMaxCluster; ++j) {
      if (!(st[j].y > 0.f)) continue;  // an empty contribution
      const float w = exp2f(st[j].x - mx) * st[j].y;
      lsum += w;
      const __half2 *hv = reinterpret_cast<const __half2 *>(&v[j]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(hv[e]);
        acc[2 * e] = fmaf(w, f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(w, f.y, acc[2 * e + 1]);
      }
    }
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    if (sh.lse_out && ch == 0)  // the row's log-sum-exp over its key set: (M + log2 L) ln 2
      sh.lse_out[((size_t)s * sh.B + b) * sh.Hq + (size_t)h * sh.G + g] =
          lsum > 0.f ? (mx + log2f(lsum)) * 0.6931471805599453f : -INFINITY;
    uint4 outv;
    uint32_t *po = reinterpret_cast<uint32_t *>(&outv);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 bv = __floats2bfloat162_rn(acc[2 * e] * inv, acc[2 * e + 1] * inv);
      po[e] = *reinterpret_cast<uint32_t *>(&bv);
    }
    *reinterpret_cast<uint4 *>(a.o_out + (((size_t)s * sh.B + b) * sh.Hq + (size_t)h * sh.G + g) * D +
                               ch * 8) = outv;
  }
  if (threadIdx.x == 0) DSA_TRACE_EVENT(10);
  eng.teardown();
  if (threadIdx.x == 0) DSA_TRACE_EVENT(11);
}

// Clusters of each size (1..kMaxCluster) that can be resident at once with this
// kernel, queried once per device.
template <auto K>
const int *active_clusters(size_t smem) {
  static int cached[64][kMaxCluster + 1];
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (!done[dev]) {
    const bool big =
        cudaFuncSetAttribute(K, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    cudaGetLastError();
    for (int cs = 0; cs <= kMaxCluster; ++cs) {
      cached[dev][cs] = 0;
      if (cs == 0 || (cs > 8 && !big)) continue;
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
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, K, &cfg) == cudaSuccess) cached[dev][cs] = n;
      cudaGetLastError();
    }
    done[dev] = true;
  }
  return cached[dev];
}

// Page CTAs per cluster for `nclusters` clusters sharing `kmax` pages each (one
// more CTA takes the block's own tokens): the count with the smallest
// (waves x tiles of the busiest CTA), more CTAs on ties.
inline int choose_page_ctas(const int *active, int nclusters, int kmax, int page, int blk_tiles) {
  int best = 1;
  long long best_cost = -1;
  for (int cp = kMaxCluster - 1; cp >= 1; --cp) {
    const int cs = cp + 1;
    if (active[cs] < 1) continue;
    const int ppc = (kmax + cp - 1) / cp;
    if (cp > 1 && (long long)(cp - 1) * ppc >= kmax) continue;  // a page CTA would be idle
    const long long tiles = std::max((ppc * page + tc::kBN - 1) / tc::kBN, blk_tiles);
    const long long waves = (nclusters + active[cs] - 1) / active[cs];
    const long long cost = waves * (tiles + 1);  // +1: fixed per-CTA cost
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = cp;
    }
  }
  return best;
}

constexpr size_t kMaxSmem = 227 * 1024;

// Kernel attributes set once per device: the dynamic shared memory and clusters
// beyond the portable 8 CTAs.
template <auto K>
cudaError_t prepare_kernel_once() {
  cudaError_t err = set_smem_once<K>(kMaxSmem);
  if (err != cudaSuccess) return err;
  static unsigned long long done = 0;  // bit per device ordinal < 64
  int dev = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (__atomic_load_n(&done, __ATOMIC_ACQUIRE) & bit)) return cudaSuccess;
  err = cudaFuncSetAttribute(K, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (err == cudaSuccess && bit) __atomic_fetch_or(&done, bit, __ATOMIC_ACQ_REL);
  return err;
}

template <int D, int PAGE, int STG>
cudaError_t launch_staged(const Shape &sh, const SparsePlan &plan, const SparseArgs &a,
                          cudaStream_t stream) {
  using M = SparseLayout<D, STG>;
  constexpr auto kern = sparse_attn<D, PAGE, STG>;
  cudaError_t err = prepare_kernel_once<kern>();
  if (err != cudaSuccess) return err;
  const size_t smem = M::smem(plan.ppc);
  if (smem > kMaxSmem) return cudaErrorInvalidValue;
  CUtensorMap kmap, vmap, kmap4, vmap4, bkmap, bvmap;
  const long long rows = sh.n_phys * sh.Hkv * PAGE;
  if ((err = make_kv_tensor_map(&kmap, a.k, rows, D, PAGE)) != cudaSuccess) return err;
  if ((err = make_kv_tensor_map(&vmap, a.v, rows, D, PAGE)) != cudaSuccess) return err;
  if ((err = make_kv_pages_tensor_map(&kmap4, a.k, sh.n_phys, sh.Hkv, PAGE, D, tc::kBN / PAGE)) !=
      cudaSuccess)
    return err;
  if ((err = make_kv_pages_tensor_map(&vmap4, a.v, sh.n_phys, sh.Hkv, PAGE, D, tc::kBN / PAGE)) !=
      cudaSuccess)
    return err;
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
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = plan.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // the set-up before grid_dep_wait() may overlap the kernel ahead on the stream
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  err = cudaLaunchKernelEx(&cfg, kern, prm, kmap, vmap, kmap4, vmap4, bkmap, bvmap);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

// Cluster shape from the device's cluster capacity, then the stage count: with
// early gathering a page CTA holds all its tiles at once when they fit in four
// stages; otherwise two stages stream them.
template <int D, int PAGE>
cudaError_t launch_typed(const Shape &sh, const SparsePlan &plan_in, const SparseArgs &a,
                         cudaStream_t stream) {
  constexpr auto probe = sparse_attn<D, PAGE, 2>;
  cudaError_t err = prepare_kernel_once<probe>();
  if (err != cudaSuccess) return err;
  SparsePlan plan = plan_in;
  const int *active = active_clusters<probe>(SparseLayout<D, 2>::smem(std::max(sh.kmax, 64)));
  const int cp = choose_page_ctas(active, sh.Hkv * sh.S * plan.rowtiles, sh.kmax, PAGE, plan.blk_tiles);
  plan.cluster = cp + 1;
  plan.ppc = (sh.kmax + cp - 1) / cp;
  const int tiles = (plan.ppc * PAGE + tc::kBN - 1) / tc::kBN;
  if (sh.early_gather && tiles > 2) return launch_staged<D, PAGE, 4>(sh, plan, a, stream);
  return launch_staged<D, PAGE, 2>(sh, plan, a, stream);
}

}  // namespace

DSA_TRACE_EXPORT(dsa_trace_sparse)

SparsePlan plan_sparse(const Shape &sh, int /*num_sms*/) {
  SparsePlan p{};
  p.rowtiles = (sh.BG + kRowsPerCta - 1) / kRowsPerCta;
  p.cluster = kMaxCluster;  // refined at launch from the device's cluster capacity
  p.ppc = (sh.kmax + kMaxCluster - 2) / (kMaxCluster - 1);
  p.blk_tiles = (sh.B + tc::kBN - 1) / tc::kBN;
  p.off_xchg = 4096;  // after the status header
  p.xchg_slot = 128u * (2u * (size_t)sh.d + 8u);
  p.total = p.off_xchg + (size_t)sh.S * sh.Hkv * p.rowtiles * kMaxCluster * p.xchg_slot;
  return p;
}

cudaError_t launch_sparse(const Shape &sh, const SparsePlan &plan, const SparseArgs &a,
                          cudaStream_t stream) {
  cudaError_t err = cudaSuccess;
  if (launch_sparse_resident(sh, a, stream, &err)) return err;
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
