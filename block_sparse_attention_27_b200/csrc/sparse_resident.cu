// sparse_resident.cu -- sparse pass for denoising steps 2..T ("MAGE: All-[MASK]
// Block Already Knows Where to Look in Block Diffusion LLM", Approach: the step-1
// indices are reused for every later step), for shapes in which every CTA can
// hold all of its keys in shared memory at once.  Each query row attends to the
// tokens of the selected pages of its KV head plus the block's own B tokens, with
// no mask inside the block.
//
// One thread-block cluster of C CTAs serves one (sequence, KV head, row tile).
// The head's selected pages are split in whole pages over the C CTAs; the last
// CTA also takes the block's tokens.  A CTA's keys (at most 256) and its query
// tile sit in shared memory together, so a step is one pass with no pipeline:
//   1. key side: the CTA's page-table rows, key mask and the TMA gather of its
//      pages' K and V.  With dims.early_gather this runs before the dependency
//      wait (programmatic dependent launch), while the kernel ahead still runs;
//   2. after the wait: TMA of the query tile (and of the block's K and V);
//   3. S = Q K^T for all the CTA's keys (one MMA chain, N = its keys);
//   4. the softmax of each row over those keys in one pass, no online
//      rescaling: four warpgroups take a quarter of the keys each, meet once for
//      the row max, then write P = 2^(s - max) in bf16 into TMEM over S;
//   5. O = P V into TMEM (one MMA chain);
//   6. each row, normalised (O / l in fp16, a quarter of the columns per
//      warpgroup) with its (max, sum), is stored into the shared memory of the
//      CTA of the cluster that owns the row (distributed shared memory), between
//      two cluster barriers;
//   7. each CTA merges the C contributions of the rows it owns (one pass with a
//      running max per work item) and writes o_out (and lse_out).
// Warp roles (576 threads): warp 0 issues the TMA loads (all lanes) and the MMAs
// (lane 0); warp 1 owns TMEM; warps 2..17 are four warpgroups over the 128 rows
// (TMEM lane = row).  The step is bound by the latency of this chain, so the
// work of each phase is spread over as many warps as TMEM's lane quarters allow.
#include <cuda_fp16.h>

#include <algorithm>

#include "launch.h"
#include "sm100.cuh"
#include "trace.cuh"

namespace dsa {
namespace {

constexpr int kRThreads = 576;
constexpr int kRowWarps = 16;
constexpr int kRMaxCluster = 16;
constexpr int kRMaxKeys = 256;  // keys one CTA holds
constexpr int kWin = 64;        // keys of one warpgroup (a quarter of at most 256)

template <int D>
struct RLayout {
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kQHalf = 128u * 128u;                 // 128 rows x 128 B
  static constexpr uint32_t kKHalf = (uint32_t)kRMaxKeys * 128u;   // 256 keys x 128 B
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kHalves * kQHalf;
  static constexpr uint32_t kOffV = kOffK + kHalves * kKHalf;
  static constexpr uint32_t kOffBar = kOffV + kHalves * kKHalf;   // 5 mbarriers in 8 slots
  static constexpr int kMaxPages = kRMaxKeys / 16;
  static constexpr uint32_t kOffTab = kOffBar + 8u * 8u;          // int2 (lp, phys) per page
  static constexpr uint32_t kOffMask = kOffTab + 8u * kMaxPages;  // one bit per key (+ 2 spare words)
  static constexpr uint32_t kOffRed = kOffMask + kRMaxKeys / 8 + 8u;  // [4 warpgroups][128 rows] fp32
  static constexpr uint32_t kOffMisc = kOffRed + 4u * 128u * 4u;  // TMEM address, abort flag
  static constexpr uint32_t kBytes = kOffMisc + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // room to align the base to 1 KB
  // the merge area lies over Q and K, which are dead once every CTA of the
  // cluster has completed its S MMAs
  static constexpr uint32_t kRecvLimit = kOffV;
  // TMEM: S (and P over it) in columns [0, 256), then O
  static constexpr uint32_t kTmemS = 0;
  static constexpr uint32_t kTmemO = 256;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(D == 64 || D == 128, "head dimension");
};

struct ResidentPlan {
  int cluster;   // C: CTAs per (sequence, KV head, row tile)
  int bpt;       // block tokens per row tile (rows = bpt * G <= 128)
  int rowtiles;  // ceil(B / bpt)
  int bp;        // block tokens rounded up to 16 (MMA granularity)
  int qmax;      // page-equivalents per CTA when every head has kmax pages
};

struct ResidentParams {
  Shape sh;
  ResidentPlan plan;
  SparseArgs a;
};

// Bytes of the merge area for C CTAs and rpc rows owned per CTA: fp16 rows, then
// (max, sum) per row and contribution.
template <int D>
__host__ __device__ constexpr uint32_t recv_bytes(int C, int rpc) {
  return (uint32_t)C * rpc * (uint32_t)(2 * D + 8);
}

// First key of warpgroup k's quarter of n keys, in 16-key blocks (the quarters
// differ by at most one block).
__device__ __forceinline__ int quarter_start(int n, int k) { return 16 * ((n / 16) * k / 4); }

template <int D, int PAGE>
__global__ void __launch_bounds__(kRThreads, 1)
    sparse_resident(const __grid_constant__ ResidentParams prm, const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap qmap,
                    const __grid_constant__ CUtensorMap bkmap, const __grid_constant__ CUtensorMap bvmap) {
  using L = RLayout<D>;
  using namespace sm100;
  extern __shared__ unsigned char smem_raw[];
  const Shape &sh = prm.sh;
  const ResidentPlan &plan = prm.plan;
  const SparseArgs &a = prm.a;
  const int C = plan.cluster;
  const int c = blockIdx.x;  // rank in the cluster
  const int h = blockIdx.y;
  const int s = blockIdx.z / plan.rowtiles, rt = blockIdx.z % plan.rowtiles;
  const size_t sh_idx = (size_t)s * sh.Hkv + h;
  const bool blk_cta = c == C - 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool early = sh.early_gather != 0;

  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char *smem = smem_raw + (base - raw);
  const uint32_t bar_kv = base + L::kOffBar;  // pages
  const uint32_t bar_q = bar_kv + 8;           // query tile (+ block keys)
  const uint32_t bar_s = bar_kv + 16;          // S complete
  const uint32_t bar_p = bar_kv + 24;          // P written (all row threads)
  const uint32_t bar_o = bar_kv + 32;          // O complete
  int2 *tab = reinterpret_cast<int2 *>(smem + L::kOffTab);
  uint32_t *mask = reinterpret_cast<uint32_t *>(smem + L::kOffMask);
  float *red = reinterpret_cast<float *>(smem + L::kOffRed);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
  const WaitCtx ctx{abort_flag, a.status};
  volatile int never = 0;
  const WaitCtx drain_ctx{&never, a.status};

  if (threadIdx.x == 0) DSA_TRACE_EVENT(0);
  // ---- set-up that reads nothing the caller passes
  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    mbar_init(bar_q, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_p, kRowWarps * 32);
    mbar_init(bar_o, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&kmap);
    tma_prefetch_map(&vmap);
    tma_prefetch_map(&qmap);
    tma_prefetch_map(&bkmap);
    tma_prefetch_map(&bvmap);
  }
  if (warp == 1) {
    tmem_alloc(base + L::kOffMisc, L::kTmemCols);
    tmem_relinquish();
  }

  // ---- key side: this CTA's pages [pb, pb + npg) of the head's cnt, whole pages;
  //      the last CTA also takes the block's B tokens (bp rows, the rest masked)
  int pb = 0, npg = 0, nkeys = 0;
  auto key_side = [&]() {
    const int32_t *idx_head = a.idx + sh_idx * sh.kmax;
    // this CTA's slice when the head has all kmax pages, loaded with the count
    const int spec_e = c * plan.qmax + lane;
    int lp_spec = -1;
    if (warp == 0 && lane < plan.qmax && spec_e < sh.kmax) lp_spec = idx_head[spec_e];
    const int n_raw = a.n_ctx[s];
    int cnt = a.idx_cnt[sh_idx];
    const bool reporter = threadIdx.x == 0 && c == 0 && rt == 0;
    const int n = clamp_prefix(n_raw, sh.max_pages, PAGE, a.status, reporter && h == 0);
    if (cnt < 0 || cnt > sh.kmax) {
      if (reporter) raise_status(a.status, kStatusBadIndex);
      cnt = max(0, min(cnt, sh.kmax));
    }
    const int bu = (plan.bp + PAGE - 1) / PAGE;
    const int q = (cnt + bu + C - 1) / C;
    pb = min(cnt, c * q);
    const int pe = blk_cta ? cnt : min(cnt, (c + 1) * q);
    npg = pe - pb;
    nkeys = npg * PAGE + (blk_cta ? plan.bp : 0);
    if (warp != 0) return;
    // warp 0: page-table rows, the gather, then the key mask
    const int32_t *page_row = sh.page_table ? sh.page_table + (size_t)s * sh.max_pages : nullptr;
    const int np = (n + PAGE - 1) / PAGE;
    const bool spec_ok = pb == c * plan.qmax;
    int nvalid = 0;
    for (int e = lane; e < npg; e += 32) {
      const int lp = (spec_ok && e == lane) ? lp_spec : idx_head[pb + e];
      int phys = -1;
      if (lp >= 0 && lp < np) {
        const long long p = page_row ? (long long)page_row[lp] : (long long)s * sh.max_pages + lp;
        if (p >= 0 && p < sh.n_phys) phys = (int)p;
      }
      if (phys < 0) raise_status(a.status, kStatusBadIndex);
      nvalid += phys >= 0;
      tab[e] = make_int2(lp, phys);
    }
    nvalid = __reduce_add_sync(0xffffffffu, nvalid);
    if (lane == 0) mbar_arrive_expect_tx(bar_kv, (uint32_t)nvalid * PAGE * 128u * L::kHalves * 2u);
    __syncwarp();
    // one box per (page, half, K|V), one lane each
    for (int i = lane; i < npg * L::kHalves * 2; i += 32) {
      const int e = i / (L::kHalves * 2), r = i % (L::kHalves * 2);
      const int hf = r % L::kHalves;
      const bool isv = r >= L::kHalves;
      const int phys = tab[e].y;
      if (phys < 0) continue;
      tma_load_2d(base + (isv ? L::kOffV : L::kOffK) + hf * L::kKHalf + e * PAGE * 128u, isv ? &vmap : &kmap,
                  bar_kv, hf * 64, (int)(((long long)phys * sh.Hkv + h) * PAGE));
    }
    // key mask, 32 keys per ballot, and two zero words past the last key
    for (int k0 = 0; k0 < kRMaxKeys + 64; k0 += 32) {
      const int k = k0 + lane;
      bool on = false;
      if (k < npg * PAGE) {
        const int2 t = tab[k / PAGE];
        on = t.y >= 0 && t.x * PAGE + (k % PAGE) < n;
      } else if (blk_cta && k < kRMaxKeys) {
        on = k - npg * PAGE < sh.B;
      }
      const uint32_t bits = __ballot_sync(0xffffffffu, on);
      if (lane == 0) mask[k0 >> 5] = bits;
    }
  };

  const int b0 = rt * plan.bpt;
  const int rows_here = max(0, min(plan.bpt, sh.B - b0)) * sh.G;
  if (early) key_side();
  if (threadIdx.x == 0) DSA_TRACE_EVENT(32);
  // L2 prefetch of the query tile (and the block's tokens): hints only, they may
  // name memory the kernel ahead of this one is still writing
  if (warp == 1) {
    for (int bb = lane; bb < min(plan.bpt, sh.B - b0); bb += 32)
      prefetch_l2_bulk(a.q + (((size_t)s * sh.B + b0 + bb) * sh.Hq + (size_t)h * sh.G) * D, sh.G * D * 2);
    if (blk_cta)
      for (int u = lane; u < sh.B; u += 32) {
        prefetch_l2_bulk(a.blk_k + (((size_t)s * sh.B + u) * sh.Hkv + h) * D, D * 2);
        prefetch_l2_bulk(a.blk_v + (((size_t)s * sh.B + u) * sh.Hkv + h) * D, D * 2);
      }
  }
  // everything below may read what the kernel ahead of this one wrote
  grid_dep_wait();
  grid_dep_launch_dependents();
  if (threadIdx.x == 0) DSA_TRACE_EVENT(33);
  if (!early) key_side();

  // ---- the query tile, and the block's K and V for the last CTA
  if (warp == 0 && nkeys > 0) {
    const uint32_t qbytes = (uint32_t)plan.bpt * sh.G * 128u * L::kHalves;
    const uint32_t bbytes = blk_cta ? (uint32_t)plan.bp * 128u * L::kHalves * 2u : 0u;
    if (lane == 0) mbar_arrive_expect_tx(bar_q, qbytes + bbytes);
    __syncwarp();
    if (lane < L::kHalves) {
      tma_load_3d(base + L::kOffQ + lane * L::kQHalf, &qmap, bar_q, lane * 64, h * sh.G, s * sh.B + b0);
    } else if (blk_cta && lane >= 8 && lane < 8 + 2 * L::kHalves) {
      const int r = lane - 8, hf = r % L::kHalves;
      const bool isv = r >= L::kHalves;
      tma_load_3d(base + (isv ? L::kOffV : L::kOffK) + hf * L::kKHalf + npg * PAGE * 128u, isv ? &bvmap : &bkmap,
                  bar_q, hf * 64, h, s * sh.B);
    }
  }
  tc_fence_before();
  __syncthreads();  // tables, mask and the TMEM address are visible from here on
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + L::kOffMisc);
  if (threadIdx.x == 0) DSA_TRACE_EVENT(1);

  // rows this CTA owns in the merge, and the merge area's layout (offsets)
  const int rpc = (rows_here + C - 1) / C;
  const uint32_t recv_data = L::kOffQ;                                       // [C][rpc][D/8][16 B]
  const uint32_t recv_ml = recv_data + (uint32_t)C * rpc * (uint32_t)D * 2u; // [C][rpc] (m, l)
  const float sl2 = sh.sl2;

  if (warp == 0) {
    // ------------------------------------------------------------ MMA issuer --
    bool issued_s = false;
    if (lane == 0 && nkeys > 0 && mbar_wait(bar_kv, 0, ctx) && mbar_wait(bar_q, 0, ctx)) {
      tc_fence_after();
      DSA_TRACE_EVENT(3);
      const uint32_t ids = idesc_bf16(128, nkeys, false, false);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t hf = kk >> 2, sub = kk & 3;
        const uint64_t ad = sdesc_sw128(base + L::kOffQ + hf * L::kQHalf + sub * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(base + L::kOffK + hf * L::kKHalf + sub * 32, 16, 1024);
        umma_bf16(tmem + L::kTmemS, ad, bd, ids, kk > 0 ? 1u : 0u);
      }
      umma_commit(bar_s);
      issued_s = true;
    }
    issued_s = __shfl_sync(0xffffffffu, issued_s, 0);
    if (issued_s) mbar_wait(bar_s, 0, drain_ctx);  // Q and K are no longer read
    __syncwarp();
    cluster_arrive();  // phase A
    if (lane == 0 && issued_s && mbar_wait(bar_p, 0, ctx)) {
      tc_fence_after();
      DSA_TRACE_EVENT(26);
      // P of warpgroup k's keys sits at columns [k0, k0 + (k1 - k0) / 2) of its
      // own quarter; 16 keys take 8 columns
      const uint32_t ido = idesc_bf16(128, D, false, true);
      for (int k = 0; k < 4; ++k) {
        const int k0 = quarter_start(nkeys, k), k1 = quarter_start(nkeys, k + 1);
        for (int kb = k0; kb < k1; kb += 16) {
          const uint64_t bd = sdesc_sw128(base + L::kOffV + kb * 128, L::kKHalf, 1024);
          umma_bf16_ts(tmem + L::kTmemO, tmem + L::kTmemS + k0 + (kb - k0) / 2, bd, ido, kb > 0 ? 1u : 0u);
        }
      }
      umma_commit(bar_o);
      mbar_wait(bar_o, 0, drain_ctx);  // every issued MMA completes before TMEM is freed
    }
    __syncwarp();
    cluster_wait();
  } else if (warp == 1) {
    cluster_arrive();  // phase A (this warp reads neither Q nor K)
    cluster_wait();
  } else {
    // ------------------------------------------------------ row threads --
    const int k = (warp - 2) >> 2;      // warpgroup: a quarter of the keys and of the columns
    const int quarter = warp & 3;       // TMEM lane quarter
    const int r = quarter * 32 + lane;  // row of the tile
    const uint32_t lt = tmem + ((uint32_t)(quarter * 32) << 16);
    const int k0 = quarter_start(nkeys, k), n = quarter_start(nkeys, k + 1) - k0;  // n <= 64
    bool alive = true;
    if (nkeys > 0) alive = __all_sync(0xffffffffu, mbar_wait(bar_s, 0, ctx));
    tc_fence_after();
    cluster_arrive();  // phase A: S is complete, Q and K are dead
    float ms = 0.f, lsum = 0.f;
    const bool work = nkeys > 0 && alive;  // warp-uniform
    // this warpgroup's keys of the row, in registers (keys that take no part, and
    // columns past them, read as -inf)
    float x[kWin];
#pragma unroll
    for (int j = 0; j < kWin; ++j) x[j] = -INFINITY;
    if (work && n > 0) {
      if (r == 0 && k == 0) DSA_TRACE_EVENT(4);
      tmem_ld64(lt + L::kTmemS + k0, *reinterpret_cast<uint32_t(*)[64]>(&x[0]));
      const int wd = k0 >> 5, sft = k0 & 31;  // k0 is a multiple of 16
      uint64_t bits = (uint64_t)mask[wd] | ((uint64_t)mask[wd + 1] << 32);
      if (sft) bits = (bits >> sft) | ((uint64_t)mask[wd + 2] << (64 - sft));
      if (n < 64) bits &= (1ull << n) - 1ull;
      if (bits != ~0ull) {
#pragma unroll
        for (int j = 0; j < kWin; ++j)
          if (!((bits >> j) & 1ull)) x[j] = -INFINITY;
      }
    }
    float m8[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) m8[u] = x[u];
#pragma unroll
    for (int j = 8; j < kWin; ++j) m8[j & 7] = fmaxf(m8[j & 7], x[j]);
    // the row max over the four warpgroups' keys (every row thread takes part in
    // the barriers of its lane quarter, whatever it computed)
    red[k * 128 + r] = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
    named_barrier(1 + quarter, 128);  // the four warps of this lane quarter
    const float mx = fmaxf(fmaxf(red[r], red[128 + r]), fmaxf(red[256 + r], red[384 + r]));
    if (r == 0 && k == 0) DSA_TRACE_EVENT(13);
    const bool any = mx > -INFINITY;
    ms = any ? mx * sl2 : 0.f;
    if (work) {
      if (n > 0) {
        float l4[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[kWin / 2];
#pragma unroll
        for (int j = 0; j < kWin / 2; ++j) {
          const float p0 = fast_exp2(fmaf(x[2 * j], sl2, -ms));
          const float p1 = fast_exp2(fmaf(x[2 * j + 1], sl2, -ms));
          l4[j & 3] += p0 + p1;
          pk[j] = pack_bf16x2(p0, p1);
        }
        lsum = (l4[0] + l4[1]) + (l4[2] + l4[3]);
        // exactly this warpgroup's P columns [k0, k0 + n/2): they hold S it has
        // already read; a wider store would reach into another warpgroup's S
        const uint32_t pcol = lt + L::kTmemS + k0;
        const int pc = n / 2;  // 8, 16, 24 or 32 (warp-uniform)
        if (pc == 32) {
          tmem_st32(pcol, pk);
        } else if (pc == 8) {
          tmem_st8(pcol, &pk[0]);
        } else {
          tmem_st16(pcol, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
          if (pc == 24) tmem_st8(pcol + 16, &pk[16]);
        }
        // value rows of this quarter's keys that take no part are zeroed, so that
        // 0 * stale data (a skipped page, tokens past n_ctx, block padding) cannot
        // reach O (thread r looks after key k0 + r of its warpgroup, r < n <= 64)
        const int kz = k0 + r;
        if (r < n && !((mask[kz >> 5] >> (kz & 31)) & 1u) && mbar_wait(bar_kv, 0, ctx) &&
            mbar_wait(bar_q, 0, ctx)) {
#pragma unroll
          for (int hf = 0; hf < L::kHalves; ++hf)
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<uint4 *>(smem + L::kOffV + hf * L::kKHalf + kz * 128 + q * 16) =
                  make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      mbar_arrive(bar_p);
      if (r == 0 && k == 0) DSA_TRACE_EVENT(5);
    }
    // the row sum over the four warpgroups (after everyone read the maxima)
    named_barrier(1 + quarter, 128);
    red[k * 128 + r] = lsum;
    named_barrier(1 + quarter, 128);
    const float Lr = (red[r] + red[128 + r]) + (red[256 + r] + red[384 + r]);
    const bool has = work && any && Lr > 0.f;
    if (work) {
      alive = __all_sync(0xffffffffu, mbar_wait(bar_o, 0, ctx));
      tc_fence_after();
      if (r == 0 && k == 0) DSA_TRACE_EVENT(6);
    }
    const float inv = has && alive ? 1.f / Lr : 0.f;
    cluster_wait();  // phase A complete: every CTA's merge area is free
    // ---- push this warpgroup's columns of the row, [k D/4, (k+1) D/4),
    //      normalised, into the row owner's merge area; warpgroup 0 adds the row's
    //      (max, sum).  All lanes take part in the warp-collective TMEM loads.
    const bool mine = r < rows_here;
    const int owner = mine ? r / rpc : 0, i = r - owner * rpc;
    const uint32_t slot = (uint32_t)(c * rpc + i);
    const uint32_t dst = mine ? cluster_map(base + recv_data + slot * (uint32_t)D * 2u, (uint32_t)owner) : 0u;
    constexpr int kCols = D / 4;  // 32 or 16
    uint32_t o[kCols];
    if constexpr (kCols == 32)
      tmem_ld32(lt + L::kTmemO + k * kCols, o);
    else
      tmem_ld16(lt + L::kTmemO + k * kCols, o);
#pragma unroll
    for (int q = 0; q < kCols / 8; ++q) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (inv > 0.f) {  // a row without keys holds no data (possibly stale TMEM): never multiplied
        uint32_t *pv = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          __half2 hv = __floats2half2_rn(__uint_as_float(o[8 * q + 2 * e]) * inv,
                                         __uint_as_float(o[8 * q + 2 * e + 1]) * inv);
          pv[e] = *reinterpret_cast<uint32_t *>(&hv);
        }
      }
      if (mine) st_cluster_v4(dst + (uint32_t)(k * kCols / 8 + q) * 16u, v);
    }
    if (mine && k == 0)
      st_cluster_f2(cluster_map(base + recv_ml + slot * 8u, (uint32_t)owner),
                    make_float2(inv > 0.f ? ms : -INFINITY, inv > 0.f ? Lr : 0.f));
    if (r == 0 && k == 0) DSA_TRACE_EVENT(7);
  }
  cluster_arrive();  // phase B (release): this CTA's rows are in their owners' areas
  cluster_wait();    // acquire: so are every CTA's
  if (threadIdx.x == 0) DSA_TRACE_EVENT(9);

  // ---- merge the rows this CTA owns, a work item being 8 columns of one row:
  //      one pass over its C contributions that keeps the running max M, sum L
  //      and weighted values (each contribution's (max, sum) and values are
  //      loaded first); an empty contribution (sum 0) is skipped.
  const int r0 = c * rpc;
  const int nown = max(0, min(rpc, rows_here - r0));
  const float2 *mlr = reinterpret_cast<const float2 *>(smem + recv_ml);
  constexpr int kChunks = D / 8;
  for (int t = threadIdx.x; t < nown * kChunks; t += kRThreads) {
    const int i = t / kChunks, ch = t % kChunks;
    const unsigned char *src = smem + recv_data + (uint32_t)i * (uint32_t)D * 2u + ch * 16;
    const uint32_t jstride = (uint32_t)rpc * (uint32_t)D * 2u;
    float M = -INFINITY, Lsum = 0.f;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int j = 0; j < C; ++j) {
      const float2 ml = mlr[j * rpc + i];
      const uint4 xv = *reinterpret_cast<const uint4 *>(src + j * jstride);
      if (!(ml.y > 0.f)) continue;
      const float mn = fmaxf(M, ml.x);
      const float sc = fast_exp2(M - mn);  // 0 while M = -inf
      const float w = fast_exp2(ml.x - mn) * ml.y;
      M = mn;
      Lsum = fmaf(Lsum, sc, w);
      const __half2 *hv = reinterpret_cast<const __half2 *>(&xv);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(hv[e]);
        acc[2 * e] = fmaf(w, f.x, acc[2 * e] * sc);
        acc[2 * e + 1] = fmaf(w, f.y, acc[2 * e + 1] * sc);
      }
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    const int ri = r0 + i;
    const size_t orow = ((size_t)s * sh.B + b0 + ri / sh.G) * sh.Hq + (size_t)h * sh.G + ri % sh.G;
    if (sh.lse_out && ch == 0)  // the row's log-sum-exp over its key set: (M + log2 L) ln 2
      sh.lse_out[orow] = Lsum > 0.f ? (M + log2f(Lsum)) * 0.6931471805599453f : -INFINITY;
    uint4 outv;
    uint32_t *po = reinterpret_cast<uint32_t *>(&outv);
#pragma unroll
    for (int e = 0; e < 4; ++e) po[e] = pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
    *reinterpret_cast<uint4 *>(a.o_out + orow * D + ch * 8) = outv;
  }
  if (threadIdx.x == 0) DSA_TRACE_EVENT(10);
  // ---- teardown: every TMEM access is complete (loads wait inline; the issuer
  //      drained its MMAs), then the owner frees TMEM
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
  if (threadIdx.x == 0) DSA_TRACE_EVENT(11);
}

// Dynamic shared memory and clusters beyond 8 CTAs, once per device, and the
// number of clusters of each size (1..16) that can be resident at once.
template <auto K>
const int *resident_capacity(size_t smem) {
  static int cached[64][kRMaxCluster + 1];
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
        cudaFuncSetAttribute(K, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    for (int cs = 0; cs <= kRMaxCluster; ++cs) {
      cached[dev][cs] = 0;
      if (cs == 0) continue;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(cs, 1, 1);
      cfg.blockDim = dim3(kRThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cs;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int nc = 0;
      if (cudaOccupancyMaxActiveClusters(&nc, K, &cfg) == cudaSuccess) cached[dev][cs] = nc;
      cudaGetLastError();
    }
    done[dev] = true;
  }
  return cached[dev];
}

// Cost of a cluster size: waves of clusters for this step together with the
// next one's early gathering (two kernels' clusters resident at once), times the
// keys of the busiest CTA plus a fixed per-step cost in key equivalents (launch,
// query load, exchange, merge).
long long resident_cost(const int *cap, int C, int nclusters, int keys_per_cta) {
  if (!cap || cap[C] < 1) return -1;
  const long long waves = (2LL * nclusters + cap[C] - 1) / cap[C];
  return waves * (keys_per_cta + 384);
}

template <int D, int PAGE>
cudaError_t launch_resident_typed(const Shape &sh, const ResidentPlan &plan, const SparseArgs &a,
                                  cudaStream_t stream) {
  using L = RLayout<D>;
  constexpr auto kern = sparse_resident<D, PAGE>;
  CUtensorMap kmap, vmap, qmap, bkmap, bvmap;
  cudaError_t err;
  const long long rows = sh.n_phys * sh.Hkv * PAGE;
  if ((err = make_kv_tensor_map(&kmap, a.k, rows, D, PAGE)) != cudaSuccess) return err;
  if ((err = make_kv_tensor_map(&vmap, a.v, rows, D, PAGE)) != cudaSuccess) return err;
  if ((err = make_q_tensor_map(&qmap, a.q, (long long)sh.S * sh.B, sh.Hq, D, sh.G, plan.bpt)) != cudaSuccess)
    return err;
  if ((err = make_blk_tensor_map(&bkmap, a.blk_k, (long long)sh.S * sh.B, sh.Hkv, D, plan.bp)) != cudaSuccess)
    return err;
  if ((err = make_blk_tensor_map(&bvmap, a.blk_v, (long long)sh.S * sh.B, sh.Hkv, D, plan.bp)) != cudaSuccess)
    return err;
  ResidentParams prm{sh, plan, a};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.cluster, sh.Hkv, sh.S * plan.rowtiles);
  cfg.blockDim = dim3(kRThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = plan.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  err = cudaLaunchKernelEx(&cfg, kern, prm, kmap, vmap, qmap, bkmap, bvmap);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

// The cheapest cluster size for this shape, or cluster = 0 when no CTA can hold
// its share of keys (or a row tile cannot hold a token's G heads).
template <int D, int PAGE>
ResidentPlan plan_resident_typed(const Shape &sh) {
  ResidentPlan best{};
  if (sh.G > 128) return best;
  const int bpt = 128 / sh.G;
  const int bp = (sh.B + 15) / 16 * 16;
  if (bp > kRMaxKeys) return best;
  const int rowtiles = (sh.B + bpt - 1) / bpt;
  const int bu = (bp + PAGE - 1) / PAGE;
  const int nclusters = sh.S * sh.Hkv * rowtiles;
  const int rows = std::min(bpt, sh.B) * sh.G;
  const int *cap = resident_capacity<sparse_resident<D, PAGE>>(RLayout<D>::kAlloc);
  long long best_cost = -1;
  for (int C = 2; C <= kRMaxCluster; ++C) {
    const int q = (sh.kmax + bu + C - 1) / C;
    if (q * PAGE > kRMaxKeys) continue;
    const int rpc = (rows + C - 1) / C;
    if (recv_bytes<D>(C, rpc) > RLayout<D>::kRecvLimit) continue;
    const long long cost = resident_cost(cap, C, nclusters, q * PAGE);
    if (cost < 0) continue;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = ResidentPlan{C, bpt, rowtiles, bp, q};
    }
  }
  return best;
}

template <int D, int PAGE>
bool launch_resident_page(const Shape &sh, const SparseArgs &a, cudaStream_t stream, cudaError_t *err) {
  const ResidentPlan plan = plan_resident_typed<D, PAGE>(sh);
  if (plan.cluster == 0) return false;
  *err = launch_resident_typed<D, PAGE>(sh, plan, a, stream);
  return true;
}

}  // namespace

DSA_TRACE_EXPORT(dsa_trace_resident)

int sparse_resident_cluster(const Shape &sh) {
  if (sh.active) return 0;
  if (sh.d == 128) {
    if (sh.P == 16) return plan_resident_typed<128, 16>(sh).cluster;
    if (sh.P == 32) return plan_resident_typed<128, 32>(sh).cluster;
    if (sh.P == 64) return plan_resident_typed<128, 64>(sh).cluster;
  } else if (sh.d == 64) {
    if (sh.P == 16) return plan_resident_typed<64, 16>(sh).cluster;
    if (sh.P == 32) return plan_resident_typed<64, 32>(sh).cluster;
    if (sh.P == 64) return plan_resident_typed<64, 64>(sh).cluster;
  }
  return 0;
}

bool launch_sparse_resident(const Shape &sh, const SparseArgs &a, cudaStream_t stream, cudaError_t *err) {
  if (sh.active) return false;  // prefix-part reuse runs on the streaming kernel
  if (sh.d == 128) {
    if (sh.P == 16) return launch_resident_page<128, 16>(sh, a, stream, err);
    if (sh.P == 32) return launch_resident_page<128, 32>(sh, a, stream, err);
    if (sh.P == 64) return launch_resident_page<128, 64>(sh, a, stream, err);
  } else if (sh.d == 64) {
    if (sh.P == 16) return launch_resident_page<64, 16>(sh, a, stream, err);
    if (sh.P == 32) return launch_resident_page<64, 32>(sh, a, stream, err);
    if (sh.P == 64) return launch_resident_page<64, 64>(sh, a, stream, err);
  }
  return false;
}

}  // namespace dsa
