// tc_attn.cuh -- the tcgen05 attention engine shared by the selection and the
// sparse pass: one CTA runs up to 128 query rows of one KV head against a list
// of 64-key tiles that a Policy describes.
//
// Warp roles (320 threads):
//   warp 0      TMA producer: Policy::load_tile, run by all 32 lanes, issues
//               the tile's K and V boxes (one lane per box, so one warp
//               instruction per tile) into a STAGES-deep ring of
//               128-byte-swizzled shared tiles;
//   warp 1      TMEM owner and MMA issuer: S_k = Q K_k^T into a double-buffered
//               TMEM S (64 fp32 columns each), O += P_k V_k into TMEM O.  With
//               PAIR, the S of tiles 2m and 2m + 1 is one MMA chain of N = 128
//               (their K tiles sit in adjacent stages, their S buffers in
//               adjacent TMEM columns): half the S instructions, and the Q
//               operand is read from shared memory once per two tiles;
//   warps 2..9  two softmax warpgroups that take alternate tiles (group g
//               the tiles k with k % 2 == g), so that one group's exp phase
//               overlaps the other's loads and stores.  Thread (g, r) owns query
//               row r (TMEM lane r): online softmax in the log2 domain with lazy
//               rescaling (the reference max moves only when a tile beats it by
//               more than 2^8), per-unit sums (32 keys at most) handed to
//               Policy::after_tile, P in bf16 into TMEM over the tile's S
//               (the A operand of the PV MMA).
//               Each group accumulates into its own TMEM O.
// After run() every softmax thread holds its group's (m, l); finish() joins the
// two groups' statistics, and the kernel combines the two O accumulators
// (load_o) with the weights it returns before calling teardown().
//
// Every wait is time-bounded (sm100::mbar_wait); a timeout aborts the CTA,
// which still drains its copies and MMAs before TMEM is freed.
#pragma once

#include "common.cuh"
#include "sm100.cuh"
#include "trace.cuh"

namespace dsa {
namespace tc {

constexpr int kBN = 64;          // keys per tile
constexpr int kHalfBN = kBN / 2; // keys per softmax warpgroup
constexpr int kThreads = 320;    // 10 warps
constexpr int kSoftmaxThreads = 256;
constexpr float kRescaleLog2 = 8.f;

// The unit of the per-page partial sums: min(PAGE, 32) keys of one page (a
// 64-token page is two units).
template <int PAGE>
struct Units {
  static constexpr int kKeys = PAGE < kHalfBN ? PAGE : kHalfBN;   // keys per unit
  static constexpr int kPerTile = kBN / kKeys;                     // units per tile
  static constexpr int kPerPage = PAGE / kKeys;                    // units per page
};

template <int D, int STAGES>
struct Layout {
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kQHalf = 128 * 128;           // 128 rows x 128 B
  static constexpr uint32_t kKVHalf = kBN * 128;          // 64 keys x 128 B
  static constexpr uint32_t kKBytes = kHalves * kKVHalf;
  static constexpr uint32_t kStageBytes = 2 * kKBytes;    // K tile then V tile
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffKV = kOffQ + kHalves * kQHalf;
  static constexpr uint32_t kOffBar = kOffKV + STAGES * kStageBytes;
  static constexpr int kNumBars = 2 * STAGES + 17;  // the last one is the kernel's own
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
  static constexpr uint32_t kOffML = kOffQ;  // [2 groups][128] (m, l), once Q is dead
  static constexpr uint32_t kBytes = kOffMisc + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // room to align the base to 1 KB
  // TMEM: four S buffers of 64 columns (two per softmax group: buffer 2g+i;
  // the softmax overwrites the first 32 columns of a tile's buffer with its P
  // in bf16, the A operand of the PV MMA), then the O accumulators of group 0
  // and group 1
  static constexpr uint32_t kTmemO = 4 * kBN;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(D == 64 || D == 128, "head dimension");
};

template <int D, int STAGES, bool PAIR = false>
struct Engine {
  using L = Layout<D, STAGES>;
  static_assert(!PAIR || (STAGES % 2 == 0 && STAGES >= 4), "tile pairs fill adjacent stages");
  // Distance between the two 64-element halves of a K or V tile in shared
  // memory.  With PAIR a pair of stages is [K half 0: tile 2m, tile 2m + 1][K
  // half 1: ...][V half 0: ...][V half 1: ...], so that the K rows of both tiles
  // of a half are one 128-row operand.
  static constexpr uint32_t kHalfStride = PAIR ? 2 * L::kKVHalf : L::kKVHalf;
  uint32_t base;         // 1 KB-aligned shared address of the layout
  unsigned char *smem;   // same, generic pointer
  uint32_t tmem;         // TMEM base address (lane 0, column 0)
  sm100::WaitCtx ctx;
  int warp, lane;

  __device__ __forceinline__ uint32_t bar(int i) const { return base + L::kOffBar + 8u * (uint32_t)i; }
  __device__ __forceinline__ uint32_t kv_full(int st) const { return bar(st); }
  __device__ __forceinline__ uint32_t kv_empty(int st) const { return bar(STAGES + st); }
  __device__ __forceinline__ uint32_t s_full(int sb) const { return bar(2 * STAGES + sb); }
  __device__ __forceinline__ uint32_t s_free(int sb) const { return bar(2 * STAGES + 4 + sb); }
  // P of a group's m-th tile is announced on p_full(g, m & 1): with two
  // barriers per group the group can complete at most one phase ahead of the
  // MMA issuer's wait on a barrier (its next tile on the same barrier needs an
  // S that the issuer sends only after that wait), so parity waits stay exact
  __device__ __forceinline__ uint32_t p_full(int g, int m) const { return bar(2 * STAGES + 8 + 2 * g + (m & 1)); }
  __device__ __forceinline__ uint32_t pv_done(int g) const { return bar(2 * STAGES + 12 + g); }
  __device__ __forceinline__ uint32_t q_full() const { return bar(2 * STAGES + 14); }
  __device__ __forceinline__ uint32_t drain() const { return bar(2 * STAGES + 15); }
  __device__ __forceinline__ uint32_t user_bar() const { return bar(2 * STAGES + 16); }
  // tile k runs on softmax group k % 2 as that group's (k / 2)-th tile, in S buffer
  // 2 * group + (k / 2) % 2; with PAIR in buffer 2 * ((k / 2) % 2) + group, so
  // that the two tiles of a pair have adjacent buffers.  Either way a group's
  // tiles alternate between its two buffers.
  static __device__ __forceinline__ int s_buf(int k) {
    return PAIR ? 2 * ((k >> 1) & 1) + (k & 1) : 2 * (k & 1) + ((k >> 1) & 1);
  }
  // half 0 of stage st's K and V tiles (half 1 is kHalfStride further)
  __device__ __forceinline__ uint32_t stage_k(int st) const {
    return PAIR ? base + L::kOffKV + (st >> 1) * 2 * L::kStageBytes + (st & 1) * L::kKVHalf
                : base + L::kOffKV + st * L::kStageBytes;
  }
  __device__ __forceinline__ uint32_t stage_v(int st) const {
    return stage_k(st) + (PAIR ? 2 * L::kKBytes : L::kKBytes);
  }
  __device__ __forceinline__ volatile int *abort_flag() const {
    return reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
  }

  // Softmax-thread geometry --------------------------------------------------
  __device__ __forceinline__ int quarter() const { return warp & 3; }
  __device__ __forceinline__ int row_in_tile() const { return quarter() * 32 + lane; }
  __device__ __forceinline__ int group() const { return (warp - 2) >> 2; }  // softmax group 0 or 1
  __device__ __forceinline__ uint32_t lane_tmem() const { return tmem + ((uint32_t)(quarter() * 32) << 16); }

  // Set-up that reads no memory the caller passes: shared-memory carve-up,
  // barrier init, tensor-map prefetch (thread 0) and the TMEM allocation (warp
  // 1).  Every thread of the CTA calls it; a kernel launched as a programmatic
  // dependent runs it before waiting for the kernel ahead of it, so that it
  // overlaps that kernel's tail.
  template <class Policy>
  __device__ __forceinline__ void setup(unsigned char *smem_raw, const Policy &pol) {
    using namespace sm100;
    const uint32_t raw = smem_addr(smem_raw);
    base = (raw + 1023u) & ~1023u;
    smem = smem_raw + (base - raw);
    warp = threadIdx.x >> 5;
    lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
      for (int st = 0; st < STAGES; ++st) {
        mbar_init(kv_full(st), 1);
        mbar_init(kv_empty(st), 1);
      }
      for (int sb = 0; sb < 4; ++sb) {
        mbar_init(s_full(sb), 1);
        mbar_init(s_free(sb), kSoftmaxThreads / 2);
      }
      for (int g = 0; g < 2; ++g) {
        mbar_init(p_full(g, 0), kSoftmaxThreads / 2);
        mbar_init(p_full(g, 1), kSoftmaxThreads / 2);
        mbar_init(pv_done(g), 1);
      }
      mbar_init(q_full(), kSoftmaxThreads);
      mbar_init(drain(), 1);
      mbar_init(user_bar(), 1);
      *abort_flag() = 0;
      fence_mbar_init();
      pol.prefetch();
    }
    if (warp == 1) {
      tmem_alloc(base + L::kOffMisc, L::kTmemCols);
      tmem_relinquish();
    }
  }

  // The key side of the set-up, for a policy whose tile addresses need no
  // barrier (kIssueBeforeSync): the policy's per-CTA tables and the producer's
  // loads of the first min(STAGES, num_tiles) tiles.  All threads call it; a
  // kernel that may read the key side before its dependency wait calls it there,
  // then init() with staged = true.
  template <class Policy>
  __device__ __forceinline__ void stage(Policy &pol, int num_tiles) {
    static_assert(Policy::kIssueBeforeSync, "staging needs tables that warp 0 builds itself");
    pol.prepare(smem);
    if (threadIdx.x == 0) DSA_TRACE_EVENT(35);
    if (warp == 0 && num_tiles > 0) issue_first(pol, num_tiles);
  }

  // The data part of the set-up, after setup(): the policy's per-CTA tables, the
  // query rows copied by the softmax threads into the Q tile, and (for a policy
  // that allows it) the producer's loads of the first STAGES tiles, all before
  // the CTA-wide barrier.  With staged = true, stage() has already built the
  // tables and issued those loads.
  template <class Policy>
  __device__ __forceinline__ void init(uint32_t *status, Policy &pol, int num_tiles,
                                       bool staged = false) {
    using namespace sm100;
    if (!staged) {
      pol.prepare(smem);  // per-CTA tables of the policy (all threads)
      if (threadIdx.x == 0) DSA_TRACE_EVENT(35);
    }
    if (warp >= 2) {    // half of this row's query into the swizzled Q tile (zeros past the end)
      const int r = row_in_tile();
      constexpr int kChunks = D / 16;  // 16-byte chunks per half row
      const int c0 = group() * kChunks;
      const uint4 *src = reinterpret_cast<const uint4 *>(pol.q_row(r));
      uint4 v[kChunks];
#pragma unroll
      for (int i = 0; i < kChunks; ++i) v[i] = src ? __ldg(src + c0 + i) : make_uint4(0, 0, 0, 0);
      if (r == 0 && group() == 0) DSA_TRACE_AFTER(37, v[0].x);
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        const int c = c0 + i;
        *reinterpret_cast<uint4 *>(smem + L::kOffQ + (c >> 3) * L::kQHalf + sw128_offset(r, c & 7)) = v[i];
      }
      fence_proxy_async_smem();
    }
    // warp 0 is the producer: the first tiles' loads go out right away
    if (!staged && Policy::kIssueBeforeSync && warp == 0 && num_tiles > 0) issue_first(pol, num_tiles);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pol.ready();  // tables built by prepare() are complete from here on
    // (a policy whose first tile addresses need those tables issues them now)
    if (!Policy::kIssueBeforeSync && warp == 0 && num_tiles > 0) issue_first(pol, num_tiles);
    tmem = *reinterpret_cast<volatile uint32_t *>(smem + L::kOffMisc);
    ctx = sm100::WaitCtx{abort_flag(), status};
    if (warp >= 2) mbar_arrive(q_full());
    if (threadIdx.x == 0) DSA_TRACE_EVENT(1);
  }

  // Loads of the first STAGES tiles; all 32 lanes of warp 0 (the policy issues a
  // tile's boxes from several lanes at once).
  template <class Policy>
  __device__ __forceinline__ void issue_first(Policy &pol, int num_tiles) {
    if (lane == 0) DSA_TRACE_EVENT(36);
    for (int k = 0; k < min(STAGES, num_tiles); ++k)
      pol.load_tile(k, stage_k(k), stage_v(k), kHalfStride, kv_full(k), lane);
    if (lane == 0) DSA_TRACE_EVENT(2);
  }

  // Runs the pipeline over `num_tiles` tiles.  Softmax threads return their
  // row's (m, l) in the log2 domain (l over both halves) and whether the CTA is
  // still alive.
  //
  // Phase accounting.  A parity wait on an mbarrier tells apart only two
  // consecutive phases, so every wait below is made while the barrier has
  // completed either the phase before the one waited for or that phase itself:
  // never two behind (the wait would return at once) and never one past (it
  // would block until the timeout).  For each barrier: who completes it, who
  // waits for which completion, and why the completion after it cannot have
  // happened yet; the one before it always has, because each waiter waited for
  // it (or for a later event that follows it) on its previous use.  This holds
  // for any STAGES >= 3 with kLook = 2; with STAGES = 2, kLook = 1 and the same
  // arguments hold one tile closer.
  //   kv_full(st)  TMA of tile k (the (k / STAGES)-th fill of stage st).  The MMA
  //                issuer (S(k)) and softmax thread r (value-row zeroing) wait
  //                for it; the next fill of st is tile k + STAGES, issued after
  //                kv_empty(st) of PV(k), which follows both waits.
  //   kv_empty(st) commit after PV(j), j % STAGES == st; the producer waits for
  //                PV(k - STAGES) before it loads tile k into st; the next commit,
  //                PV(k), needs tile k loaded.
  //   s_full(sb)   commit of S(k) into buffer s_buf(k); softmax group k % 2 waits
  //                for it as its (mine / 2)-th use of sb; S(k + 4) into sb needs
  //                s_free(sb) from this very read.
  //   s_free(sb)   128 softmax arrivals once S(k) is read; the issuer waits for
  //                the one of tile k - 4 before S(k); the next (tile k) needs S(k).
  //   p_full(g, m & 1)  128 arrivals once P of group g's m-th tile is in TMEM, two
  //                barriers used alternately; the issuer waits for it before
  //                PV; the next arrival on the same barrier is for m + 2, whose S
  //                the issuer sends only after this wait.
  //   pv_done(g)   commit after each PV of group g.  The issuer waits, before
  //                S(k) overwrites the TMEM buffer that held P(k - 4), for
  //                PV(k - 4): at that point it has issued PVs up to k - 3, so
  //                PV(k - 4) is the latest of its group.  Softmax group g waits,
  //                before rescaling O for its m-th tile, for the PV of its
  //                (m - 1)-th; PV of the m-th needs this group's P first, and PV
  //                of the (m - 2)-th completed before S of the m-th was issued.
  //                With PAIR, pair m + 1 (tiles k = 2m + 2 and 2m + 3) waits at
  //                the top of iteration 2m, when PVs up to 2m - 1 are out:
  //                PV(k - 4) is again the latest of tile k's group.
  //   drain        one commit after the issuer's last MMA; a one-phase barrier,
  //                waited for once by every softmax thread before O is read.
  template <int PAGE, class Policy>
  __device__ __forceinline__ bool run(Policy &pol, int num_tiles, float &m_out, float &l_out) {
    using namespace sm100;
    using U = Units<PAGE>;
    volatile int never = 0;
    const WaitCtx drain_ctx{&never, ctx.status};
    bool alive = true;
    m_out = -INFINITY;
    l_out = 0.f;
    if (warp == 0) {
      // ---------------------------------------------------------- producer --
      if (num_tiles > 0) {  // the whole warp: a tile's boxes go out from several lanes
        int issued = min(STAGES, num_tiles);  // issued during init
        for (int k = issued; k < num_tiles; ++k) {
          const int st = k % STAGES;
          if (!__all_sync(0xffffffffu, mbar_wait(kv_empty(st), ((k / STAGES) - 1) & 1, ctx))) break;
          pol.load_tile(k, stage_k(st), stage_v(st), kHalfStride, kv_full(st), lane);
          if (k == STAGES && lane == 0) DSA_TRACE_EVENT(24);
          issued = k + 1;
        }
        // copies in flight land before the CTA's shared memory is released
        if (lane == 0)
          for (int k = max(0, issued - STAGES); k < issued; ++k)
            mbar_wait(kv_full(k % STAGES), (k / STAGES) & 1, drain_ctx);
      }
    } else if (warp == 1) {
      // --------------------------------------------------------- MMA issuer --
      if (lane == 0 && num_tiles > 0) {
        constexpr uint32_t kIdS = idesc_bf16(128, kBN, false, false);
        constexpr uint32_t kIdO = idesc_bf16(128, D, false, true);
        // S of tile j + kLook is issued before P of tile j is awaited, so that a
        // softmax group finds its next S ready; kLook stays below STAGES because
        // that tile's K/V stage is freed by PV_{j + kLook - STAGES}
        constexpr int kLook = STAGES >= 3 ? 2 : 1;
        auto issue_s = [&](int k) -> bool {
          const int st = k % STAGES, sb = s_buf(k);
          if (!mbar_wait(kv_full(st), (k / STAGES) & 1, ctx)) return false;
          if (k == 0) DSA_TRACE_EVENT(3);
          if (k >= 4 && !mbar_wait(s_free(sb), (((k >> 1) - 2) >> 1) & 1, ctx)) return false;
          // the buffer still holds P of tile k - 4, which PV(k - 4) reads from TMEM:
          // that MMA must have completed (not only been issued) before S(k) lands
          // there.  S(k) is issued at the top of iteration k - kLook, after PV of
          // tile k - 2 * ((kLook + 2) / 2), the latest PV of this group so far
          // (k - 4 or later): waiting for that one, whose pv_done phase is the
          // current one, covers PV(k - 4) (commits complete in order).
          if (k >= 4 && !mbar_wait(pv_done(k & 1), ((k >> 1) - (kLook + 2) / 2) & 1, ctx)) return false;
          tc_fence_after();
          const uint32_t sk = stage_k(st);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t hf = kk >> 2, sub = kk & 3;
            const uint64_t ad = sdesc_sw128(base + L::kOffQ + hf * L::kQHalf + sub * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(sk + hf * kHalfStride + sub * 32, 16, 1024);
            umma_bf16(tmem + sb * kBN, ad, bd, kIdS, kk > 0 ? 1u : 0u);
          }
          umma_commit(s_full(sb));
          if (k == 1) DSA_TRACE_EVENT(25);
          if (k == 4) DSA_TRACE_EVENT(15);
          return true;
        };
        // PAIR: S of tiles 2m and 2m + 1 (of tile 2m alone when it is the last)
        // as one chain of N = 2 kBN into their adjacent buffers.  Pair m + 1 is
        // issued at the top of iteration 2m, after the PVs up to 2m - 1, so that
        // the PV(k - 4) it waits for is the latest PV of tile k's group.  (Sent
        // instead after PV(2m), it leaves group 0 without an S for the length
        // of PV(2m) and the pair's MMAs: a slower loop, although that needs no
        // wait for a PV just issued.)
        constexpr uint32_t kIdS2 = idesc_bf16(128, 2 * kBN, false, false);
        auto issue_pair = [&](int m) -> bool {
          const int k0 = 2 * m;
          const int nk = k0 + 1 < num_tiles ? 2 : 1;
          for (int t = 0; t < nk; ++t) {
            const int k = k0 + t;
            if (!mbar_wait(kv_full(k % STAGES), (k / STAGES) & 1, ctx)) return false;
            if (k >= 4) {
              if (!mbar_wait(s_free(s_buf(k)), (((k >> 1) - 2) >> 1) & 1, ctx)) return false;
              if (!mbar_wait(pv_done(k & 1), ((k >> 1) - 2) & 1, ctx)) return false;
            }
          }
          if (k0 == 0) DSA_TRACE_EVENT(3);
          tc_fence_after();
          const uint32_t sk = stage_k(k0 % STAGES);  // tile k0's rows, then tile k0 + 1's
          const uint32_t dst = tmem + s_buf(k0) * kBN;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t hf = kk >> 2, sub = kk & 3;
            const uint64_t ad = sdesc_sw128(base + L::kOffQ + hf * L::kQHalf + sub * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(sk + hf * kHalfStride + sub * 32, 16, 1024);
            umma_bf16(dst, ad, bd, nk == 2 ? kIdS2 : kIdS, kk > 0 ? 1u : 0u);
          }
          umma_commit(s_full(s_buf(k0)));
          if (nk == 2) umma_commit(s_full(s_buf(k0 + 1)));
          return true;
        };
        bool ok = mbar_wait(q_full(), 0, ctx);
        DSA_TRACE_EVENT(12);
        if constexpr (PAIR) {
          if (ok) ok = issue_pair(0);
          if (ok && num_tiles > 2) ok = issue_pair(1);
        } else {
          for (int k = 0; ok && k < kLook && k < num_tiles; ++k) ok = issue_s(k);
        }
        for (int j = 0; ok && j < num_tiles; ++j) {
          if constexpr (PAIR) {
            if ((j & 1) == 0 && j >= 2 && j + 2 < num_tiles && !issue_pair((j >> 1) + 1)) break;
          } else {
            if (j + kLook < num_tiles && !issue_s(j + kLook)) break;
          }
          const int st = j % STAGES, g = j & 1;
          if (!mbar_wait(p_full(g, j >> 1), (j >> 2) & 1, ctx)) break;
          if (j == 2) DSA_TRACE_EVENT(14);
          tc_fence_after();
          const uint32_t sv = stage_v(st);
          const uint32_t pa = tmem + s_buf(j) * kBN;  // P_j in TMEM: 8 columns per 16 keys
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint64_t bd = sdesc_sw128(sv + kk * 16 * 128, kHalfStride, 1024);
            umma_bf16_ts(tmem + L::kTmemO + g * D, pa + kk * 8, bd, kIdO, (j > 1 || kk > 0) ? 1u : 0u);
          }
          umma_commit(pv_done(g));
          umma_commit(kv_empty(st));
          if (j == 0) DSA_TRACE_EVENT(26);
        }
        // every issued MMA completes before TMEM can be released
        umma_commit(drain());
        mbar_wait(drain(), 0, drain_ctx);
      }
    } else {
      // ---------------------------------------------------- softmax groups --
      const int r = row_in_tile();
      const int g = group();
      const uint32_t lt = lane_tmem();
      const uint32_t o_col = L::kTmemO + g * D;
      float m_used = -INFINITY, l = 0.f;
      int mine = 0;  // tiles this group has finished
      for (int k = g; k < num_tiles; k += 2, ++mine) {
        const int st = k % STAGES, sb = s_buf(k);
        alive = __all_sync(0xffffffffu, mbar_wait(s_full(sb), (mine >> 1) & 1, ctx));
        if (!alive) break;
        const bool lead = r == 0;
        const bool tr = k == 1 && lead;
        if (k == 0 && lead) DSA_TRACE_EVENT(4);
        if (tr) DSA_TRACE_EVENT(16);
        if (k == 2 && lead) DSA_TRACE_EVENT(27);
        if (k == 4 && lead) DSA_TRACE_EVENT(28);
        tc_fence_after();
        uint32_t sraw[kBN];
        tmem_ld32(lt + sb * kBN, *reinterpret_cast<uint32_t(*)[32]>(&sraw[0]));
        tmem_ld32(lt + sb * kBN + 32, *reinterpret_cast<uint32_t(*)[32]>(&sraw[32]));
        if (tr) DSA_TRACE_EVENT(17);
        const uint64_t key_ok = pol.key_mask(k);  // bit j: key j of the tile takes part
        if (tr) DSA_TRACE_EVENT(18);
        float x[kBN];  // raw logits q.k; keys that take no part become -inf
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (key_ok == ~0ull) {
#pragma unroll
          for (int j = 0; j < kBN; ++j) {
            x[j] = __uint_as_float(sraw[j]);
            mx[j & 3] = fmaxf(mx[j & 3], x[j]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < kBN; ++j) {
            x[j] = ((key_ok >> j) & 1ull) ? __uint_as_float(sraw[j]) : -INFINITY;
            mx[j & 3] = fmaxf(mx[j & 3], x[j]);
          }
        }
        // tile max in the log2 domain (the scale is positive, so it commutes with max)
        const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * pol.sl2;
        if (tr) DSA_TRACE_EVENT(19);
        // PV of this group's previous tile must have landed before O is rescaled.
        // It is the only PV of the group that may still run here (the one before
        // completed before this tile's S was issued), so the parity wait below is
        // unambiguous.  P goes into this tile's own S buffer, whose last reader,
        // PV of the tile four earlier, has completed for the same reason.
        const bool need = tmax > m_used + kRescaleLog2 || (m_used == -INFINITY && tmax > -INFINITY);
        if (__any_sync(0xffffffffu, need)) {
          float alpha = 1.f;
          if (need) {
            alpha = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - tmax);
            m_used = tmax;
            l *= alpha;
          }
          if (mine > 0) {  // O holds this group's earlier tiles: scale it
            alive = __all_sync(0xffffffffu, mbar_wait(pv_done(g), (mine - 1) & 1, ctx));
            if (!alive) break;
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(lt + o_col + c0, o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(lt + o_col + c0, o);
            }
          }
        }
        const float mu = (m_used == -INFINITY) ? 0.f : m_used;
        float usum[U::kPerTile];
#pragma unroll
        for (int u = 0; u < U::kPerTile; ++u) usum[u] = 0.f;
#pragma unroll
        for (int j = 0; j < kBN; ++j) {
          const float p = fast_exp2(fmaf(x[j], pol.sl2, -mu));
          x[j] = p;
          usum[j / U::kKeys] += p;
        }
#pragma unroll
        for (int u = 0; u < U::kPerTile; ++u) l += usum[u];
        if (tr) DSA_TRACE_EVENT(20);
        {  // P in bf16 over the first 32 columns of the tile's S buffer
          uint32_t pk[kBN / 2];
#pragma unroll
          for (int c = 0; c < kBN / 2; ++c) pk[c] = pack_bf16x2(x[2 * c], x[2 * c + 1]);
          tmem_st32(lt + sb * kBN, pk);
        }
        if (tr) DSA_TRACE_EVENT(21);
        // value rows of keys that take no part are zeroed so that 0 * stale data
        // cannot reach O (thread r < 64 looks after key r of the tile)
        if (r < kBN && !((key_ok >> r) & 1ull) && mbar_wait(kv_full(st), (k / STAGES) & 1, ctx)) {
          unsigned char *vrow = smem + (stage_v(st) - base) + r * 128;
#pragma unroll
          for (int hf = 0; hf < L::kHalves; ++hf)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4 *>(vrow + hf * kHalfStride + c * 16) = make_uint4(0, 0, 0, 0);
        }
        pol.after_tile(k, r, m_used, usum);
        if (tr) DSA_TRACE_EVENT(22);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(s_free(sb));
        mbar_arrive(p_full(g, mine));
        if (tr) DSA_TRACE_EVENT(23);
        if (k == 2 && lead) DSA_TRACE_EVENT(13);
        if (k == 4 && lead) DSA_TRACE_EVENT(29);
        if (k >= num_tiles - 2 && lead && g == ((num_tiles - 1) & 1)) DSA_TRACE_EVENT(5);
      }
      if (alive && mine > 0) {  // the group's last PV has landed in its O
        // The MMA issuer commits `drain` once, after its last MMA: a one-phase
        // barrier, unlike pv_done, whose parity cannot tell a group's last PV
        // from the one before it once either may already have completed.
        alive = __all_sync(0xffffffffu, mbar_wait(drain(), 0, ctx));
        if (alive) tc_fence_after();
        if (r == 0 && g == ((num_tiles - 1) & 1)) DSA_TRACE_EVENT(6);
      }
      m_out = m_used;
      l_out = (alive && mine > 0) ? l : 0.f;
    }
    return alive;
  }

  // Joins the two softmax groups' statistics of each row; every thread of the
  // CTA calls it (it contains a CTA barrier).  For softmax threads it returns
  // the row's merged (m, l) and the weights wa, wb with which the groups' O
  // accumulators combine: O = wa * O_0 + wb * O_1 (a weight is 0 for a group
  // that saw no keys, whose accumulator holds no data).
  __device__ __forceinline__ void finish(float m, float l, float &m_row, float &l_row, float &wa,
                                         float &wb) {
    float2 *ml = reinterpret_cast<float2 *>(smem + L::kOffML);
    const int r = row_in_tile();
    // both groups have seen their last PV complete, hence every MMA (which all
    // read Q) is done: only then may the statistics area in the Q tile be written
    __syncthreads();
    if (warp >= 2) ml[group() * 128 + r] = make_float2(m, l);
    __syncthreads();
    m_row = -INFINITY;
    l_row = 0.f;
    wa = wb = 0.f;
    if (warp >= 2) {
      const float2 a = ml[r], b = ml[128 + r];
      const float M = fmaxf(a.y > 0.f ? a.x : -INFINITY, b.y > 0.f ? b.x : -INFINITY);
      wa = a.y > 0.f ? exp2f(a.x - M) : 0.f;
      wb = b.y > 0.f ? exp2f(b.x - M) : 0.f;
      m_row = M;
      l_row = wa * a.y + wb * b.y;
    }
    __syncthreads();  // the statistics area (in the Q tile) may be reused after this
  }

  // 32 columns [c0, c0+32) of group `which`'s O accumulator for this thread's
  // row (warp-collective).
  __device__ __forceinline__ void load_o(int which, int c0, uint32_t (&o)[32]) const {
    sm100::tmem_ld32(lane_tmem() + L::kTmemO + which * D + c0, o);
  }
  // Columns [c0, c0+32) of both groups' O accumulators, with one wait.
  __device__ __forceinline__ void load_o2(int c0, uint32_t (&o0)[32], uint32_t (&o1)[32]) const {
    sm100::tmem_ld32x2(lane_tmem() + L::kTmemO + c0, o0, lane_tmem() + L::kTmemO + D + c0, o1);
  }

  // All threads: waits for everybody, then the TMEM owner frees TMEM.
  __device__ __forceinline__ void teardown() {
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
      sm100::tc_fence_after();
      sm100::tmem_dealloc(tmem, L::kTmemCols);
    }
  }
};

}  // namespace tc
}  // namespace dsa
