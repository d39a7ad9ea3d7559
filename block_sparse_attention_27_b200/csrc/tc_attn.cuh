// tc_attn.cuh -- the tcgen05 attention engine shared by the selection and the
// sparse pass: one CTA runs up to 128 query rows of one KV head against a list
// of 64-token key tiles that a Policy describes.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: Policy::load_tile issues the tile's K and V boxes
//               into a STAGES-deep ring of 128-byte-swizzled shared tiles;
//   warp 1      TMEM owner and MMA issuer: S_k = Q K_k^T into a double-buffered
//               TMEM S (64 fp32 columns each), O += P_k V_k into TMEM O;
//   warps 2..5  one query row per thread (TMEM lane = row): online softmax in the
//               log2 domain with lazy rescaling (the reference max moves only
//               when a tile beats it by more than 2^8), per-page sums handed to
//               Policy::after_tile, P in bf16 to shared memory for the PV MMA.
// After run() the softmax threads hold (m, l) of their row and O sits in TMEM;
// the kernel reads it (Engine::load_o) and then calls Engine::teardown.
//
// Every wait is time-bounded (sm100::mbar_wait); a timeout aborts the CTA,
// which still drains its copies and MMAs before TMEM is freed.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dsa {
namespace tc {

constexpr int kBN = 64;          // keys per tile
constexpr int kThreads = 192;    // 6 warps
constexpr float kRescaleLog2 = 8.f;

template <int D, int STAGES>
struct Layout {
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kQHalf = 128 * 128;           // 128 rows x 128 B
  static constexpr uint32_t kKVHalf = kBN * 128;          // 64 keys x 128 B
  static constexpr uint32_t kKBytes = kHalves * kKVHalf;
  static constexpr uint32_t kStageBytes = 2 * kKBytes;    // K tile then V tile
  static constexpr uint32_t kPBytes = 128 * 128;          // 128 rows x 64 keys bf16
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffKV = kOffQ + kHalves * kQHalf;
  static constexpr uint32_t kOffP = kOffKV + STAGES * kStageBytes;
  static constexpr uint32_t kOffBar = kOffP + 2 * kPBytes;
  static constexpr int kNumBars = 2 * STAGES + 10;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kOffMisc + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // room to align the base to 1 KB
  static constexpr uint32_t kTmemCols = 256;         // S0 [0,64) S1 [64,128) O [128,128+D)
  static constexpr uint32_t kTmemO = 128;
  static_assert(D == 64 || D == 128, "head dimension");
};

template <int D, int STAGES>
struct Engine {
  using L = Layout<D, STAGES>;
  uint32_t base;         // 1 KB-aligned shared address of the layout
  unsigned char *smem;   // same, generic pointer
  uint32_t tmem;         // TMEM base address (lane 0, column 0)
  sm100::WaitCtx ctx;
  int warp, lane;

  __device__ __forceinline__ uint32_t bar(int i) const { return base + L::kOffBar + 8u * (uint32_t)i; }
  __device__ __forceinline__ uint32_t kv_full(int st) const { return bar(st); }
  __device__ __forceinline__ uint32_t kv_empty(int st) const { return bar(STAGES + st); }
  __device__ __forceinline__ uint32_t s_full(int b) const { return bar(2 * STAGES + b); }
  __device__ __forceinline__ uint32_t s_free(int b) const { return bar(2 * STAGES + 2 + b); }
  __device__ __forceinline__ uint32_t p_full(int b) const { return bar(2 * STAGES + 4 + b); }
  __device__ __forceinline__ uint32_t pv_done(int b) const { return bar(2 * STAGES + 6 + b); }
  __device__ __forceinline__ uint32_t q_full() const { return bar(2 * STAGES + 8); }
  __device__ __forceinline__ uint32_t drain() const { return bar(2 * STAGES + 9); }
  __device__ __forceinline__ uint32_t stage_k(int st) const { return base + L::kOffKV + st * L::kStageBytes; }
  __device__ __forceinline__ uint32_t stage_v(int st) const { return stage_k(st) + L::kKBytes; }
  __device__ __forceinline__ volatile int *abort_flag() const {
    return reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
  }

  // Barrier init and TMEM allocation; every thread of the CTA calls it.
  __device__ __forceinline__ void init(unsigned char *smem_raw, uint32_t *status) {
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
      for (int b = 0; b < 2; ++b) {
        mbar_init(s_full(b), 1);
        mbar_init(s_free(b), 128);
        mbar_init(p_full(b), 128);
        mbar_init(pv_done(b), 1);
      }
      mbar_init(q_full(), 128);
      mbar_init(drain(), 1);
      *abort_flag() = 0;
      fence_mbar_init();
    }
    if (warp == 1) {
      tmem_alloc(base + L::kOffMisc, L::kTmemCols);
      tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem = *reinterpret_cast<volatile uint32_t *>(smem + L::kOffMisc);
    ctx = sm100::WaitCtx{abort_flag(), status};
  }

  // Softmax-thread helpers --------------------------------------------------
  __device__ __forceinline__ int row_in_tile() const { return (warp & 3) * 32 + lane; }
  __device__ __forceinline__ uint32_t lane_tmem() const { return tmem + ((uint32_t)((warp & 3) * 32) << 16); }

  // Runs the pipeline over `num_tiles` tiles.  Softmax threads return their
  // row's (m, l) in the log2 domain and whether the CTA is still alive.
  template <int PAGE, class Policy>
  __device__ __forceinline__ bool run(Policy &pol, int num_tiles, float &m_out, float &l_out) {
    using namespace sm100;
    volatile int never = 0;
    const WaitCtx drain_ctx{&never, ctx.status};
    bool alive = true;
    m_out = -INFINITY;
    l_out = 0.f;
    if (warp == 0) {
      // ---------------------------------------------------------- producer --
      if (lane == 0 && num_tiles > 0) {
        pol.prefetch();
        int issued = 0;
        for (int k = 0; k < num_tiles; ++k) {
          const int st = k % STAGES;
          if (k >= STAGES && !mbar_wait(kv_empty(st), ((k / STAGES) - 1) & 1, ctx)) break;
          pol.load_tile(k, stage_k(st), stage_v(st), L::kKVHalf, kv_full(st));
          issued = k + 1;
        }
        // copies in flight land before the CTA's shared memory is released
        for (int k = max(0, issued - STAGES); k < issued; ++k)
          mbar_wait(kv_full(k % STAGES), (k / STAGES) & 1, drain_ctx);
      }
    } else if (warp == 1) {
      // --------------------------------------------------------- MMA issuer --
      if (lane == 0 && num_tiles > 0) {
        constexpr uint32_t kIdS = idesc_bf16(128, kBN, false, false);
        constexpr uint32_t kIdO = idesc_bf16(128, D, false, true);
        bool ok = mbar_wait(q_full(), 0, ctx);
        for (int k = 0; ok && k <= num_tiles; ++k) {
          if (k < num_tiles) {
            const int st = k % STAGES, b = k & 1;
            if (!mbar_wait(kv_full(st), (k / STAGES) & 1, ctx)) break;
            if (k >= 2 && !mbar_wait(s_free(b), ((k - 2) >> 1) & 1, ctx)) break;
            tc_fence_after();
            const uint32_t sk = stage_k(st);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t hf = kk >> 2, sub = kk & 3;
              const uint64_t ad = sdesc_sw128(base + L::kOffQ + hf * L::kQHalf + sub * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(sk + hf * L::kKVHalf + sub * 32, 16, 1024);
              umma_bf16(tmem + b * kBN, ad, bd, kIdS, kk > 0 ? 1u : 0u);
            }
            umma_commit(s_full(b));
          }
          if (k >= 1) {
            const int j = k - 1, st = j % STAGES, b = j & 1;
            if (!mbar_wait(p_full(b), (j >> 1) & 1, ctx)) break;
            tc_fence_after();
            const uint32_t sv = stage_v(st);
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk) {
              const uint64_t ad = sdesc_sw128(base + L::kOffP + b * L::kPBytes + kk * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(sv + kk * 16 * 128, L::kKVHalf, 1024);
              umma_bf16(tmem + L::kTmemO, ad, bd, kIdO, (j > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(pv_done(b));
            umma_commit(kv_empty(st));
          }
        }
        // every issued MMA completes before TMEM can be released
        umma_commit(drain());
        mbar_wait(drain(), 0, drain_ctx);
      }
    } else {
      // ------------------------------------------------------ softmax rows --
      const int r = row_in_tile();
      const uint32_t lt = lane_tmem();
      {  // this row's query into the swizzled Q tile (zeros for rows past the end)
        const uint4 *src = reinterpret_cast<const uint4 *>(pol.q_row(r));
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 v = src ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4 *>(smem + L::kOffQ + (c >> 3) * L::kQHalf + sw128_offset(r, c & 7)) = v;
        }
        fence_proxy_async_smem();
        mbar_arrive(q_full());
      }
      float m_used = -INFINITY, l = 0.f;
      for (int k = 0; k < num_tiles; ++k) {
        const int st = k % STAGES, b = k & 1;
        alive = __all_sync(0xffffffffu, mbar_wait(s_full(b), (k >> 1) & 1, ctx));
        if (!alive) break;
        tc_fence_after();
        uint32_t sraw[kBN];
        tmem_ld32(lt + b * kBN, *reinterpret_cast<uint32_t(*)[32]>(&sraw[0]));
        tmem_ld32(lt + b * kBN + 32, *reinterpret_cast<uint32_t(*)[32]>(&sraw[32]));
        uint64_t key_ok = pol.key_mask(k);  // bit j: key j of the tile takes part
        float x[kBN];
        float tmax = -INFINITY;
#pragma unroll
        for (int j = 0; j < kBN; ++j) {
          x[j] = ((key_ok >> j) & 1ull) ? __uint_as_float(sraw[j]) * pol.sl2 : -INFINITY;
          tmax = fmaxf(tmax, x[j]);
        }
        const bool need = tmax > m_used + kRescaleLog2 || (m_used == -INFINITY && tmax > -INFINITY);
        if (__any_sync(0xffffffffu, need)) {
          float alpha = 1.f;
          if (need) {
            alpha = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - tmax);
            m_used = tmax;
            l *= alpha;
          }
          if (k > 0) {  // O holds earlier tiles: let PV_{k-1} land, then scale it
            alive = __all_sync(0xffffffffu, mbar_wait(pv_done((k - 1) & 1), ((k - 1) >> 1) & 1, ctx));
            if (!alive) break;
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(lt + L::kTmemO + c0, o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(lt + L::kTmemO + c0, o);
            }
          }
        }
        const float mu = (m_used == -INFINITY) ? 0.f : m_used;
        float psum[kBN / PAGE];
#pragma unroll
        for (int pi = 0; pi < kBN / PAGE; ++pi) psum[pi] = 0.f;
#pragma unroll
        for (int j = 0; j < kBN; ++j) {
          const float p = fast_exp2(x[j] - mu);
          x[j] = p;
          psum[j / PAGE] += p;
        }
#pragma unroll
        for (int pi = 0; pi < kBN / PAGE; ++pi) l += psum[pi];
        if (k >= 2) {  // P buffer b was read by PV_{k-2}
          alive = __all_sync(0xffffffffu, mbar_wait(pv_done(b), ((k - 2) >> 1) & 1, ctx));
          if (!alive) break;
        }
        unsigned char *prow = smem + L::kOffP + b * L::kPBytes;
#pragma unroll
        for (int c = 0; c < kBN / 8; ++c) {
          uint4 v;
          v.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
          v.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
          v.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
          v.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
          *reinterpret_cast<uint4 *>(prow + sw128_offset(r, c)) = v;
        }
        // value rows of keys that take no part are zeroed so that 0 * stale data
        // cannot reach O (thread r < 64 looks after key r of the tile)
        if (r < kBN && !((key_ok >> r) & 1ull) && mbar_wait(kv_full(st), (k / STAGES) & 1, ctx)) {
          unsigned char *vrow = smem + (stage_v(st) - base) + r * 128;
#pragma unroll
          for (int hf = 0; hf < L::kHalves; ++hf)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4 *>(vrow + hf * L::kKVHalf + c * 16) = make_uint4(0, 0, 0, 0);
        }
        pol.after_tile(k, r, m_used, psum);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(s_free(b));
        mbar_arrive(p_full(b));
      }
      if (alive && num_tiles > 0) {
        const int j = num_tiles - 1;
        alive = __all_sync(0xffffffffu, mbar_wait(pv_done(j & 1), (j >> 1) & 1, ctx));
        if (alive) tc_fence_after();
      }
      m_out = m_used;
      l_out = l;
      alive = alive && num_tiles > 0;
    }
    return alive;
  }

  // 32 columns [c0, c0+32) of this softmax thread's O row (warp-collective).
  __device__ __forceinline__ void load_o(int c0, uint32_t (&o)[32]) const {
    sm100::tmem_ld32(lane_tmem() + L::kTmemO + c0, o);
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
