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
#include <cuda_fp16.h>

#include <algorithm>

#include "launch.h"
#include "sm100.cuh"
#include "tc_attn.cuh"

namespace dsa {
namespace {

constexpr int kSpStages = 2;
constexpr int kRowsPerCta = 128;
constexpr int kMaxCluster = 16;

// Exchange buffers of the cluster merge.  A row is the CTA's normalised output
// row O/l in fp16 (D values) followed by (m, l, -, -) in fp32; the receive
// buffer (128 rows: rpc rows from each of the C CTAs) lies after every region
// the attention engine uses, so data from a CTA that finished early cannot
// land on tiles that are still being read.
template <int D>
struct MergeLayout {
  static constexpr uint32_t kRowBytes = D * 2 + 16;
  template <int STAGES>
  static constexpr uint32_t kRecvOffset() {
    return (tc::Layout<D, STAGES>::kBytes + 1023u) & ~1023u;
  }
  // the page table of the CTA's selected entries (int2 each) follows
  template <int STAGES>
  static constexpr uint32_t kTableOffset() {
    return kRecvOffset<STAGES>() + 128u * kRowBytes;
  }
  template <int STAGES>
  static constexpr size_t kSmem(int ppc) {
    return kTableOffset<STAGES>() + 8u * (uint32_t)ppc + 1024u;  // + alignment slack
  }
};

struct SparseParams {
  Shape sh;
  SparsePlan plan;
  SparseArgs a;
};

template <int D, int PAGE>
struct SparsePolicy {
  // the CTA's selected pages are resolved once (prepare) into a shared-memory
  // table of (logical page, physical page); the first loads wait for it
  static constexpr bool kIssueBeforeSync = false;
  static constexpr int kPagesPerTile = tc::kBN / PAGE;
  const CUtensorMap *kmap, *vmap, *kmap4, *vmap4, *bkmap, *bvmap;
  const int32_t *idx_row;       // idx[s, h, :]
  const int32_t *page_row;      // page-table row of the sequence, or null (identity)
  const __nv_bfloat16 *q_head;  // q[s, 0, h*G, 0]
  uint32_t *status;
  const int2 *tab;              // shared: (lp, phys) per entry of this CTA, phys < 0 = unusable
  uint32_t tab_off;             // byte offset of the table in the aligned shared memory
  long long n_phys, phys0;
  int Hkv, h, G, Hq, B, BG, s, n, np, e_begin, e_end, sel_tiles, row_base;
  float sl2;

  __device__ __forceinline__ void prepare(unsigned char *smem) {
    int2 *t = reinterpret_cast<int2 *>(smem + tab_off);
    for (int e = e_begin + (int)threadIdx.x; e < e_end; e += (int)blockDim.x) {
      const int lp = idx_row[e];
      int phys = -1;
      if (lp >= 0 && lp < np) {
        const long long p = page_row ? (long long)page_row[lp] : phys0 + lp;
        if (p >= 0 && p < n_phys) phys = (int)p;
      }
      if (phys < 0) raise_status(status, kStatusBadIndex);
      t[e - e_begin] = make_int2(lp, phys);
    }
    tab = t;
  }
  __device__ __forceinline__ void prefetch() const {
    sm100::tma_prefetch_map(kmap);
    sm100::tma_prefetch_map(vmap);
    sm100::tma_prefetch_map(kmap4);
    sm100::tma_prefetch_map(vmap4);
    sm100::tma_prefetch_map(bkmap);
    sm100::tma_prefetch_map(bvmap);
  }
  __device__ __forceinline__ int2 entry(int e) const {
    return e < e_end ? tab[e - e_begin] : make_int2(-1, -1);
  }
  __device__ __forceinline__ void load_tile(int k, uint32_t sk, uint32_t sv, uint32_t half_bytes,
                                            uint32_t bar) const {
    if (k < sel_tiles) {
      const int e0 = e_begin + k * kPagesPerTile;
      int phys[kPagesPerTile];
      uint32_t nvalid = 0;
      bool run = true;  // all pages usable and physically consecutive
#pragma unroll
      for (int pi = 0; pi < kPagesPerTile; ++pi) {
        phys[pi] = entry(e0 + pi).y;
        nvalid += phys[pi] >= 0;
        run = run && phys[pi] >= 0 && phys[pi] == phys[0] + pi;
      }
      sm100::mbar_arrive_expect_tx(bar, nvalid * PAGE * 128u * (D / 64) * 2u);
      if (kPagesPerTile > 1 && run) {  // the whole tile in one box per half
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          sm100::tma_load_4d(sk + hf * half_bytes, kmap4, bar, hf * 64, 0, h, phys[0]);
          sm100::tma_load_4d(sv + hf * half_bytes, vmap4, bar, hf * 64, 0, h, phys[0]);
        }
        return;
      }
#pragma unroll
      for (int pi = 0; pi < kPagesPerTile; ++pi) {
        if (phys[pi] < 0) continue;
        const int y = (int)(((long long)phys[pi] * Hkv + h) * PAGE);
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
        sm100::tma_load_3d(sk + hf * half_bytes, bkmap, bar, hf * 64, h, s * B + j * 64);
        sm100::tma_load_3d(sv + hf * half_bytes, bvmap, bar, hf * 64, h, s * B + j * 64);
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
    uint64_t m = 0;
    if (k < sel_tiles) {
      const int e0 = e_begin + k * kPagesPerTile;
#pragma unroll
      for (int pi = 0; pi < kPagesPerTile; ++pi) {
        const int2 t = entry(e0 + pi);
        if (t.y < 0) continue;
        const int cnt = min(PAGE, n - t.x * PAGE);
        if (cnt > 0) m |= ((cnt >= 64) ? ~0ull : ((1ull << cnt) - 1ull)) << (pi * PAGE);
      }
    } else {
      const int cnt = min(64, B - (k - sel_tiles) * 64);
      if (cnt > 0) m = (cnt >= 64) ? ~0ull : ((1ull << cnt) - 1ull);
    }
    return m;
  }
  __device__ __forceinline__ void after_tile(int, int, float, const float *) const {}
};

template <int D, int PAGE>
__global__ void __launch_bounds__(tc::kThreads, 1)
    sparse_attn(const __grid_constant__ SparseParams prm, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap kmap4,
                const __grid_constant__ CUtensorMap vmap4, const __grid_constant__ CUtensorMap bkmap,
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

  SparsePolicy<D, PAGE> pol;
  pol.kmap = &kmap;
  pol.vmap = &vmap;
  pol.kmap4 = &kmap4;
  pol.vmap4 = &vmap4;
  pol.bkmap = &bkmap;
  pol.bvmap = &bvmap;
  pol.idx_row = a.idx + sh_idx * sh.kmax;
  pol.page_row = sh.page_table ? sh.page_table + (size_t)s * sh.max_pages : nullptr;
  pol.q_head = a.q + ((size_t)s * sh.B * sh.Hq + (size_t)h * sh.G) * D;
  pol.status = a.status;
  pol.tab = nullptr;
  pol.tab_off = MergeLayout<D>::template kTableOffset<kSpStages>();
  pol.n_phys = sh.n_phys;
  pol.phys0 = (long long)s * sh.max_pages;
  pol.Hkv = sh.Hkv;
  pol.h = h;
  pol.G = sh.G;
  pol.Hq = sh.Hq;
  pol.B = sh.B;
  pol.BG = sh.BG;
  pol.s = s;
  pol.n = n;
  pol.np = (n + PAGE - 1) / PAGE;
  pol.e_begin = e_begin;
  pol.e_end = e_end;
  pol.sel_tiles = sel_tiles;
  pol.row_base = row_base;
  pol.sl2 = sh.sl2;
  if (threadIdx.x == 0) DSA_TRACE_EVENT(0);
  tc::Engine<D, kSpStages> eng;
  eng.init(smem_raw, a.status, pol, num_tiles);
  // this CTA will receive one slice of rpc rows from every CTA of the cluster
  using M = MergeLayout<D>;
  const int rpc = kRowsPerCta / C;  // C is a power of two <= 16
  if (threadIdx.x == 0) sm100::mbar_arrive_expect_tx(eng.user_bar(), kRowsPerCta * M::kRowBytes);
  sm100::cluster_arrive();  // barrier init and expected bytes are visible to the cluster

  float m, l;
  eng.template run<PAGE>(pol, num_tiles, m, l);
  float m_row, l_row, wa, wb;
  eng.finish(m, l, m_row, l_row, wa, wb);

  // ---- stage: this CTA's rows, normalised (O / l) in fp16, with (m, l) in fp32,
  //      into the send buffer (the Q / K/V area, free now that every MMA is done)
  unsigned char *sendb = eng.smem;
  if (eng.warp >= 2) {
    const int r = eng.row_in_tile();
    const int g = eng.group();
    const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
    const float ca = wa * inv, cb = wb * inv;
    unsigned char *row = sendb + r * M::kRowBytes;
#pragma unroll
    for (int c0 = g * (D / 2); c0 < (g + 1) * (D / 2); c0 += 32) {
      uint32_t oa[32], ob[32];
      eng.load_o(0, c0, oa);
      eng.load_o(1, c0, ob);
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
            f[z] = (ca > 0.f ? ca * __uint_as_float(oa[i]) : 0.f) +
                   (cb > 0.f ? cb * __uint_as_float(ob[i]) : 0.f);
          }
          __half2 hv = __floats2half2_rn(f[0], f[1]);
          pv[e] = *reinterpret_cast<uint32_t *>(&hv);
        }
        *reinterpret_cast<uint4 *>(row + c0 * 2 + q * 16) = v;
      }
    }
    if (g == 0) *reinterpret_cast<float4 *>(row + D * 2) = make_float4(m_row, l_row, 0.f, 0.f);
    sm100::fence_proxy_async_smem();
    if (r == 0 && g == 0) DSA_TRACE_EVENT(7);
  }
  __syncthreads();
  sm100::cluster_wait();  // every CTA of the cluster has armed its receive barrier
  if (threadIdx.x == 0) DSA_TRACE_EVENT(8);
  const uint32_t recv = eng.base + M::template kRecvOffset<kSpStages>();
  if (threadIdx.x == 0) {
    const uint32_t send = smem_addr(sendb);
    for (int j = 0; j < C; ++j)
      sm100::bulk_copy_to_cluster(sm100::cluster_map(recv + c * rpc * M::kRowBytes, j),
                                  send + j * rpc * M::kRowBytes, rpc * M::kRowBytes,
                                  sm100::cluster_map(eng.user_bar(), j));
    sm100::bulk_commit();
  }

  // ---- receive this CTA's rows from every CTA and merge them
  const bool got = __syncthreads_and(sm100::mbar_wait(eng.user_bar(), 0, eng.ctx));
  if (threadIdx.x == 0) DSA_TRACE_EVENT(9);
  const int rows_here = min(kRowsPerCta, sh.BG - row_base);
  const int r0 = c * rpc;
  const unsigned char *rb = eng.smem + M::template kRecvOffset<kSpStages>();
  constexpr int kChunks = D / 8;  // 8 values (16 bytes of fp16) per work item
  for (int t = threadIdx.x; got && t < rpc * kChunks; t += blockDim.x) {
    const int rl = t / kChunks, ch = t % kChunks;
    if (r0 + rl >= rows_here) continue;
    float mx = -INFINITY;
    for (int j = 0; j < C; ++j) {
      const float2 st = *reinterpret_cast<const float2 *>(rb + (j * rpc + rl) * M::kRowBytes + D * 2);
      if (st.y > 0.f) mx = fmaxf(mx, st.x);
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float lsum = 0.f;
    for (int j = 0; j < C; ++j) {
      const unsigned char *src = rb + (j * rpc + rl) * M::kRowBytes;
      const float2 st = *reinterpret_cast<const float2 *>(src + D * 2);
      if (!(st.y > 0.f)) continue;  // an empty partial
      const float w = exp2f(st.x - mx) * st.y;
      lsum += w;
      const uint4 v = *reinterpret_cast<const uint4 *>(src + ch * 16);
      const __half2 *hv = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(hv[e]);
        acc[2 * e] += w * f.x;
        acc[2 * e + 1] += w * f.y;
      }
    }
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    const int grow = row_base + r0 + rl;
    const int b = grow / sh.G, g = grow % sh.G;
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
  if (threadIdx.x == 0) {
    DSA_TRACE_EVENT(10);
    sm100::bulk_wait_read_all();  // outgoing copies have read the send buffer
  }
  eng.teardown();
  if (threadIdx.x == 0) DSA_TRACE_EVENT(11);
}

// Clusters of `cs` CTAs that can be resident at once with this kernel's shared
// memory (index log2(cs)), queried once per device.
template <auto K>
const int *active_clusters(size_t smem) {
  static int cached[64][5];
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (!done[dev]) {
    for (int lg = 0; lg <= 4; ++lg) {
      const int cs = 1 << lg;
      cached[dev][lg] = 0;
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
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, K, &cfg) == cudaSuccess) cached[dev][lg] = n;
      cudaGetLastError();
    }
    done[dev] = true;
  }
  return cached[dev];
}

// Cluster size for `nclusters` clusters sharing `kmax` pages each: the size with
// the smallest (waves x pages per CTA), larger clusters on ties.
inline int choose_cluster(const int *active, int nclusters, int kmax, int cap) {
  int best = 1;
  long long best_cost = -1;
  for (int lg = 4; lg >= 0; --lg) {
    const int cs = 1 << lg;
    if (cs > cap || active[lg] < 1) continue;
    const long long waves = (nclusters + active[lg] - 1) / active[lg];
    const long long cost = waves * ((kmax + cs - 1) / cs + 1);  // +1: fixed per-CTA cost
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = cs;
    }
  }
  return best;
}

template <int D, int PAGE>
cudaError_t launch_typed(const Shape &sh, const SparsePlan &plan_in, const SparseArgs &a,
                         cudaStream_t stream) {
  constexpr auto kern = sparse_attn<D, PAGE>;
  constexpr size_t kMaxSmem = 227 * 1024;
  cudaError_t err = set_smem_once<kern>(kMaxSmem);
  if (err != cudaSuccess) return err;
  SparsePlan plan = plan_in;
  const int cs = choose_cluster(active_clusters<kern>(MergeLayout<D>::template kSmem<kSpStages>(
                                    (sh.kmax + plan.cluster - 1) / plan.cluster)),
                                sh.Hkv * sh.S * plan.rowtiles, sh.kmax, plan.cluster);
  plan.cluster = cs;
  plan.ppc = (sh.kmax + cs - 1) / cs;
  const size_t smem = MergeLayout<D>::template kSmem<kSpStages>(plan.ppc);
  if (smem > kMaxSmem) return cudaErrorInvalidValue;
  CUtensorMap kmap, vmap, kmap4, vmap4, bkmap, bvmap;
  const long long rows = sh.n_phys * sh.Hkv * PAGE;
  if ((err = make_kv_tensor_map(&kmap, a.k, rows, D, PAGE)) != cudaSuccess) return err;
  if ((err = make_kv_tensor_map(&vmap, a.v, rows, D, PAGE)) != cudaSuccess) return err;
  if ((err = make_kv_pages_tensor_map(&kmap4, a.k, sh.n_phys, sh.Hkv, PAGE, D, tc::kBN / PAGE)) != cudaSuccess)
    return err;
  if ((err = make_kv_pages_tensor_map(&vmap4, a.v, sh.n_phys, sh.Hkv, PAGE, D, tc::kBN / PAGE)) != cudaSuccess)
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
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = plan.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, kern, prm, kmap, vmap, kmap4, vmap4, bkmap, bvmap);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

DSA_TRACE_EXPORT(dsa_trace_sparse)

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
