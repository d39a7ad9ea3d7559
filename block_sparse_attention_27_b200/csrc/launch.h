// launch.h -- internal interface between the C-ABI host code (api.cu) and the
// kernel files.  Not installed; the public interface is include/dsa.h.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dsa {

// Shape of one call, resolved on the host.
struct Shape {
  int S, B, Hq, Hkv, G, BG, d, P, max_pages, kmax;
  long long n_phys;
  const int32_t *page_table;  // may be null (identity)
  float sl2;                  // log2(e) / sqrt(d)
  int sm_limit;               // selection pass: SMs it may hold (0 = all)
  float *lse_out;             // optional [S, B, Hq]: each row's log-sum-exp (natural log)
  int head_budget;            // selection pass: 1 = one budget of Hkv*kp pages per sequence
  const uint8_t *active;      // sparse pass: optional [S, B] active tokens (prefix-part reuse)
  __nv_bfloat16 *prefix_o;    // with active: [S, B, Hq, D] normalised prefix parts
  float *prefix_lse;          // with active: [S, B, Hq] their log-sum-exps (natural log)
  int early_gather;           // sparse pass: gather the selected pages before the dependency wait
};

// TMA map of a paged cache [n_phys, Hkv, P, D] viewed as rows of D bf16; boxes of
// box_rows rows x 64 elements with the 128-byte swizzle (tmap.cu).
cudaError_t make_kv_tensor_map(CUtensorMap *out, const void *base, long long rows, int D,
                               int box_rows);

// The same cache as 4-D (D, P, Hkv, n_phys); boxes of 64 elements x P tokens x 1 head
// x `pages` consecutive physical pages (tmap.cu).
cudaError_t make_kv_pages_tensor_map(CUtensorMap *out, const void *base, long long n_phys, int Hkv,
                                     int P, int D, int pages);

// The block's own keys/values [S*B, Hkv, D] bf16; boxes of 64 elements x 1 head x
// box_tokens tokens with the 128-byte swizzle (tmap.cu).
cudaError_t make_blk_tensor_map(CUtensorMap *out, const void *base, long long tokens, int Hkv,
                                int D, int box_tokens = 64);

// The block's queries [S*B, Hq, D] bf16; boxes of 64 elements x G heads x
// box_tokens tokens with the 128-byte swizzle (tmap.cu).
cudaError_t make_q_tensor_map(CUtensorMap *out, const void *base, long long tokens, int Hq, int D,
                              int G, int box_tokens);

// Kernel launches issued by one dsa_select (when all its (sequence, KV head)
// groups fit in one co-resident launch; see SelectPlan::launches) and by one
// dsa_sparse_attn call.
constexpr int kSelectLaunches = 1;
// extra launch of the selection pass under the head-adaptive budget, and the
// most KV heads it supports
constexpr int kGlobalLaunches = 1;
constexpr int kMaxHeadsAdaptive = 64;
constexpr int kSparseLaunches = 1;
constexpr int kMergeLaunches = 1;

// dsa_merge_attn (merge.cu)
cudaError_t launch_merge(const __nv_bfloat16 *o_a, const float *lse_a, const __nv_bfloat16 *o_b,
                         const float *lse_b, __nv_bfloat16 *o_out, float *lse_out, long long rows,
                         int d, cudaStream_t stream);

// ---- selection pass ----
struct SelectPlan {
  int rowtiles;          // ceil(BG / 128)
  int splits;            // key splits per (seq, KV head, row tile)
  int tiles_per_split;   // 64-token tiles per split
  int max_tiles;         // ceil(max_pages * P / 64)
  int group_ctas;        // CTAs of one (seq, KV head) group: splits * rowtiles
  int groups_per_launch; // groups of one co-resident (cooperative) launch
  int launches;          // ceil(S * Hkv / groups_per_launch)
  int bgp;               // BG rounded up to a multiple of 4: row stride of pagepart / mtile
  int slot_len;          // entries of one CTA's candidate list
  size_t off_counters;   // in the zeroed header: four counters per group of a launch
  size_t off_part_o, off_part_ml, off_pagepart, off_mtile, off_scores, off_cand, off_ccnt, off_hsel,
      off_hcnt, total;
};

// Counters of a group (barrier arrivals, candidate hand-offs, output rows taken,
// CTAs done with output rows): 4 per group, in the workspace header after its
// first 256 bytes.
constexpr int kMaxGroupsPerLaunch = 240;

struct SelectArgs {
  const __nv_bfloat16 *q, *k, *v;
  const int32_t *n_ctx, *topk;
  int32_t *idx_out, *cnt_out;
  __nv_bfloat16 *o_out;
  float *part_o;      // [S*Hkv][splits][BG][D] unnormalised split outputs
  float *part_ml;     // [S*Hkv][splits][BG] (m, l) of each split (log2 domain)
  float *pagepart;    // [S*Hkv][max_tiles][bgp][units per tile]
  float *mtile;       // [S*Hkv][max_tiles][bgp]
  float *scores;      // [S*Hkv][max_pages]
  uint64_t *cand;     // [S*Hkv][group_ctas][slot_len] local candidates (score bits << 32 | ~page)
  int32_t *ccnt;      // [S*Hkv][group_ctas] candidates of each CTA
  int32_t *hsel;      // [S*Hkv][max_pages] head-adaptive budget: each head's best pages
  int32_t *hcnt;      // [S*Hkv] their number
  uint32_t *counters; // [groups_per_launch][4] (arrive, leave, output rows, done)
  uint32_t *status;
};

SelectPlan plan_select(const Shape &sh, int num_sms);
cudaError_t launch_select(const Shape &sh, const SelectPlan &plan, const SelectArgs &a,
                          cudaStream_t stream);

// ---- sparse pass ----
struct SparsePlan {
  int rowtiles;   // ceil(BG / 128)
  int cluster;    // CTAs per (seq, KV head, row tile): one thread-block cluster
  int ppc;        // selected pages per CTA of the cluster
  int blk_tiles;  // ceil(B / 64): tiles over the block's own tokens (last CTA)
  size_t off_xchg;    // workspace offset of the partial-row exchange area
  size_t xchg_slot;   // bytes of one CTA's partial rows in that area
  size_t total;       // workspace bytes
};

struct SparseArgs {
  const __nv_bfloat16 *q, *k, *v, *blk_k, *blk_v;
  const int32_t *idx, *idx_cnt, *n_ctx;
  __nv_bfloat16 *o_out;
  uint32_t *status;
  unsigned char *xchg;  // partial rows of every cluster, [S][Hkv][rowtiles][16 slots]
};

SparsePlan plan_sparse(const Shape &sh, int num_sms);
// The sparse pass on the kernel whose CTAs hold all their keys in shared memory
// (sparse_resident.cu): returns false (nothing launched) when the shape does not
// fit it or uses prefix-part reuse; else launches and sets *err.
bool launch_sparse_resident(const Shape &sh, const SparseArgs &a, cudaStream_t stream, cudaError_t *err);
// Cluster size the all-keys-resident kernel would use for this shape on the
// current device, 0 when the streaming kernel serves it.
int sparse_resident_cluster(const Shape &sh);
cudaError_t launch_sparse(const Shape &sh, const SparsePlan &plan, const SparseArgs &a,
                          cudaStream_t stream);

}  // namespace dsa
