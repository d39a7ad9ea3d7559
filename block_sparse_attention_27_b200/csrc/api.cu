// api.cu -- the C ABI declared in include/dsa.h: argument checks, workspace
// layout, launches.  No allocation, no synchronisation (except dsa_get_status).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "dsa.h"
#include "launch.h"

namespace {

using dsa::Shape;

constexpr int kMaxDevices = 64;

int num_sms_current() {
  static int cache[kMaxDevices] = {0};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates dims; fills Shape.  Returns DSA_OK or an error code.
int make_shape(const dsa_dims *dims, Shape *out) {
  if (!dims) return DSA_ERR_INVALID_ARG;
  const dsa_dims &d = *dims;
  if (d.S <= 0 || d.B <= 0 || d.Hq <= 0 || d.Hkv <= 0 || d.d <= 0 || d.page <= 0 ||
      d.max_pages <= 0 || d.kmax <= 0 || d.n_phys <= 0)
    return DSA_ERR_INVALID_ARG;
  if (d.Hq % d.Hkv != 0) return DSA_ERR_INVALID_ARG;
  if (d.d != 64 && d.d != 128) return DSA_ERR_UNSUPPORTED;
  if (d.page != 16 && d.page != 32 && d.page != 64) return DSA_ERR_UNSUPPORTED;
  const int G = d.Hq / d.Hkv;
  if ((long long)d.B * G > 256) return DSA_ERR_UNSUPPORTED;
  if ((long long)d.max_pages * d.page > (1LL << 30)) return DSA_ERR_UNSUPPORTED;
  if (d.sm_limit < 0) return DSA_ERR_INVALID_ARG;
  if (d.head_budget != 0 && d.head_budget != 1) return DSA_ERR_INVALID_ARG;
  if (d.head_budget && d.Hkv > dsa::kMaxHeadsAdaptive) return DSA_ERR_UNSUPPORTED;
  if (d.early_gather != 0 && d.early_gather != 1) return DSA_ERR_INVALID_ARG;
  Shape s{};
  s.S = d.S; s.B = d.B; s.Hq = d.Hq; s.Hkv = d.Hkv; s.G = G; s.BG = d.B * G;
  s.d = d.d; s.P = d.page; s.max_pages = d.max_pages; s.kmax = d.kmax;
  s.n_phys = d.n_phys;
  s.page_table = d.page_table;
  s.sl2 = (float)(1.4426950408889634 / std::sqrt((double)d.d));
  s.sm_limit = d.sm_limit;
  s.lse_out = d.lse_out;
  s.head_budget = d.head_budget;
  s.active = d.active;
  s.prefix_o = static_cast<__nv_bfloat16 *>(d.prefix_o_cache);
  s.prefix_lse = d.prefix_lse_cache;
  s.early_gather = (d.early_gather && !d.active) ? 1 : 0;  // prefix-part reuse decides per step
  *out = s;
  return DSA_OK;
}

// SMs the selection pass plans for: the device's, or fewer when the caller sets
// a budget so that it runs beside other work
int select_sms(const Shape &sh) {
  const int n = num_sms_current();
  return sh.sm_limit > 0 ? std::min(n, sh.sm_limit) : n;
}

template <class T>
T *at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<unsigned char *>(ws) + off);
}

}  // namespace

// Scratch of dsa_select_static_scratch, for callers that may not allocate (a
// runtime plugin handed only its inputs and outputs, a path running while the
// memory pool is fully reserved).  The CUDA module sets it aside on each device
// when it is loaded; no allocation call is involved.  One array per device, so
// calls on one device must not overlap in time.
static __device__ __align__(256) unsigned char select_static_scratch[DSA_SELECT_STATIC_SCRATCH_BYTES];

namespace {

// Device address of select_static_scratch on the current device, looked up once
// per device (the lookup may load the module, hence: first call outside capture).
void *static_scratch_current() {
  static void *cache[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, select_static_scratch) != cudaSuccess) return nullptr;
    cache[dev] = p;
  }
  return cache[dev];
}

}  // namespace

extern "C" {

int dsa_version(void) { return 100; }

int dsa_kernels_per_call(int pass) {
  if (pass == 0) return dsa::kSelectLaunches;
  if (pass == 1) return dsa::kSparseLaunches;
  if (pass == 2) return dsa::kMergeLaunches;
  return DSA_ERR_INVALID_ARG;
}

const char *dsa_strerror(int code) {
  switch (code) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad shape or value)";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape (d must be 64 or 128, page 16/32/64, B*Hq/Hkv <= 256)";
    case DSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case DSA_ERR_CUDA: return "CUDA runtime or launch error";
    case DSA_ERR_DEVICE_TIMEOUT: return "a bounded device wait gave up";
    case DSA_ERR_BAD_INDEX: return "page index or page-table entry out of range";
    case DSA_ERR_NONFINITE: return "non-finite page score (non-finite inputs)";
    case DSA_ERR_SCRATCH_LIMIT:
      return "shape needs more scratch than the 16 MiB static array of dsa_select_static_scratch "
             "(use dsa_select with a caller workspace)";
    default: return "unknown status code";
  }
}

int dsa_sparse_kernel(const dsa_dims *dims) {
  Shape sh;
  const int rc = make_shape(dims, &sh);
  if (rc != DSA_OK) return rc;
  const int c = dsa::sparse_resident_cluster(sh);
  return c > 0 ? 1 + c : 1;
}

int dsa_select_launches(const dsa_dims *dims) {
  Shape sh;
  const int rc = make_shape(dims, &sh);
  if (rc != DSA_OK) return rc;
  return dsa::plan_select(sh, select_sms(sh)).launches + (sh.head_budget ? dsa::kGlobalLaunches : 0);
}

size_t dsa_select_workspace_size(const dsa_dims *dims) {
  Shape sh;
  if (make_shape(dims, &sh) != DSA_OK) return 0;
  return dsa::plan_select(sh, select_sms(sh)).total;
}

size_t dsa_sparse_workspace_size(const dsa_dims *dims) {
  Shape sh;
  if (make_shape(dims, &sh) != DSA_OK) return 0;
  return dsa::plan_sparse(sh, num_sms_current()).total;
}

int dsa_workspace_init(void *workspace, size_t ws_bytes, dsa_stream_t stream) {
  if (!workspace || ws_bytes < dsa::kWorkspaceHeader || !aligned16(workspace))
    return DSA_ERR_INVALID_ARG;
  if (cudaMemsetAsync(workspace, 0, dsa::kWorkspaceHeader, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

int dsa_get_status(const void *workspace, dsa_stream_t stream) {
  if (!workspace) return DSA_ERR_INVALID_ARG;
  uint32_t word = 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  if (word & dsa::kStatusTimeout) return DSA_ERR_DEVICE_TIMEOUT;
  if (word & dsa::kStatusBadIndex) return DSA_ERR_BAD_INDEX;
  if (word & dsa::kStatusNonfinite) return DSA_ERR_NONFINITE;
  return DSA_OK;
}

int dsa_select(const void *q_blk, const void *k_cache, const void *v_cache,
               const int32_t *n_ctx, int32_t page, const int32_t *topk,
               int32_t *idx_out, void *o_out, dsa_stream_t stream,
               const dsa_dims *dims, int32_t *cnt_out,
               void *workspace, size_t ws_bytes) {
  Shape sh;
  int rc = make_shape(dims, &sh);
  if (rc != DSA_OK) return rc;
  if (page != sh.P) return DSA_ERR_INVALID_ARG;
  if (!q_blk || !k_cache || !v_cache || !n_ctx || !topk || !idx_out || !o_out || !cnt_out ||
      !workspace)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_blk) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o_out) ||
      !aligned16(workspace))
    return DSA_ERR_INVALID_ARG;
  const dsa::SelectPlan plan = dsa::plan_select(sh, select_sms(sh));
  if (ws_bytes < plan.total) return DSA_ERR_WORKSPACE_TOO_SMALL;
  dsa::SelectArgs a{};
  a.q = static_cast<const __nv_bfloat16 *>(q_blk);
  a.k = static_cast<const __nv_bfloat16 *>(k_cache);
  a.v = static_cast<const __nv_bfloat16 *>(v_cache);
  a.n_ctx = n_ctx;
  a.topk = topk;
  a.idx_out = idx_out;
  a.cnt_out = cnt_out;
  a.o_out = static_cast<__nv_bfloat16 *>(o_out);
  a.part_o = at<float>(workspace, plan.off_part_o);
  a.part_ml = at<float>(workspace, plan.off_part_ml);
  a.pagepart = at<float>(workspace, plan.off_pagepart);
  a.mtile = at<float>(workspace, plan.off_mtile);
  a.scores = at<float>(workspace, plan.off_scores);
  a.cand = at<uint64_t>(workspace, plan.off_cand);
  a.ccnt = at<int32_t>(workspace, plan.off_ccnt);
  a.hsel = at<int32_t>(workspace, plan.off_hsel);
  a.hcnt = at<int32_t>(workspace, plan.off_hcnt);
  a.counters = at<uint32_t>(workspace, plan.off_counters);
  a.status = at<uint32_t>(workspace, 0);
  if (dsa::launch_select(sh, plan, a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

int dsa_select_static_scratch(const void *q_blk, const void *k_cache, const void *v_cache,
                              const int32_t *n_ctx, int32_t page, const int32_t *topk,
                              int32_t *idx_out, void *o_out, dsa_stream_t stream,
                              const dsa_dims *dims, int32_t *cnt_out, uint32_t *status) {
  Shape sh;
  int rc = make_shape(dims, &sh);
  if (rc != DSA_OK) return rc;
  if (page != sh.P) return DSA_ERR_INVALID_ARG;
  if (!q_blk || !k_cache || !v_cache || !n_ctx || !topk || !idx_out || !o_out || !cnt_out ||
      !status)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_blk) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o_out) ||
      (reinterpret_cast<uintptr_t>(status) & 3u) != 0)
    return DSA_ERR_INVALID_ARG;
  const dsa::SelectPlan plan = dsa::plan_select(sh, select_sms(sh));
  if (plan.total > DSA_SELECT_STATIC_SCRATCH_BYTES) return DSA_ERR_SCRATCH_LIMIT;
  void *scratch = static_scratch_current();
  if (scratch == nullptr) return DSA_ERR_CUDA;
  dsa::SelectArgs a{};
  a.q = static_cast<const __nv_bfloat16 *>(q_blk);
  a.k = static_cast<const __nv_bfloat16 *>(k_cache);
  a.v = static_cast<const __nv_bfloat16 *>(v_cache);
  a.n_ctx = n_ctx;
  a.topk = topk;
  a.idx_out = idx_out;
  a.cnt_out = cnt_out;
  a.o_out = static_cast<__nv_bfloat16 *>(o_out);
  a.part_o = at<float>(scratch, plan.off_part_o);
  a.part_ml = at<float>(scratch, plan.off_part_ml);
  a.pagepart = at<float>(scratch, plan.off_pagepart);
  a.mtile = at<float>(scratch, plan.off_mtile);
  a.scores = at<float>(scratch, plan.off_scores);
  a.cand = at<uint64_t>(scratch, plan.off_cand);
  a.ccnt = at<int32_t>(scratch, plan.off_ccnt);
  a.hsel = at<int32_t>(scratch, plan.off_hsel);
  a.hcnt = at<int32_t>(scratch, plan.off_hcnt);
  a.counters = at<uint32_t>(scratch, plan.off_counters);
  a.status = status;  // the caller's word; the array's header holds only the group counters
  if (dsa::launch_select(sh, plan, a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

int dsa_merge_attn(const void *o_a, const float *lse_a, const void *o_b, const float *lse_b,
                   void *o_out, float *lse_out, int64_t rows, int32_t d, dsa_stream_t stream) {
  if (!o_a || !lse_a || !o_b || !lse_b || !o_out || rows < 0 || d <= 0 || d % 8 != 0)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(o_a) || !aligned16(o_b) || !aligned16(o_out)) return DSA_ERR_INVALID_ARG;
  if (rows == 0) return DSA_OK;
  if (dsa::launch_merge(static_cast<const __nv_bfloat16 *>(o_a), lse_a,
                        static_cast<const __nv_bfloat16 *>(o_b), lse_b,
                        static_cast<__nv_bfloat16 *>(o_out), lse_out, rows, d,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

int dsa_sparse_attn(const void *q_blk, const void *k_cache, const void *v_cache,
                    const int32_t *idx, const void *blk_k, const void *blk_v,
                    void *o_out, dsa_stream_t stream,
                    const dsa_dims *dims, const int32_t *n_ctx, const int32_t *idx_cnt,
                    void *workspace, size_t ws_bytes) {
  Shape sh;
  int rc = make_shape(dims, &sh);
  if (rc != DSA_OK) return rc;
  if (!q_blk || !k_cache || !v_cache || !idx || !blk_k || !blk_v || !o_out || !n_ctx ||
      !idx_cnt || !workspace)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_blk) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(blk_k) ||
      !aligned16(blk_v) || !aligned16(o_out) || !aligned16(workspace))
    return DSA_ERR_INVALID_ARG;
  if (sh.active && (!sh.prefix_o || !sh.prefix_lse || !aligned16(sh.prefix_o) ||
                    (reinterpret_cast<uintptr_t>(sh.prefix_lse) & 3u) != 0))
    return DSA_ERR_INVALID_ARG;
  const dsa::SparsePlan plan = dsa::plan_sparse(sh, num_sms_current());
  if (ws_bytes < plan.total) return DSA_ERR_WORKSPACE_TOO_SMALL;
  dsa::SparseArgs a{};
  a.q = static_cast<const __nv_bfloat16 *>(q_blk);
  a.k = static_cast<const __nv_bfloat16 *>(k_cache);
  a.v = static_cast<const __nv_bfloat16 *>(v_cache);
  a.blk_k = static_cast<const __nv_bfloat16 *>(blk_k);
  a.blk_v = static_cast<const __nv_bfloat16 *>(blk_v);
  a.idx = idx;
  a.idx_cnt = idx_cnt;
  a.n_ctx = n_ctx;
  a.o_out = static_cast<__nv_bfloat16 *>(o_out);
  a.status = at<uint32_t>(workspace, 0);
  a.xchg = at<unsigned char>(workspace, plan.off_xchg);
  if (dsa::launch_sparse(sh, plan, a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

}  // extern "C"
