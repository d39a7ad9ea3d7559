/*
 * dsa.h -- C ABI of libdsa: shared-index top-k sparse KV attention for
 * block-diffusion LLMs on NVIDIA B200 (sm_100a).
 *
 * The method ("MAGE: All-[MASK] Block Already Knows Where to Look in Block
 * Diffusion LLM"): all B query tokens of a denoising block share ONE set of KV
 * pages per KV head (Problem section).  Step 1 of the block runs one exact
 * attention pass over the whole prefix and keeps the top-k pages (Approach:
 * selection), every later denoising step attends only to those pages plus the
 * block's own tokens, reusing the step-1 indices (Approach: reuse).  Selection is
 * meant to run on a second CUDA stream (Approach: "async CUDA stream").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  Element types: q/k/v/blk_k/blk_v/o are bf16 (2-byte IEEE bfloat16); index
 *  arrays are int32.  Every pointer passed here is a DEVICE pointer unless the
 *  argument says "host".  The caller owns all memory; the library allocates
 *  nothing and keeps no state except a per-device cache of the SM count (and the
 *  fixed scratch array of dsa_select_static_scratch, see there).
 *
 *  Layouts (row-major, innermost last):
 *    q_blk        [S, B, Hq, d]          queries of the block (post-RoPE)
 *    k_cache      [n_phys, Hkv, page, d] paged key cache
 *    v_cache      [n_phys, Hkv, page, d] paged value cache
 *    page_table   [S, max_pages]         logical page -> physical page (int32);
 *                                        NULL = identity, physical = s*max_pages + lp
 *    n_ctx        [S]                    prefix length of each sequence (tokens)
 *    topk         [S]                    page budget of each sequence in TOKENS,
 *                                        a multiple of `page`
 *    idx          [S, Hkv, kmax]         selected LOGICAL pages, ascending, -1 padded
 *    idx_cnt      [S, Hkv]               number of valid entries of each idx row
 *    blk_k, blk_v [S, B, Hkv, d]         the block's own keys / values
 *    o_out        [S, B, Hq, d]          attention output (bf16)
 *  Query head j uses KV head j / (Hq/Hkv) (contiguous GQA groups).  The softmax
 *  scale is 1/sqrt(d).  A prefix token t of sequence s lives in logical page
 *  t / page, slot t % page; tokens t >= n_ctx[s] of the last page are ignored.
 *
 *  Alignment: q_blk, k_cache, v_cache, blk_k, blk_v and o_out must be 16-byte
 *  aligned.  Supported shapes: d in {64, 128}; page in {16, 32, 64};
 *  Hq % Hkv == 0; B * Hq/Hkv <= 256; kmax >= 1 (it may exceed the pages of a
 *  prefix: the extra entries are -1).
 *
 *  Return values: 0 on success, or a negative DSA_ERR_* code.  Argument errors
 *  are detected on the host before anything is launched.  All work is queued
 *  asynchronously on `stream`; no call synchronises except dsa_get_status().
 *  Errors found by the kernels (a bad page index, a page-table entry outside the
 *  cache, non-finite scores, a device wait that gave up) never fault: the kernel
 *  skips the offending access, finishes, and sets a bit in the status word at
 *  the start of the workspace, which dsa_get_status() reads.
 *
 *  Workspace: each call takes a caller-owned device workspace of at least
 *  dsa_*_workspace_size() bytes.  Zero it once with dsa_workspace_init() after
 *  allocation.  Calls that may run concurrently (the selection pass on one stream
 *  and sparse steps on another) need separate workspaces.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes (negative).  The first four are returned synchronously; the last
 * three are reported through the workspace status word. */
#define DSA_OK 0
#define DSA_ERR_INVALID_ARG (-1)        /* null/misaligned pointer, bad shape or value */
#define DSA_ERR_UNSUPPORTED (-2)        /* valid but outside the supported shapes */
#define DSA_ERR_WORKSPACE_TOO_SMALL (-3)
#define DSA_ERR_CUDA (-4)               /* a CUDA launch or runtime call failed */
#define DSA_ERR_DEVICE_TIMEOUT (-5)     /* a bounded device wait gave up */
#define DSA_ERR_BAD_INDEX (-6)          /* idx entry >= number of pages, or page-table entry outside the cache */
#define DSA_ERR_NONFINITE (-7)          /* a page score was NaN or Inf (non-finite inputs) */
#define DSA_ERR_SCRATCH_LIMIT (-8)      /* shape needs more than DSA_SELECT_STATIC_SCRATCH_BYTES (dsa_select_static_scratch only) */

/* Size of the library-held scratch array used by dsa_select_static_scratch. */
#define DSA_SELECT_STATIC_SCRATCH_BYTES ((size_t)16 << 20)

typedef struct dsa_dims {
  int32_t S;          /* sequences in the batch */
  int32_t B;          /* query tokens per block */
  int32_t Hq;         /* query heads */
  int32_t Hkv;        /* KV heads; Hq % Hkv == 0 */
  int32_t d;          /* head dimension (64 or 128) */
  int32_t page;       /* tokens per KV page (16, 32 or 64) */
  int32_t max_pages;  /* length of a page-table row: logical pages per sequence, upper bound */
  int32_t kmax;       /* length of an idx row: selected pages per (sequence, KV head), upper bound */
  int64_t n_phys;     /* physical pages held by k_cache / v_cache */
  const int32_t *page_table; /* device [S, max_pages] or NULL (identity) */
  int32_t sm_limit;   /* selection pass: the most SMs its attention kernel may hold at once,
                         so that it can run on its own stream beside the sparse steps
                         (which then keep the other SMs); 0 = every SM of the device.
                         When a (sequence, KV head)'s CTAs number at most 16 (the split
                         count follows from the SMs), they are launched as one thread-block
                         cluster and the pass shares the device with other streams;
                         otherwise the pass is one cooperative launch that holds the device.
                         Workspace sizes depend on it: query them with the same dims. */
  float *lse_out;     /* optional device fp32 [S, B, Hq], NULL = not written: the call that
                         receives these dims stores, per query row, the natural log of the sum
                         of exp(q.k / sqrt(d)) over the keys it attends to (-inf for none),
                         so that two attention results can be merged (dsa_merge_attn). */
  int32_t head_budget; /* selection pass: 0 = kp = topk[s]/page pages per KV head (MAGE);
                         1 = one budget of Hkv*kp pages per sequence shared by its KV heads
                         (head-adaptive budget, Step-dLLM page, abstract): all (KV head, page)
                         pairs of the sequence are ranked by page score, ties going to the
                         lower head, then the lower page, so a head whose attention is
                         concentrated keeps fewer pages; a head may keep none.  idx_out then
                         holds a different count per head (cnt_out); kmax must hold every
                         head's count (min(max_pages, Hkv*kp) always does), else the call
                         reports DSA_ERR_BAD_INDEX and keeps that head's first kmax pages. */
  const uint8_t *active; /* sparse pass: optional device [S, B], NULL = every token active.
                         Reuse of the prefix part for stable tokens (LoSA page, abstract): a
                         row (b, query head) splits its attention into the prefix part (the
                         selected pages) and the block part (the block's B tokens).  For
                         active[s,b] != 0 the prefix part is computed and written to the two
                         caches below; for a stable token (0) it is read from them.  The block
                         part is always computed and the row's output is the log-sum-exp
                         merge of the two parts.  A (sequence, KV head, 128-row tile) whose
                         tokens are all stable loads no page at all. */
  void *prefix_o_cache;  /* with active: device bf16 [S, B, Hq, d], 16-byte aligned: each row's
                         normalised prefix part (softmax over the selected pages times V) */
  float *prefix_lse_cache; /* with active: device fp32 [S, B, Hq]: its log-sum-exp, natural log
                         (-inf: no prefix key).  A stable row reads whatever its cache holds:
                         fill the caches with a call whose tokens are all active first. */
  int32_t early_gather; /* sparse pass: 0 = read nothing the caller passes before the kernel
                         launched just before this one on `stream` has completed; 1 = gather
                         the selected pages early.  Every dsa_sparse_attn kernel is a
                         programmatic dependent launch, so its CTAs can start while that
                         preceding kernel still runs.  With early_gather = 1 they read n_ctx,
                         idx_cnt, idx, the page table, k_cache and v_cache in that time and
                         load the selected pages into shared memory; only q_blk, blk_k,
                         blk_v (and o_out, lse_out, the workspace) wait for the preceding
                         kernel.  CONTRACT: the kernel launched immediately before the call on
                         the same stream writes none of n_ctx, idx_cnt, idx, page_table,
                         k_cache, v_cache.  That holds when the page set is reused over a
                         block's denoising steps (MAGE page, Approach) and the prefix cache
                         is not appended to by that kernel: the indices come from a selection
                         pass that ended before (on another stream, joined by an event, which
                         orders it fully).  Work that is not a kernel (a copy, an event wait)
                         is always fully ordered.  Ignored (treated as 0) with `active`. */
} dsa_dims;

/* cudaStream_t without including the CUDA headers. */
typedef struct CUstream_st *dsa_stream_t;

/*
 * Selection pass (MAGE page, Approach): exact attention of the block's step-1
 * queries over the whole prefix of every sequence.
 *   - o_out receives, for each query row, softmax(q K^T / sqrt(d)) V over the
 *     prefix tokens only (the block's own tokens are not part of this pass).
 *   - For each (sequence, KV head) the attention probabilities are averaged over
 *     the B queries and the G = Hq/Hkv query heads of the group, summed inside
 *     each page, and the kp = topk[s]/page pages with the largest sums are kept;
 *     on equal sums the lower page index wins.  idx_out receives them in
 *     ascending order, padded with -1; cnt_out receives min(kp, pages of the
 *     prefix).  Requires topk[s]/page <= kmax.  With dims->head_budget = 1 the
 *     kp-per-head cut is replaced by the head-adaptive budget (see dsa_dims).
 * Arguments: q_blk, k_cache, v_cache (bf16, layouts above); n_ctx (device int32
 * [S]); page (must equal dims->page); topk (DEVICE int32 [S], tokens); idx_out
 * (device int32 [S,Hkv,kmax]); o_out (device bf16 [S,B,Hq,d]); stream; dims;
 * cnt_out (device int32 [S,Hkv]); workspace/ws_bytes (device, see above).
 * Launches: dsa_select_launches(dims) kernels in all: the selection kernel once
 * per batch of (sequence, KV head) groups whose CTAs are all resident at once
 * (one batch when S * Hkv * ceil(B * Hq/Hkv / 128) does not exceed the SMs it may
 * use), each group a thread-block cluster when it has at most 16 CTAs, else the
 * batch one cooperative launch; with head_budget = 1, one more kernel for the
 * shared budget.  The CTAs of a (sequence, KV head) wait for one another at one
 * point, with a bounded wait (DSA_ERR_DEVICE_TIMEOUT if it gives up).
 */
int dsa_select(const void *q_blk, const void *k_cache, const void *v_cache,
               const int32_t *n_ctx, int32_t page, const int32_t *topk,
               int32_t *idx_out, void *o_out, dsa_stream_t stream,
               const dsa_dims *dims, int32_t *cnt_out,
               void *workspace, size_t ws_bytes);

/*
 * Sparse pass, denoising steps 2..T (MAGE page, Approach: the step-1 indices are
 * reused for every later step).  For each query row (b, j) of sequence s:
 * softmax attention, scale 1/sqrt(d), over the key set
 *   { prefix tokens t < n_ctx[s] of the pages idx[s, j/G, 0 .. idx_cnt-1] }
 *   U { the block's own tokens u = 0..B-1 with keys blk_k[s,u,j/G], values blk_v[s,u,j/G] }
 * with no mask inside the block (bidirectional, self included).  idx entries
 * must be distinct logical pages below ceil(n_ctx[s]/page); an entry outside
 * that range is skipped and reported as DSA_ERR_BAD_INDEX through the status word.
 * Launches: one kernel, a programmatic dependent of the kernel ahead of it on
 * `stream` (see dims->early_gather).  Thread-block clusters split each (sequence,
 * KV head)'s keys; dsa_sparse_kernel() tells which of the two kernels runs.
 */
int dsa_sparse_attn(const void *q_blk, const void *k_cache, const void *v_cache,
                    const int32_t *idx, const void *blk_k, const void *blk_v,
                    void *o_out, dsa_stream_t stream,
                    const dsa_dims *dims, const int32_t *n_ctx, const int32_t *idx_cnt,
                    void *workspace, size_t ws_bytes);

/* Workspace bytes each pass needs for `dims` on the current CUDA device
 * (0 if dims is invalid). */
size_t dsa_select_workspace_size(const dsa_dims *dims);
size_t dsa_sparse_workspace_size(const dsa_dims *dims);

/* Zeroes the status word and counters of a freshly allocated workspace
 * (asynchronous on `stream`). */
int dsa_workspace_init(void *workspace, size_t ws_bytes, dsa_stream_t stream);

/* Synchronises `stream`, reads the workspace status word and returns DSA_OK or
 * the most severe device-side code recorded since dsa_workspace_init(); the word
 * is left as it is (sticky).  Returns DSA_ERR_CUDA if the read fails.  After a
 * DSA_ERR_DEVICE_TIMEOUT, bits 16..31 of the word (read it directly) identify the
 * first wait that gave up: bits 16..23 its barrier's shared-memory address / 8
 * (mod 256), or 255 for the selection pass's wait on the other CTAs of its
 * (sequence, KV head); bits 24..31 the waiting warp.  The word is sticky: clear
 * it with dsa_workspace_init() (for dsa_select_static_scratch, write 0 to the
 * caller's status word).  Nothing else needs resetting after a wait ran out: the
 * selection pass's group counters return to zero at the end of every call, since
 * every CTA still reaches it. */
int dsa_get_status(const void *workspace, dsa_stream_t stream);

/*
 * Selection pass without a workspace.  The MAGE page has no counterpart of this
 * entry point: it serves deployment, not the method.
 *
 * Who needs it: a caller that is handed only its inputs and outputs and may not
 * allocate device memory at this point (for instance a plugin of an inference
 * runtime whose host hands it no workspace, or a path that runs while the
 * process's memory pool is fully reserved) cannot supply the workspace
 * dsa_select needs.  This variant launches the same kernel as dsa_select
 * with its scratch placed in a fixed device array that the library itself
 * holds: a file-scope __device__ array of DSA_SELECT_STATIC_SCRATCH_BYTES
 * (16 MiB) per device, set aside when the CUDA module is loaded, not by an
 * allocation call.  The call allocates nothing.
 *
 * Limit: the shape's dsa_select_workspace_size() must not exceed
 * DSA_SELECT_STATIC_SCRATCH_BYTES; a larger shape returns DSA_ERR_SCRATCH_LIMIT
 * before anything is launched (use dsa_select with a caller workspace).  On a
 * 148-SM B200 this admits an 8K prefix with 8 KV heads, 32 query tokens,
 * d = 128, page 16 (10.7 MiB) and a 32K prefix with 4 KV heads, page 64
 * (13.3 MiB), not a 128K prefix with 8 KV heads (49.5 MiB).
 *
 * Arguments: those of dsa_select without workspace/ws_bytes, plus
 *   status: device uint32, caller-owned, 4-byte aligned, receiving the device
 *   status bits.  It must hold 0 before the first call; the kernels only OR bits
 *   into it (sticky, like the workspace status word).  dsa_get_status(status,
 *   stream) reads it (it only reads the first word of what it is given); writing
 *   0 clears it.
 * The scratch array needs no zeroing: every word of it a call reads was written
 * earlier in the same call, except the counters of the selection pass's group
 * wait in its first 4 KiB, which are zero when the module is loaded and which
 * every call leaves at zero.
 *
 * Concurrency: the scratch array is one per device, shared by every call on that
 * device.  Calls on one device must not overlap in time: issue them on one
 * stream or order them with events.  Two calls in flight together on different
 * streams of one device race on the scratch and return wrong results without
 * any error.  Calls on different devices are independent.
 *
 * First call on a device: the array's address is looked up
 * (cudaGetSymbolAddress, with that device current) and cached per device.  The
 * lookup may load the library's CUDA module, so make the first call on each
 * device outside stream capture.
 */
int dsa_select_static_scratch(const void *q_blk, const void *k_cache, const void *v_cache,
                              const int32_t *n_ctx, int32_t page, const int32_t *topk,
                              int32_t *idx_out, void *o_out, dsa_stream_t stream,
                              const dsa_dims *dims, int32_t *cnt_out, uint32_t *status);

/*
 * Merge of two softmax-attention results over disjoint key sets into the result
 * over their union.  Not a step of the MAGE page's method: it gives the exact
 * step-1 output (prefix and block), from the selection pass's prefix-only
 * output and the sparse pass run with idx_cnt = 0 (the block alone), both with
 * dims.lse_out set.  For each of `rows` rows:
 *   lse = log(exp(lse_a) + exp(lse_b)),
 *   o_out = exp(lse_a - lse) * o_a + exp(lse_b - lse) * o_b,
 * with o_out = 0 and lse = -inf where both are -inf.  o_a, o_b, o_out: device bf16
 * [rows, d], 16-byte aligned; lse_a, lse_b: device fp32 [rows]; lse_out: device fp32
 * [rows] or NULL; d a positive multiple of 8.  o_out may alias o_a or o_b.  One
 * kernel launch on `stream`; returns DSA_OK or DSA_ERR_INVALID_ARG / DSA_ERR_CUDA.
 */
int dsa_merge_attn(const void *o_a, const float *lse_a, const void *o_b, const float *lse_b,
                   void *o_out, float *lse_out, int64_t rows, int32_t d, dsa_stream_t stream);

/* Static description of a status code. */
const char *dsa_strerror(int code);

/* Number of kernel launches one call issues on its stream: pass 0 = dsa_select
 * when its groups fit in one launch (dsa_select_launches() gives the count for
 * a shape), pass 1 = dsa_sparse_attn, pass 2 = dsa_merge_attn
 * (DSA_ERR_INVALID_ARG otherwise).  Useful when capturing calls into a CUDA
 * graph or counting launches. */
int dsa_kernels_per_call(int pass);

/* Which kernel dsa_sparse_attn runs for these dims on the current device:
 *   1      the streaming kernel (a ring of 64-key tiles per CTA; prefix-part
 *          reuse, or more selected pages than 16 CTAs of a cluster can hold);
 *   1 + C  the kernel whose CTAs hold all their keys in shared memory at once
 *          (at most 256 each), in thread-block clusters of C CTAs per
 *          (sequence, KV head, row tile);
 * or a negative DSA_ERR_* code for bad dims.  Both compute the same result. */
int dsa_sparse_kernel(const dsa_dims *dims);

/* Kernel launches of one dsa_select (or dsa_select_static_scratch) call with
 * these dims on the current device, or a negative DSA_ERR_* code for bad dims. */
int dsa_select_launches(const dsa_dims *dims);

/* Library version, major*10000 + minor*100 + patch. */
int dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
