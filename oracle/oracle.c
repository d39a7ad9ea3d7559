/*
 * oracle.c -- plain fp64 CPU reference for shared-index top-k sparse KV attention
 * in block-diffusion LLMs.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the tests, the smoke check and the bench's CPU-baseline leg do.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (sources are the web pages this library follows):
 *
 *  - Selection pass ("MAGE: All-[MASK] Block Already Knows Where to Look in Block
 *    Diffusion LLM", Approach): one exact attention pass of the block's step-1
 *    queries over the whole KV prefix.  The per-token probabilities are averaged
 *    over the block's B queries and over the G query heads that share one KV head
 *    (the "block-average query" of the Approach section; the one shared per-block
 *    KV subset of the Problem section), summed inside each page, and the top-k
 *    pages per KV head are kept.  Ties go to the lower page index.
 *  - Sparse pass (same page, summary and Approach: the step-1 indices are reused
 *    for all later denoising steps): every query of the block attends to the
 *    tokens of the selected pages plus the block's own B tokens, with no mask
 *    inside the block (bidirectional, self included).
 *
 * Readings taken where the pages are silent (each one is restated in the design
 * notes of the repository):
 *   - the selection softmax runs over the prefix only, and the selection pass
 *     returns that prefix-only output;
 *   - a page score is the SUM of the averaged token probabilities in the page;
 *     tokens t >= n_ctx of a partial last page do not exist;
 *   - query head j belongs to KV head j / G (contiguous GQA groups);
 *   - scale c = 1/sqrt(d); inputs are taken after RoPE;
 *   - the selected pages are returned in ascending page order, padded with -1.
 *
 * Arithmetic: every bf16 input is widened exactly to double; all sums, exps and
 * products run in double (libm exp/log).  The loop order is the definition's
 * order: no blocking, no online softmax, no split.
 *
 * Layouts (all row-major, element counts):
 *   q        [S, B, Hq, d]            bf16 bits (uint16)
 *   k, v     [n_phys, Hkv, P, d]      bf16 bits, paged cache
 *   page_table [S, max_pages]         int32, logical page -> physical page;
 *                                     NULL means physical = s*max_pages + logical
 *   n_ctx    [S]                      prefix length of each sequence
 *   topk     [S]                      budget in TOKENS, a multiple of P
 *   idx      [S, Hkv, kmax]           int32 selected logical pages, -1 padded
 *   cnt      [S, Hkv]                 number of valid entries in idx
 *   blk_k, blk_v [S, B, Hkv, d]       the block's own keys / values (bf16 bits)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_EPAGE (-2)
#define ORACLE_EINDEX (-3)
#define ORACLE_ENOMEM (-4)

static double widen_bf16(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Physical page of logical page `lp` of sequence `s`; -1 if out of range. */
static long phys_page(const int32_t *page_table, int s, int lp, int max_pages, long n_phys) {
  long p = page_table ? (long)page_table[(size_t)s * max_pages + lp]
                      : (long)s * max_pages + lp;
  if (p < 0 || p >= n_phys) return -1;
  return p;
}

static const uint16_t *cache_row(const uint16_t *cache, long phys, int h, int slot,
                                 int Hkv, int P, int d) {
  return cache + (((size_t)phys * Hkv + h) * P + slot) * (size_t)d;
}

static int check_dims(int S, int B, int Hq, int Hkv, int d, int P, int max_pages) {
  if (S <= 0 || B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || P <= 0 || max_pages <= 0)
    return ORACLE_EINVAL;
  if (Hq % Hkv != 0) return ORACLE_EINVAL;
  return ORACLE_OK;
}

struct score_item {
  double score;
  int page;
};

/* Order for top-k: larger score first; on equal score the lower page wins. */
static int by_score_then_page(const void *pa, const void *pb) {
  const struct score_item *a = (const struct score_item *)pa;
  const struct score_item *b = (const struct score_item *)pb;
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  return (a->page > b->page) - (a->page < b->page);
}

static int by_int(const void *pa, const void *pb) {
  int a = *(const int *)pa, b = *(const int *)pb;
  return (a > b) - (a < b);
}

/*
 * Selection pass.  Outputs:
 *   idx_out [S,Hkv,kmax], cnt_out [S,Hkv]        the top-k page set per KV head
 *   o_out   [S,B,Hq,d] (double)                   prefix-only attention output
 *   lse_out [S,B,Hq] (double, may be NULL)        log(sum_t exp(s_t)) of each row
 *   score_out [S,Hkv,max_pages] (double, may be NULL)   page scores (0 beyond NP)
 *   mass_out [S,Hkv,max_pages*P] (double, may be NULL)  averaged token probabilities
 */
int oracle_select(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                  const int32_t *page_table, const int32_t *n_ctx, const int32_t *topk,
                  int S, int B, int Hq, int Hkv, int d, int P, int max_pages, long n_phys,
                  int kmax, int32_t *idx_out, int32_t *cnt_out, double *o_out,
                  double *lse_out, double *score_out, double *mass_out) {
  if (check_dims(S, B, Hq, Hkv, d, P, max_pages) != ORACLE_OK || kmax <= 0)
    return ORACLE_EINVAL;
  for (int s = 0; s < S; ++s) {
    if (n_ctx[s] <= 0 || n_ctx[s] > max_pages * P) return ORACLE_EINVAL;
    if (topk[s] <= 0 || topk[s] % P != 0 || topk[s] / P > kmax) return ORACLE_EINVAL;
    int np = (n_ctx[s] + P - 1) / P;
    for (int lp = 0; lp < np; ++lp)
      if (phys_page(page_table, s, lp, max_pages, n_phys) < 0) return ORACLE_EPAGE;
  }
  const int G = Hq / Hkv;
  const double c = 1.0 / sqrt((double)d);
  int status = ORACLE_OK;

#pragma omp parallel for schedule(dynamic, 1)
  for (int sh = 0; sh < S * Hkv; ++sh) {
    const int s = sh / Hkv, h = sh % Hkv;
    const int n = n_ctx[s];
    const int np = (n + P - 1) / P;
    double *logit = (double *)malloc(sizeof(double) * (size_t)n);
    double *mass = (double *)calloc((size_t)n, sizeof(double));
    double *qd = (double *)malloc(sizeof(double) * (size_t)d);
    double *od = (double *)malloc(sizeof(double) * (size_t)d);
    struct score_item *items = (struct score_item *)malloc(sizeof(struct score_item) * (size_t)np);
    int *chosen = (int *)malloc(sizeof(int) * (size_t)np);
    if (!logit || !mass || !qd || !od || !items || !chosen) {
#pragma omp atomic write
      status = ORACLE_ENOMEM;
      free(logit); free(mass); free(qd); free(od); free(items); free(chosen);
      continue;
    }
    for (int b = 0; b < B; ++b) {
      for (int g = 0; g < G; ++g) {
        const int j = h * G + g; /* contiguous GQA groups */
        const size_t qoff = (((size_t)s * B + b) * Hq + j) * (size_t)d;
        for (int i = 0; i < d; ++i) qd[i] = widen_bf16(q[qoff + i]);
        /* logits over the prefix only */
        double mx = -INFINITY;
        for (int t = 0; t < n; ++t) {
          long pp = phys_page(page_table, s, t / P, max_pages, n_phys);
          const uint16_t *kr = cache_row(k, pp, h, t % P, Hkv, P, d);
          double dot = 0.0;
          for (int i = 0; i < d; ++i) dot += qd[i] * widen_bf16(kr[i]);
          logit[t] = c * dot;
          if (logit[t] > mx) mx = logit[t];
        }
        double sum = 0.0;
        for (int t = 0; t < n; ++t) sum += exp(logit[t] - mx);
        for (int i = 0; i < d; ++i) od[i] = 0.0;
        for (int t = 0; t < n; ++t) {
          const double p = exp(logit[t] - mx) / sum;
          long pp = phys_page(page_table, s, t / P, max_pages, n_phys);
          const uint16_t *vr = cache_row(v, pp, h, t % P, Hkv, P, d);
          for (int i = 0; i < d; ++i) od[i] += p * widen_bf16(vr[i]);
          /* block-and-group average of the token probabilities */
          mass[t] += p / (double)(B * G);
        }
        for (int i = 0; i < d; ++i) o_out[qoff + i] = od[i];
        if (lse_out) lse_out[((size_t)s * B + b) * Hq + j] = mx + log(sum);
      }
    }
    /* page score = sum of the averaged probabilities of the page's valid tokens */
    for (int lp = 0; lp < np; ++lp) {
      double sc = 0.0;
      for (int t = lp * P; t < (lp + 1) * P && t < n; ++t) sc += mass[t];
      items[lp].score = sc;
      items[lp].page = lp;
    }
    if (score_out) {
      double *row = score_out + (size_t)sh * max_pages;
      for (int lp = 0; lp < max_pages; ++lp) row[lp] = lp < np ? items[lp].score : 0.0;
    }
    if (mass_out) {
      double *row = mass_out + (size_t)sh * max_pages * P;
      for (int t = 0; t < max_pages * P; ++t) row[t] = t < n ? mass[t] : 0.0;
    }
    /* top-k: highest score first, lower page index on ties; emit ascending */
    const int kp = topk[s] / P;
    const int take = kp < np ? kp : np;
    qsort(items, (size_t)np, sizeof(struct score_item), by_score_then_page);
    for (int r = 0; r < take; ++r) chosen[r] = items[r].page;
    qsort(chosen, (size_t)take, sizeof(int), by_int);
    int32_t *dst = idx_out + (size_t)sh * kmax;
    for (int r = 0; r < kmax; ++r) dst[r] = r < take ? chosen[r] : -1;
    cnt_out[sh] = take;
    free(logit); free(mass); free(qd); free(od); free(items); free(chosen);
  }
  return status;
}

/*
 * Head-adaptive budget ("Step-dLLM: Adaptive Step-aware Sparse Attention for
 * Efficient Diffusion LLM Inference", abstract: one global budget shared by the
 * heads, so that heads whose attention is concentrated are compressed more).
 * Reading: sequence s has one budget of Hkv * kp pages, kp = topk[s]/P being the
 * per-head budget of the MAGE selection.  All (KV head, page) pairs of the
 * sequence are ranked by their page score (each head's scores sum to one over its
 * pages, so scores of different heads compare) and the best Hkv * kp pairs are
 * kept; on equal scores the lower head wins, then the lower page.  A head may
 * keep any number of pages, none included.
 *   score    [S,Hkv,max_pages]   page scores (those of oracle_select)
 *   idx_out  [S,Hkv,kmax]        each head's kept pages, ascending, -1 padded
 *   cnt_out  [S,Hkv]             each head's count
 * Returns ORACLE_EINVAL if a head keeps more than kmax pages.
 */
int oracle_select_global(const double *score, const int32_t *n_ctx, const int32_t *topk, int S,
                         int Hkv, int P, int max_pages, int kmax, int32_t *idx_out,
                         int32_t *cnt_out) {
  if (S <= 0 || Hkv <= 0 || P <= 0 || max_pages <= 0 || kmax <= 0) return ORACLE_EINVAL;
  for (int s = 0; s < S; ++s) {
    if (n_ctx[s] <= 0 || n_ctx[s] > max_pages * P) return ORACLE_EINVAL;
    if (topk[s] <= 0 || topk[s] % P != 0) return ORACLE_EINVAL;
  }
  int status = ORACLE_OK;
  for (int s = 0; s < S; ++s) {
    const int np = (n_ctx[s] + P - 1) / P;
    const int total = Hkv * np;
    const long budget = (long)Hkv * (topk[s] / P);
    const int take = budget < total ? (int)budget : total;
    /* a pair (h, page) is item h * np + page: the lower item wins a tie */
    struct score_item *items = (struct score_item *)malloc(sizeof(struct score_item) * (size_t)total);
    int *chosen = (int *)malloc(sizeof(int) * (size_t)total);
    if (!items || !chosen) {
      free(items); free(chosen);
      return ORACLE_ENOMEM;
    }
    for (int h = 0; h < Hkv; ++h)
      for (int lp = 0; lp < np; ++lp) {
        items[h * np + lp].score = score[((size_t)s * Hkv + h) * max_pages + lp];
        items[h * np + lp].page = h * np + lp;
      }
    qsort(items, (size_t)total, sizeof(struct score_item), by_score_then_page);
    for (int r = 0; r < take; ++r) chosen[r] = items[r].page;
    qsort(chosen, (size_t)take, sizeof(int), by_int); /* head-major, pages ascending */
    int r = 0;
    for (int h = 0; h < Hkv; ++h) {
      int32_t *dst = idx_out + ((size_t)s * Hkv + h) * kmax;
      int c = 0;
      while (r < take && chosen[r] / np == h) {
        if (c < kmax) dst[c] = chosen[r] % np;
        ++c;
        ++r;
      }
      if (c > kmax) status = ORACLE_EINVAL;
      for (int j = c; j < kmax; ++j) dst[j] = -1;
      cnt_out[(size_t)s * Hkv + h] = c < kmax ? c : kmax;
    }
    free(items); free(chosen);
  }
  return status;
}

/*
 * Sparse pass.  For each query row (b, j) of the block: softmax attention over
 * the valid tokens of the selected pages of KV head j/G plus the block's own B
 * tokens (keys blk_k[s,u,h], values blk_v[s,u,h], u = 0..B-1, no mask).
 *   o_out   [S,B,Hq,d] (double)
 *   lse_out [S,B,Hq]   (double, may be NULL)
 * The first cnt[s,h] entries of idx[s,h,:] are used; they must be distinct
 * logical pages in [0, NP).  Returns ORACLE_EINDEX otherwise.
 */
int oracle_sparse(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                  const int32_t *page_table, const int32_t *n_ctx, const int32_t *idx,
                  const int32_t *cnt, int kmax, const uint16_t *blk_k, const uint16_t *blk_v,
                  int S, int B, int Hq, int Hkv, int d, int P, int max_pages, long n_phys,
                  double *o_out, double *lse_out) {
  if (check_dims(S, B, Hq, Hkv, d, P, max_pages) != ORACLE_OK || kmax <= 0)
    return ORACLE_EINVAL;
  for (int s = 0; s < S; ++s) {
    if (n_ctx[s] <= 0 || n_ctx[s] > max_pages * P) return ORACLE_EINVAL;
    const int np = (n_ctx[s] + P - 1) / P;
    for (int h = 0; h < Hkv; ++h) {
      const int32_t *row = idx + ((size_t)s * Hkv + h) * kmax;
      const int c0 = cnt[(size_t)s * Hkv + h];
      if (c0 < 0 || c0 > kmax) return ORACLE_EINDEX;
      for (int r = 0; r < c0; ++r) {
        if (row[r] < 0 || row[r] >= np) return ORACLE_EINDEX;
        for (int r2 = 0; r2 < r; ++r2)
          if (row[r2] == row[r]) return ORACLE_EINDEX;
        if (phys_page(page_table, s, row[r], max_pages, n_phys) < 0) return ORACLE_EPAGE;
      }
    }
  }
  const int G = Hq / Hkv;
  const double c = 1.0 / sqrt((double)d);
  int status = ORACLE_OK;

#pragma omp parallel for schedule(dynamic, 1)
  for (int sh = 0; sh < S * Hkv; ++sh) {
    const int s = sh / Hkv, h = sh % Hkv;
    const int n = n_ctx[s];
    const int32_t *sel = idx + (size_t)sh * kmax;
    const int nsel = cnt[sh];
    /* gather the key set: valid tokens of the selected pages, then the block */
    const int nkeys_max = nsel * P + B;
    const uint16_t **krow = (const uint16_t **)malloc(sizeof(void *) * (size_t)nkeys_max);
    const uint16_t **vrow = (const uint16_t **)malloc(sizeof(void *) * (size_t)nkeys_max);
    double *logit = (double *)malloc(sizeof(double) * (size_t)nkeys_max);
    double *qd = (double *)malloc(sizeof(double) * (size_t)d);
    double *od = (double *)malloc(sizeof(double) * (size_t)d);
    if (!krow || !vrow || !logit || !qd || !od) {
#pragma omp atomic write
      status = ORACLE_ENOMEM;
      free(krow); free(vrow); free(logit); free(qd); free(od);
      continue;
    }
    int nk = 0;
    for (int r = 0; r < nsel; ++r) {
      const int lp = sel[r];
      const long pp = phys_page(page_table, s, lp, max_pages, n_phys);
      for (int slot = 0; slot < P && lp * P + slot < n; ++slot) {
        krow[nk] = cache_row(k, pp, h, slot, Hkv, P, d);
        vrow[nk] = cache_row(v, pp, h, slot, Hkv, P, d);
        ++nk;
      }
    }
    for (int u = 0; u < B; ++u) {
      const size_t off = (((size_t)s * B + u) * Hkv + h) * (size_t)d;
      krow[nk] = blk_k + off;
      vrow[nk] = blk_v + off;
      ++nk;
    }
    for (int b = 0; b < B; ++b) {
      for (int g = 0; g < G; ++g) {
        const int j = h * G + g;
        const size_t qoff = (((size_t)s * B + b) * Hq + j) * (size_t)d;
        for (int i = 0; i < d; ++i) qd[i] = widen_bf16(q[qoff + i]);
        double mx = -INFINITY;
        for (int t = 0; t < nk; ++t) {
          double dot = 0.0;
          for (int i = 0; i < d; ++i) dot += qd[i] * widen_bf16(krow[t][i]);
          logit[t] = c * dot;
          if (logit[t] > mx) mx = logit[t];
        }
        double sum = 0.0;
        for (int t = 0; t < nk; ++t) sum += exp(logit[t] - mx);
        for (int i = 0; i < d; ++i) od[i] = 0.0;
        for (int t = 0; t < nk; ++t) {
          const double p = exp(logit[t] - mx) / sum;
          for (int i = 0; i < d; ++i) od[i] += p * widen_bf16(vrow[t][i]);
        }
        for (int i = 0; i < d; ++i) o_out[qoff + i] = od[i];
        if (lse_out) lse_out[((size_t)s * B + b) * Hq + j] = mx + log(sum);
      }
    }
    free(krow); free(vrow); free(logit); free(qd); free(od);
  }
  return status;
}

/*
 * Sparse pass with reuse of the prefix part for stable tokens ("LoSA: Locality
 * Aware Sparse Attention for Block-Wise Diffusion Language Models", abstract:
 * cached prefix-attention results are reused for stable tokens and sparse
 * attention is run only for active tokens).  Reading: a query row (b, j) splits
 * its attention into the prefix part (the valid tokens of the selected pages)
 * and the block part (the block's own B tokens), each a normalised output with
 * its log-sum-exp.  For an active token (active[s,b] != 0) the prefix part is
 * computed and written to cache_o_out / cache_lse_out; for a stable token it is
 * taken from cache_o_in (bf16 bits) / cache_lse_in and passed through.  The block
 * part is always computed.  The row's output merges the two:
 *   lse = log(exp(lse_p) + exp(lse_b)),  o = exp(lse_p - lse) o_p + exp(lse_b - lse) o_b,
 * an empty part having lse = -inf and o = 0.
 *   active [S,B] uint8; cache_o_in [S,B,Hq,d] bf16 bits; cache_lse_in [S,B,Hq] double
 *   o_out, cache_o_out [S,B,Hq,d] double; lse_out, cache_lse_out [S,B,Hq] double
 */
int oracle_sparse_losa(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       const int32_t *page_table, const int32_t *n_ctx, const int32_t *idx,
                       const int32_t *cnt, int kmax, const uint16_t *blk_k, const uint16_t *blk_v,
                       const uint8_t *active, const uint16_t *cache_o_in, const double *cache_lse_in,
                       int S, int B, int Hq, int Hkv, int d, int P, int max_pages, long n_phys,
                       double *o_out, double *lse_out, double *cache_o_out, double *cache_lse_out) {
  if (check_dims(S, B, Hq, Hkv, d, P, max_pages) != ORACLE_OK || kmax <= 0)
    return ORACLE_EINVAL;
  for (int s = 0; s < S; ++s) {
    if (n_ctx[s] <= 0 || n_ctx[s] > max_pages * P) return ORACLE_EINVAL;
    const int np = (n_ctx[s] + P - 1) / P;
    for (int h = 0; h < Hkv; ++h) {
      const int32_t *row = idx + ((size_t)s * Hkv + h) * kmax;
      const int c0 = cnt[(size_t)s * Hkv + h];
      if (c0 < 0 || c0 > kmax) return ORACLE_EINDEX;
      for (int r = 0; r < c0; ++r) {
        if (row[r] < 0 || row[r] >= np) return ORACLE_EINDEX;
        for (int r2 = 0; r2 < r; ++r2)
          if (row[r2] == row[r]) return ORACLE_EINDEX;
        if (phys_page(page_table, s, row[r], max_pages, n_phys) < 0) return ORACLE_EPAGE;
      }
    }
  }
  const int G = Hq / Hkv;
  const double c = 1.0 / sqrt((double)d);
  int status = ORACLE_OK;

#pragma omp parallel for schedule(dynamic, 1)
  for (int sh = 0; sh < S * Hkv; ++sh) {
    const int s = sh / Hkv, h = sh % Hkv;
    const int n = n_ctx[s];
    const int32_t *sel = idx + (size_t)sh * kmax;
    const int nsel = cnt[sh];
    const int npre_max = nsel * P;
    const uint16_t **krow = (const uint16_t **)malloc(sizeof(void *) * (size_t)(npre_max + 1));
    const uint16_t **vrow = (const uint16_t **)malloc(sizeof(void *) * (size_t)(npre_max + 1));
    double *logit = (double *)malloc(sizeof(double) * (size_t)(npre_max + B + 1));
    double *qd = (double *)malloc(sizeof(double) * (size_t)d);
    double *op = (double *)malloc(sizeof(double) * (size_t)d);
    double *ob = (double *)malloc(sizeof(double) * (size_t)d);
    if (!krow || !vrow || !logit || !qd || !op || !ob) {
#pragma omp atomic write
      status = ORACLE_ENOMEM;
      free(krow); free(vrow); free(logit); free(qd); free(op); free(ob);
      continue;
    }
    /* the prefix key set: valid tokens of the selected pages */
    int npre = 0;
    for (int r = 0; r < nsel; ++r) {
      const int lp = sel[r];
      const long pp = phys_page(page_table, s, lp, max_pages, n_phys);
      for (int slot = 0; slot < P && lp * P + slot < n; ++slot) {
        krow[npre] = cache_row(k, pp, h, slot, Hkv, P, d);
        vrow[npre] = cache_row(v, pp, h, slot, Hkv, P, d);
        ++npre;
      }
    }
    for (int b = 0; b < B; ++b) {
      const int act = active[(size_t)s * B + b] != 0;
      for (int g = 0; g < G; ++g) {
        const int j = h * G + g;
        const size_t ro = ((size_t)s * B + b) * Hq + j;
        const size_t qoff = ro * (size_t)d;
        for (int i = 0; i < d; ++i) qd[i] = widen_bf16(q[qoff + i]);
        /* prefix part: computed for an active token, from the cache otherwise */
        double lse_p;
        if (act) {
          double mx = -INFINITY;
          for (int t = 0; t < npre; ++t) {
            double dot = 0.0;
            for (int i = 0; i < d; ++i) dot += qd[i] * widen_bf16(krow[t][i]);
            logit[t] = c * dot;
            if (logit[t] > mx) mx = logit[t];
          }
          for (int i = 0; i < d; ++i) op[i] = 0.0;
          if (npre > 0) {
            double sum = 0.0;
            for (int t = 0; t < npre; ++t) sum += exp(logit[t] - mx);
            for (int t = 0; t < npre; ++t) {
              const double p = exp(logit[t] - mx) / sum;
              for (int i = 0; i < d; ++i) op[i] += p * widen_bf16(vrow[t][i]);
            }
            lse_p = mx + log(sum);
          } else {
            lse_p = -INFINITY;
          }
        } else {
          for (int i = 0; i < d; ++i) op[i] = widen_bf16(cache_o_in[qoff + i]);
          lse_p = cache_lse_in[ro];
        }
        for (int i = 0; i < d; ++i) cache_o_out[qoff + i] = op[i];
        cache_lse_out[ro] = lse_p;
        /* block part: the block's own B tokens, no mask */
        double mx = -INFINITY;
        for (int u = 0; u < B; ++u) {
          const size_t off = (((size_t)s * B + u) * Hkv + h) * (size_t)d;
          double dot = 0.0;
          for (int i = 0; i < d; ++i) dot += qd[i] * widen_bf16(blk_k[off + i]);
          logit[u] = c * dot;
          if (logit[u] > mx) mx = logit[u];
        }
        double sum = 0.0;
        for (int u = 0; u < B; ++u) sum += exp(logit[u] - mx);
        for (int i = 0; i < d; ++i) ob[i] = 0.0;
        for (int u = 0; u < B; ++u) {
          const size_t off = (((size_t)s * B + u) * Hkv + h) * (size_t)d;
          const double p = exp(logit[u] - mx) / sum;
          for (int i = 0; i < d; ++i) ob[i] += p * widen_bf16(blk_v[off + i]);
        }
        const double lse_b = mx + log(sum);
        /* merge of the two parts */
        const double top = lse_p > lse_b ? lse_p : lse_b;
        const double wp = lse_p == -INFINITY ? 0.0 : exp(lse_p - top);
        const double wb = exp(lse_b - top);
        const double lse = top + log(wp + wb);
        for (int i = 0; i < d; ++i) o_out[qoff + i] = (wp * op[i] + wb * ob[i]) / (wp + wb);
        lse_out[ro] = lse;
      }
    }
    free(krow); free(vrow); free(logit); free(qd); free(op); free(ob);
  }
  return status;
}
