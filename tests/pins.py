"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Every pin takes an ``oracle.Oracle`` and raises AssertionError (or OracleError)
when the oracle disagrees with:
  * the textbook softmax-attention formula written with numpy matmuls over the
    concatenated key set (dense equivalence, merge identity, one-row case);
  * brute-force enumeration of every k-page subset on tiny inputs;
  * closed forms of a hand-built example;
  * invariants (page scores sum to one; page-table and query-order invariance);
  * planted needles whose correct pages are known by construction.
The planted-mistake test runs the same pins against deliberately altered builds
of oracle.c and requires each alteration to be caught.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
import torch

from block_sparse_attention_27_b200 import workloads as W


# ---------------------------------------------------------------- numpy helpers
def f64(bits_or_tensor) -> np.ndarray:
    """bf16 bits (uint16 array) or bf16 tensor -> float64 values, exactly."""
    if isinstance(bits_or_tensor, torch.Tensor):
        bits_or_tensor = W.bits(bits_or_tensor)
    b = np.ascontiguousarray(bits_or_tensor).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def prefix_kv(w: W.Workload, s: int, h: int):
    """K and V of the prefix of sequence s, KV head h, as [n, d] float64 (logical order)."""
    n = int(w.n_ctx[s])
    kc, vc = f64(w.k_cache), f64(w.v_cache)
    pages = [w.physical_page(s, lp) for lp in range(w.n_pages(s))]
    K = np.concatenate([kc[p, h] for p in pages], axis=0)[:n]
    V = np.concatenate([vc[p, h] for p in pages], axis=0)[:n]
    return K, V


def softmax_rows(x: np.ndarray) -> np.ndarray:
    m = x.max(axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=-1, keepdims=True)


def group_queries(q: np.ndarray, s: int, h: int, G: int) -> np.ndarray:
    """Rows (b, g) of KV head h: q[s, b, h*G + g] -> [B*G, d]."""
    return q[s, :, h * G:(h + 1) * G, :].reshape(-1, q.shape[-1])


def token_mass_np(w: W.Workload, q=None):
    """[S][Hkv] -> averaged token probabilities over the prefix (numpy formula)."""
    q = f64(w.q1 if q is None else q)
    c = 1.0 / math.sqrt(w.d)
    out = {}
    for s in range(w.S):
        for h in range(w.Hkv):
            K, _ = prefix_kv(w, s, h)
            p = softmax_rows(c * group_queries(q, s, h, w.G) @ K.T)
            out[(s, h)] = p.mean(axis=0)
    return out


def attention_np(Q: np.ndarray, K: np.ndarray, V: np.ndarray, c: float):
    """softmax(c Q K^T) V and the row log-sum-exp, in float64."""
    x = c * Q @ K.T
    m = x.max(axis=-1, keepdims=True)
    e = np.exp(x - m)
    ssum = e.sum(axis=-1, keepdims=True)
    return (e / ssum) @ V, (m + np.log(ssum))[:, 0]


def run(orc, w: W.Workload, **kw):
    return orc.select(W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                      w.topk.numpy(), page_table=None if w.page_table is None
                      else w.page_table.numpy(), max_pages=w.max_pages, **kw)


def run_sparse(orc, w: W.Workload, idx, cnt, q=None, bk=None, bv=None):
    return orc.sparse(W.bits(w.q1 if q is None else q), W.bits(w.k_cache), W.bits(w.v_cache),
                      w.n_ctx.numpy(), idx, cnt, W.bits(w.blk_k1 if bk is None else bk),
                      W.bits(w.blk_v1 if bv is None else bv),
                      page_table=None if w.page_table is None else w.page_table.numpy(),
                      max_pages=w.max_pages)


# --------------------------------------------------------------- small workloads
def small_paged(seed=1):
    """3 ragged sequences through a random page table, GQA group of 3, partial pages."""
    return W.make("batched", seed, S=3, n_lo=50, n_hi=300, B=3, Hq=6, Hkv=2, d=16,
                  topk_choices=(32, 64))


def brute_sized(seed=2, **kw):
    cfg = dict(n=200, topk=64, B=2, Hq=4, Hkv=2, d=32, needle_count=2)
    cfg.update(kw)
    return W.make("tiny", seed, **cfg)


# ------------------------------------------------------------------------- pins
def pin_score_sums(orc, w=None):
    """Page scores are non-negative and sum to one per (sequence, KV head)."""
    w = w or small_paged()
    r = run(orc, w)
    for s in range(w.S):
        np_ = w.n_pages(s)
        for h in range(w.Hkv):
            sc = r.score[s, h]
            assert np.all(sc[:np_] >= 0)
            assert np.all(sc[np_:] == 0)
            assert abs(sc[:np_].sum() - 1.0) < 1e-12, sc.sum()


def pin_dense_equivalence(orc, w=None):
    """With every page selected the sparse pass is softmax(cQK^T)V over prefix + block."""
    w = w or small_paged()
    idx, cnt = orc_all_pages(w)
    o, lse = run_sparse(orc, w, idx, cnt)
    q, bk, bv = f64(w.q1), f64(w.blk_k1), f64(w.blk_v1)
    c = 1.0 / math.sqrt(w.d)
    for s in range(w.S):
        for h in range(w.Hkv):
            K, V = prefix_kv(w, s, h)
            K = np.concatenate([K, bk[s, :, h]], axis=0)
            V = np.concatenate([V, bv[s, :, h]], axis=0)
            ref, ref_lse = attention_np(group_queries(q, s, h, w.G), K, V, c)
            got = o[s, :, h * w.G:(h + 1) * w.G].reshape(-1, w.d)
            got_lse = lse[s, :, h * w.G:(h + 1) * w.G].reshape(-1)
            assert np.max(np.abs(got - ref)) < 1e-12
            assert np.max(np.abs(got_lse - ref_lse)) < 1e-12


def orc_all_pages(w):
    nps = [w.n_pages(s) for s in range(w.S)]
    kmax = max(nps)
    idx = np.full((w.S, w.Hkv, kmax), -1, np.int32)
    cnt = np.zeros((w.S, w.Hkv), np.int32)
    for s in range(w.S):
        idx[s, :, :nps[s]] = np.arange(nps[s])
        cnt[s] = nps[s]
    return idx, cnt


def brute_force_best(mass_tokens: np.ndarray, n: int, P: int, kp: int):
    """Best kp-page subset by token mass; ties -> lexicographically smallest page list."""
    np_ = (n + P - 1) // P
    if kp >= np_:
        return list(range(np_))
    best, best_mass = None, -1.0
    for U in itertools.combinations(range(np_), kp):   # lexicographic order
        m = sum(mass_tokens[lp * P:min((lp + 1) * P, n)].sum() for lp in U)
        if m > best_mass + 1e-12:   # strictly better beyond rounding noise
            best, best_mass = list(U), m
    return best


def pin_topk_brute_force(orc, seeds=(2, 3, 4)):
    """Selection equals the best page subset found by enumerating all of them."""
    for seed in seeds:
        for kw in ({}, dict(B=1, Hq=1, Hkv=1, topk=48), dict(n=176, topk=80)):
            w = brute_sized(seed, **kw)
            r = run(orc, w)
            mass = token_mass_np(w)
            for h in range(w.Hkv):
                best = brute_force_best(mass[(0, h)], int(w.n_ctx[0]), w.P, w.kmax)
                got = r.idx[0, h, :r.cnt[0, h]].tolist()
                assert got == best, (seed, kw, h, got, best)


def pin_exact_tie_lower_index(orc):
    """Two bit-identical pages tied at the cut: the lower page index is kept."""
    w = brute_sized(5)
    a, b = 3, 9
    w.k_cache[b] = w.k_cache[a]
    w.v_cache[b] = w.v_cache[a]
    r0 = run(orc, w, kmax=w.max_pages)
    for h in range(w.Hkv):
        sc = r0.score[0, h]
        assert sc[a] == sc[b]
        above = int(np.sum(sc > sc[a]))
        topk = (above + 1) * w.P
        w2 = W.Workload(**{**w.__dict__, "topk": torch.tensor([topk], dtype=torch.int32)})
        r = run(orc, w2)
        got = set(r.idx[0, h, :r.cnt[0, h]].tolist())
        assert a in got and b not in got, (h, sorted(got))
        mass = token_mass_np(w2)
        best = brute_force_best(mass[(0, h)], int(w.n_ctx[0]), w.P, above + 1)
        assert sorted(got) == best


def pin_planted_needles(orc):
    """tiny workload: the 8 planted pages are exactly the selection, with margin."""
    w = W.make("tiny", 0)
    r = run(orc, w)
    planted = w.planted[(0, 0)]
    assert r.idx[0, 0].tolist() == planted
    sc = r.score[0, 0, :w.n_pages(0)]
    others = np.delete(sc, planted)
    assert sc[planted].min() > 1.5 * others.max()


def pin_needles_selected(orc, name="8k"):
    """Needle pages are inside the selected set of every KV head."""
    w = W.make(name, 0)
    r = run(orc, w)
    for (s, h), pages in w.planted.items():
        assert set(pages) <= set(r.idx[s, h, :r.cnt[s, h]].tolist()), (s, h)


def pin_merge_identity(orc, w=None):
    """Selection output is the prefix-only softmax: merging it with block-only attention
    through the log-sum-exps gives the dense output over prefix + block."""
    w = w or small_paged(7)
    sel = run(orc, w)
    idx, cnt = orc_all_pages(w)
    o_all, lse_all = run_sparse(orc, w, idx, cnt)
    q, bk, bv = f64(w.q1), f64(w.blk_k1), f64(w.blk_v1)
    c = 1.0 / math.sqrt(w.d)
    for s in range(w.S):
        for h in range(w.Hkv):
            Q = group_queries(q, s, h, w.G)
            o_b, lse_b = attention_np(Q, bk[s, :, h], bv[s, :, h], c)
            o_p = sel.o[s, :, h * w.G:(h + 1) * w.G].reshape(-1, w.d)
            lse_p = sel.lse[s, :, h * w.G:(h + 1) * w.G].reshape(-1)
            lse = np.logaddexp(lse_p, lse_b)
            merged = (np.exp(lse_p - lse)[:, None] * o_p + np.exp(lse_b - lse)[:, None] * o_b)
            got = o_all[s, :, h * w.G:(h + 1) * w.G].reshape(-1, w.d)
            assert np.max(np.abs(merged - got)) < 1e-12
            assert np.max(np.abs(lse - lse_all[s, :, h * w.G:(h + 1) * w.G].reshape(-1))) < 1e-12


def pin_selection_output_is_prefix_attention(orc, w=None):
    """o_out of the selection pass equals softmax(cQK^T)V over the prefix alone."""
    w = w or small_paged(8)
    sel = run(orc, w)
    q = f64(w.q1)
    c = 1.0 / math.sqrt(w.d)
    for s in range(w.S):
        for h in range(w.Hkv):
            K, V = prefix_kv(w, s, h)
            ref, ref_lse = attention_np(group_queries(q, s, h, w.G), K, V, c)
            got = sel.o[s, :, h * w.G:(h + 1) * w.G].reshape(-1, w.d)
            assert np.max(np.abs(got - ref)) < 1e-12


def pin_page_table_invariance(orc, w=None):
    """Moving pages through a random page table changes nothing logical."""
    w = w or W.make("tiny", 3, n=500, topk=96)
    w2 = W.with_page_table(w, seed=11)
    r1, r2 = run(orc, w), run(orc, w2)
    assert np.array_equal(r1.idx, r2.idx) and np.array_equal(r1.cnt, r2.cnt)
    assert np.max(np.abs(r1.o - r2.o)) < 1e-13
    assert np.max(np.abs(r1.score - r2.score)) < 1e-15
    o1, _ = run_sparse(orc, w, r1.idx, r1.cnt)
    o2, _ = run_sparse(orc, w2, r2.idx, r2.cnt)
    assert np.max(np.abs(o1 - o2)) < 1e-13


def pin_query_order_invariance(orc, w=None):
    """Permuting the block's queries permutes o_out and leaves the selection unchanged."""
    w = w or W.make("tiny", 4, n=700, topk=80)
    perm = torch.randperm(w.B, generator=torch.Generator().manual_seed(5))
    w2 = W.Workload(**{**w.__dict__, "q1": w.q1[:, perm].contiguous()})
    r1, r2 = run(orc, w), run(orc, w2)
    assert np.array_equal(r1.idx, r2.idx)
    assert np.max(np.abs(r1.score - r2.score)) < 1e-14
    assert np.max(np.abs(r1.o[:, perm.numpy()] - r2.o)) < 1e-13


def pin_single_row(orc):
    """B = G = 1: scores are the page sums of one softmax row; ranking by (score, page)."""
    w = W.make("tiny", 6, B=1, Hq=1, Hkv=1, n=1000, topk=160, needle_count=3)
    r = run(orc, w)
    mass = token_mass_np(w)[(0, 0)]
    n, P = 1000, w.P
    pages = np.array([mass[lp * P:min((lp + 1) * P, n)].sum() for lp in range(w.n_pages(0))])
    assert np.max(np.abs(pages - r.score[0, 0, :len(pages)])) < 1e-13
    order = np.lexsort((np.arange(len(pages)), -pages))
    assert r.idx[0, 0].tolist() == sorted(order[:10].tolist())


def pin_budget_covers_prefix(orc):
    """top-k at or above the number of pages selects every page, ascending, -1 padded."""
    w = W.make("tiny", 7, n=70, topk=128, B=2, Hq=2, Hkv=1, d=16, needle_count=1)
    r = run(orc, w)
    assert r.cnt[0, 0] == 5
    assert r.idx[0, 0].tolist() == [0, 1, 2, 3, 4, -1, -1, -1]


def pin_ascending_and_padding(orc, w=None):
    w = w or small_paged(9)
    r = run(orc, w)
    for s in range(w.S):
        kp = int(w.topk[s]) // w.P
        for h in range(w.Hkv):
            c0 = int(r.cnt[s, h])
            assert c0 == min(kp, w.n_pages(s))
            row = r.idx[s, h]
            assert np.all(np.diff(row[:c0]) > 0) and np.all(row[c0:] == -1)


def pin_worked_example(orc):
    """Closed form: q = (8, 0, ...), d = 64, so the logit of token t is its key's first
    coordinate x_t.  Page 0 has x = 0, page 1 x = 1, page 2 (8 valid tokens of 16)
    x = 2; the 8 tokens past n_ctx carry x = 100 and must be ignored.  With
    Z = 16 + 16e + 8e^2 the page scores are 16/Z, 16e/Z, 8e^2/Z, the top page is 2,
    the top two are {1, 2}, and o[0] = (0*16 + 1*16e + 2*8e^2)/Z when v_t[0] = x_t."""
    d, P, n = 64, 16, 40
    q = torch.zeros((1, 1, 1, d), dtype=torch.float32)
    q[0, 0, 0, 0] = 8.0
    k = torch.zeros((3, 1, P, d), dtype=torch.float32)
    v = torch.zeros((3, 1, P, d), dtype=torch.float32)
    k[1, 0, :, 0] = 1.0
    k[2, 0, :8, 0] = 2.0
    k[2, 0, 8:, 0] = 100.0
    v[..., 0] = k[..., 0]
    v[2, 0, 8:, 1] = 1e3
    bits = lambda t: W.bits(t.to(torch.bfloat16))
    e = math.e
    Z = 16 + 16 * e + 8 * e * e
    for topk, want in ((16, [2]), (32, [1, 2]), (48, [0, 1, 2])):
        r = orc.select(bits(q), bits(k), bits(v), np.array([n]), np.array([topk]),
                       max_pages=3)
        assert r.idx[0, 0, :r.cnt[0, 0]].tolist() == want
        assert np.allclose(r.score[0, 0], [16 / Z, 16 * e / Z, 8 * e * e / Z], rtol=1e-14)
        assert abs(r.o[0, 0, 0, 0] - (16 * e + 16 * e * e) / Z) < 1e-13
        assert abs(r.o[0, 0, 0, 1]) < 1e-15
        assert abs(r.lse[0, 0, 0] - math.log(Z)) < 1e-13


def pin_rejects_bad_indices(orc):
    from oracle import OracleError
    w = W.make("tiny", 8, n=100, topk=32, B=1, Hq=1, Hkv=1, d=16, needle_count=1)
    for bad in ([0, 7], [3, 3]):          # 7 is past the 7 pages (0..6); 3 is repeated
        idx = np.array(bad, np.int32).reshape(1, 1, 2)
        cnt = np.array([[2]], np.int32)
        try:
            run_sparse(orc, w, idx, cnt)
        except OracleError:
            continue
        raise AssertionError(f"index list {bad} was accepted")


# ------------------------------------------------- head-adaptive budget (Step-dLLM)
def run_global(orc, w: W.Workload, kmax=None):
    kmax = w.max_pages if kmax is None else kmax
    return orc.select_global(W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                             w.topk.numpy(), kmax=kmax,
                             page_table=None if w.page_table is None else w.page_table.numpy(),
                             max_pages=w.max_pages)


def brute_force_global(mass: dict, s: int, Hkv: int, n: int, P: int, budget: int):
    """Best `budget` (head, page) pairs of sequence s by page mass, by enumerating every
    subset in lexicographic (head, page) order; ties -> the first such subset."""
    np_ = (n + P - 1) // P
    items = [(h, lp) for h in range(Hkv) for lp in range(np_)]
    page_mass = {(h, lp): mass[(s, h)][lp * P:min((lp + 1) * P, n)].sum() for h, lp in items}
    if budget >= len(items):
        return items
    best, best_m = None, -1.0
    for U in itertools.combinations(items, budget):
        m = sum(page_mass[x] for x in U)
        if m > best_m + 1e-12:
            best, best_m = list(U), m
    return best


def pin_global_brute_force(orc, seeds=(2, 3)):
    """Head-adaptive selection equals the best (head, page) subset of the shared budget
    found by enumerating all of them."""
    for seed in seeds:
        for kw in (dict(n=120, topk=32, needle_count=1), dict(n=100, topk=16, Hkv=3, Hq=6, needle_count=1)):
            w = brute_sized(seed, **kw)
            r = run_global(orc, w)
            mass = token_mass_np(w)
            best = brute_force_global(mass, 0, w.Hkv, int(w.n_ctx[0]), w.P, w.Hkv * w.kmax)
            got = [(h, int(lp)) for h in range(w.Hkv) for lp in r.idx[0, h, :r.cnt[0, h]]]
            assert sorted(got) == sorted(best), (seed, kw, got, best)
            assert sum(r.cnt[0]) == w.Hkv * w.kmax


def pin_global_one_head_is_per_head(orc):
    """With one KV head the shared budget is that head's budget: the per-head selection."""
    for seed in (1, 2):
        w = brute_sized(seed, B=2, Hq=2, Hkv=1, topk=48)
        r1, r2 = run(orc, w, kmax=w.max_pages), run_global(orc, w)
        assert np.array_equal(r1.idx, r2.idx) and np.array_equal(r1.cnt, r2.cnt)


def pin_global_covers_prefix(orc):
    """A budget of at least every page of every head keeps all of them."""
    w = small_paged(3)
    w = W.Workload(**{**w.__dict__, "topk": torch.full((w.S,), w.max_pages * w.P, dtype=torch.int32)})
    r = run_global(orc, w)
    for s in range(w.S):
        for h in range(w.Hkv):
            assert r.idx[s, h, :r.cnt[s, h]].tolist() == list(range(w.n_pages(s)))


def pin_global_concentrated_head(orc):
    """A head whose attention sits on two planted pages keeps just those two; the
    diffuse head takes the rest of the shared budget (the Step-dLLM intent)."""
    w = brute_sized(7, n=208, topk=64, B=2, Hq=4, Hkv=2, needle_count=0)
    qmean = f64(w.q1)[0].reshape(w.B, w.Hkv, w.G, w.d).mean(axis=(0, 2))  # [Hkv, d]
    pages = (3, 8)
    k = w.k_cache.float()
    for lp in pages:
        k[lp, 0] += 8.0 * torch.from_numpy(qmean[0]).float()
    w.k_cache = k.to(torch.bfloat16)
    r = run_global(orc, w)
    assert r.idx[0, 0, :r.cnt[0, 0]].tolist() == list(pages), r.idx[0, 0, :r.cnt[0, 0]]
    assert r.cnt[0, 1] == w.Hkv * w.kmax - len(pages)


def pin_global_within_head_lists(orc):
    """Every (head, page) pair the shared budget keeps is among its own head's best
    min(Hkv kp, np) pages by the per-head rule: within one head both rankings order
    pages by score, then lower page.  (A two-step selection, per head first, rests on
    this.)  Ragged paged sequences, three heads, and all-equal scores (zero keys, so
    every full page ties and the tie rules alone decide)."""
    zero = brute_sized(8, n=180, topk=32, Hkv=2, Hq=4, needle_count=0)
    zero = W.Workload(**{**zero.__dict__, "k_cache": torch.zeros_like(zero.k_cache)})
    for w in (small_paged(5), brute_sized(4, Hkv=3, Hq=6, topk=16), zero):
        g = run_global(orc, w)
        cap = torch.tensor([w.n_pages(s) * w.P for s in range(w.S)], dtype=torch.int32)
        wide = W.Workload(**{**w.__dict__, "topk": torch.minimum(w.topk * w.Hkv, cap)})
        r = run(orc, wide, kmax=w.max_pages)
        for s in range(w.S):
            for h in range(w.Hkv):
                kept = set(g.idx[s, h, :g.cnt[s, h]].tolist())
                best = set(r.idx[s, h, :r.cnt[s, h]].tolist())
                assert kept <= best, (s, h, sorted(kept - best))
            assert sum(int(g.cnt[s, h]) for h in range(w.Hkv)) == min(
                w.Hkv * int(w.topk[s]) // w.P, w.Hkv * w.n_pages(s))


# ---------------------------------------------------------- LoSA prefix reuse
def run_losa(orc, w, idx, cnt, active, cache_o, cache_lse, q=None, bk=None, bv=None):
    return orc.sparse_losa(W.bits(w.q1 if q is None else q), W.bits(w.k_cache), W.bits(w.v_cache),
                           w.n_ctx.numpy(), idx, cnt, W.bits(w.blk_k1 if bk is None else bk),
                           W.bits(w.blk_v1 if bv is None else bv), active, cache_o, cache_lse,
                           page_table=None if w.page_table is None else w.page_table.numpy(),
                           max_pages=w.max_pages)


def selected_kv(w, s, h, pages):
    """K, V [n_sel, d] float64 of the valid tokens of the given logical pages."""
    n = int(w.n_ctx[s])
    kc, vc = f64(w.k_cache), f64(w.v_cache)
    Ks, Vs = [], []
    for lp in pages:
        pp = w.physical_page(s, int(lp))
        valid = min(w.P, n - int(lp) * w.P)
        Ks.append(kc[pp, h, :valid])
        Vs.append(vc[pp, h, :valid])
    return (np.concatenate(Ks, axis=0), np.concatenate(Vs, axis=0)) if Ks else (None, None)


def pin_losa(orc):
    """Reuse of the prefix part (LoSA): with a mixed active mask, an active row's prefix
    part (written to the new cache) is softmax attention over the selected pages, and
    every row's output is the log-sum-exp merge of its prefix part (fresh, or the cache's
    for a stable row) with softmax attention over the block, all written with numpy; with
    every token active the output is the plain sparse pass."""
    w = small_paged(4)
    r = run(orc, w)
    rng = np.random.default_rng(5)
    active = rng.random((w.S, w.B)) < 0.5
    active[0, 0], active[0, 1] = True, False
    cache_o = W.bits(torch.randn(w.q1.shape, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16))
    cache_lse = rng.normal(0.0, 2.0, (w.S, w.B, w.Hq))
    o, lse, co, cl = run_losa(orc, w, r.idx, r.cnt, active, cache_o, cache_lse)
    q, bk, bv, cof = f64(w.q1), f64(w.blk_k1), f64(w.blk_v1), f64(cache_o)
    c = 1.0 / math.sqrt(w.d)
    for s in range(w.S):
        for h in range(w.Hkv):
            Kp, Vp = selected_kv(w, s, h, r.idx[s, h, :r.cnt[s, h]])
            Qh = group_queries(q, s, h, w.G)                       # rows (b, g) in order
            op_f, lp_f = attention_np(Qh, Kp, Vp, c)
            ob, lb = attention_np(Qh, bk[s, :, h], bv[s, :, h], c)
            for b in range(w.B):
                for g in range(w.G):
                    row, j = b * w.G + g, h * w.G + g
                    if active[s, b]:
                        op, lp = op_f[row], lp_f[row]
                        assert np.max(np.abs(co[s, b, j] - op)) < 1e-12 and abs(cl[s, b, j] - lp) < 1e-12
                    else:
                        op, lp = cof[s, b, j], cache_lse[s, b, j]
                        assert np.array_equal(co[s, b, j], op) and cl[s, b, j] == lp
                    top = max(lp, lb[row])
                    wp, wb = math.exp(lp - top), math.exp(lb[row] - top)
                    ref = (wp * op + wb * ob[row]) / (wp + wb)
                    assert np.max(np.abs(o[s, b, j] - ref)) < 1e-12, (s, h, b, g)
                    assert abs(lse[s, b, j] - (top + math.log(wp + wb))) < 1e-12
    # every token active: the plain sparse pass
    o2, lse2, _, _ = run_losa(orc, w, r.idx, r.cnt, np.ones((w.S, w.B), bool), cache_o, cache_lse)
    ref_o, ref_lse = run_sparse(orc, w, r.idx, r.cnt)
    assert np.max(np.abs(o2 - ref_o)) < 1e-12 and np.max(np.abs(lse2 - ref_lse)) < 1e-12


FAST_PINS = [pin_score_sums, pin_dense_equivalence, pin_topk_brute_force,
             pin_exact_tie_lower_index, pin_planted_needles, pin_merge_identity,
             pin_selection_output_is_prefix_attention, pin_page_table_invariance,
             pin_query_order_invariance, pin_single_row, pin_budget_covers_prefix,
             pin_ascending_and_padding, pin_worked_example, pin_rejects_bad_indices,
             pin_global_brute_force, pin_global_one_head_is_per_head, pin_global_covers_prefix,
             pin_global_concentrated_head, pin_global_within_head_lists, pin_losa]
