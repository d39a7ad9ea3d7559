"""Comparison rules between the CUDA path and the fp64 oracle.

Index sets: bit-exact, except where the oracle's kp-th and (kp+1)-th page scores
are within 1e-5 relative of each other.  Then the window
W = {q : |S_q - s_k| <= 1e-5 * s_k} may be resolved either way: the GPU set
must hold exactly kp pages, every oracle-selected page outside W, and no
unselected page outside W.

Outputs (bf16 I/O, fp32 accumulation): max |gpu - oracle| <= 2e-2 and
mean |gpu - oracle| <= 2e-3.  The sparse pass is compared against the oracle run
with the GPU's own index sets, so a tie resolved differently cannot show up as
an output error.
"""
from __future__ import annotations

import numpy as np
import torch

TIE_REL = 1e-5
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def check_selection(gpu_idx, gpu_cnt, orc, n_pages, kp_of, rel=TIE_REL):
    """gpu_idx [S,Hkv,kmax], gpu_cnt [S,Hkv] (numpy); orc = oracle.SelectResult.

    Returns the number of (seq, head) rows that fell back to the tie-window rule."""
    S, Hkv, kmax = orc.idx.shape
    windowed = 0
    for s in range(S):
        np_ = n_pages[s]
        kp = kp_of[s]
        for h in range(Hkv):
            g = gpu_idx[s, h]
            c = int(gpu_cnt[s, h])
            assert c == int(orc.cnt[s, h]), (s, h, c, orc.cnt[s, h])
            assert np.all(g[c:] == -1), (s, h, "padding")
            assert np.all(np.diff(g[:c]) > 0), (s, h, "ascending")
            want = orc.idx[s, h, :c]
            if kp >= np_:
                assert np.array_equal(g[:c], want), (s, h)
                continue
            sc = orc.score[s, h, :np_]
            order = np.lexsort((np.arange(np_), -sc))
            s_k, s_k1 = sc[order[kp - 1]], sc[order[kp]]
            if s_k - s_k1 > rel * s_k:
                assert np.array_equal(g[:c], want), (s, h, sorted(set(g[:c]) ^ set(want)))
            else:
                windowed += 1
                W = set(np.nonzero(np.abs(sc - s_k) <= rel * s_k)[0].tolist())
                gs, ws = set(g[:c].tolist()), set(want.tolist())
                assert len(gs) == kp
                assert (ws - W) <= gs, (s, h)
                assert not ((gs - ws) - W), (s, h)
    return windowed


def check_output(gpu_o: torch.Tensor, ref: np.ndarray, what: str,
                 max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    got = gpu_o.float().cpu().numpy().astype(np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= max_abs and mean <= mean_abs, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def check_global_selection(gpu_idx, gpu_cnt, orc, n_pages, kp_of, rel=TIE_REL):
    """Head-adaptive budget: per sequence, the kept (KV head, page) pairs.  Bit-exact
    unless the oracle's K-th and (K+1)-th pair scores (K = Hkv * kp) are within `rel`;
    then pairs in the window W = {|S - s_K| <= rel * s_K} may go either way, the number
    kept must be K and every pair outside W must agree.  Returns the windowed count."""
    S, Hkv, _ = gpu_idx.shape
    windowed = 0
    for s in range(S):
        np_ = n_pages[s]
        got, want = set(), set()
        for h in range(Hkv):
            c = int(gpu_cnt[s, h])
            g = gpu_idx[s, h]
            assert np.all(g[c:] == -1), (s, h, "padding")
            assert np.all(np.diff(g[:c]) > 0), (s, h, "ascending")
            assert np.all((g[:c] >= 0) & (g[:c] < np_)), (s, h, "range")
            got |= {(h, int(q)) for q in g[:c]}
            want |= {(h, int(q)) for q in orc.idx[s, h, :orc.cnt[s, h]]}
        total = Hkv * np_
        K = min(Hkv * kp_of[s], total)
        assert len(got) == K, (s, len(got), K)
        if K == total or got == want:
            assert got == want, (s, sorted(got ^ want))
            continue
        sc = orc.score[s, :, :np_].reshape(-1)          # pair (h, q) at h * np + q
        order = np.lexsort((np.arange(total), -sc))
        s_k, s_k1 = sc[order[K - 1]], sc[order[K]]
        assert s_k - s_k1 <= rel * s_k, (s, sorted(got ^ want))
        windowed += 1
        W = {(int(i) // np_, int(i) % np_) for i in np.nonzero(np.abs(sc - s_k) <= rel * s_k)[0]}
        assert (want - W) <= got, s
        assert not ((got - want) - W), s
    return windowed
