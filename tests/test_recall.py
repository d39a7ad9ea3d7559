"""Per-step top-k recall of a reused selection (MAGE page, Surprising findings)
and anchor-step refresh: the set arithmetic on the CPU, the GPU measurement
against recall computed from the oracle's own selections."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_27_b200 import recall as R
from block_sparse_attention_27_b200 import workloads as W


def test_set_recall_arithmetic():
    exact = np.array([[[1, 2, 3, -1], [4, 5, -1, -1]]])
    ecnt = np.array([[3, 2]])
    used = np.array([[[1, 3, 7, -1], [4, 5, 6, -1]]])
    ucnt = np.array([[3, 3]])
    # head 0: {1,3} of {1,2,3} = 2/3; head 1: {4,5} of {4,5} = 1
    assert abs(R.set_recall(used, ucnt, exact, ecnt) - (2 / 3 + 1) / 2) < 1e-12
    assert R.set_recall(exact, ecnt, exact, ecnt) == 1.0
    empty = np.zeros((1, 2), np.int64)
    assert R.set_recall(used, ucnt, exact, empty) == 1.0


def _oracle_sets(w, t):
    q = w.step_inputs(t)[0]
    pt = None if w.page_table is None else w.page_table.numpy()
    r = oracle.select(W.bits(q), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                      w.topk.numpy(), page_table=pt, max_pages=w.max_pages)
    return r.idx, r.cnt


@pytest.mark.gpu
@pytest.mark.parametrize("name,kw", [("8k", dict(n=3000, topk=256)), ("tiny", {})])
def test_step_recall_matches_oracle(name, kw):
    from block_sparse_attention_27_b200 import dsa
    w = W.make(name, 0, **kw)
    T = 4
    dw = dsa.DeviceWorkload(w)
    qs = [w.step_inputs(t)[0].cuda() for t in range(1, T + 1)]
    got = R.step_recall(dw, qs)
    ref_sets = [_oracle_sets(w, t) for t in range(1, T + 1)]
    want = [R.set_recall(*ref_sets[0], *ref_sets[t]) for t in range(T)]
    assert got[0] == 1.0
    assert np.allclose(got, want, atol=1e-12), (got, want)
    # refreshing at every step uses the exact set every time
    assert R.step_recall(dw, qs, anchor=1) == [1.0] * T
    # refresh every 2 steps: steps 1 and 3 exact, 2 and 4 reuse the previous anchor
    got2 = R.step_recall(dw, qs, anchor=2)
    want2 = [1.0, R.set_recall(*ref_sets[0], *ref_sets[1]), 1.0,
             R.set_recall(*ref_sets[2], *ref_sets[3])]
    assert np.allclose(got2, want2, atol=1e-12), (got2, want2)
