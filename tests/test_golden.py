"""The oracle reproduces its stored golden output (regression fixture)."""
import json
import os

import numpy as np

import oracle
from block_sparse_attention_27_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")


def test_oracle_matches_golden():
    g = json.load(open(GOLDEN))
    w = W.make(g["workload"], g["seed"])
    r = oracle.select(W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                      w.topk.numpy())
    assert r.idx[0, 0].tolist() == g["idx"] and int(r.cnt[0, 0]) == g["cnt"]
    assert np.allclose(r.score[0, 0], g["page_score"], rtol=1e-13, atol=0)
    assert np.allclose(r.o[0, 0, 0], g["select_o_row0"], rtol=1e-12, atol=1e-15)
    assert np.allclose(r.lse.reshape(-1), g["select_lse"], rtol=1e-13)
    q2, bk2, bv2 = w.step_inputs(2)
    o2, lse2 = oracle.sparse(W.bits(q2), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                             r.idx, r.cnt, W.bits(bk2), W.bits(bv2))
    assert np.allclose(o2[0, 0, 0], g["step2_o_row0"], rtol=1e-12, atol=1e-15)
    assert np.allclose(lse2.reshape(-1), g["step2_lse"], rtol=1e-13)
