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


VARIANTS = os.path.join(os.path.dirname(__file__), "golden", "variants_oracle.json")


def test_oracle_variants_match_golden():
    """Head-adaptive budget and prefix-part reuse reproduce their stored outputs."""
    import torch
    g = json.load(open(VARIANTS))
    w = W.make(g["workload"], g["seed"], **g["overrides"])
    args = (W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(), w.topk.numpy())
    sg = oracle.select_global(*args, kmax=w.max_pages)
    assert sg.idx[0].tolist() == g["global_idx"] and sg.cnt[0].tolist() == g["global_cnt"]
    r = oracle.select(*args)
    q2, bk2, bv2 = w.step_inputs(2)
    o2, _, co2, cl2 = oracle.sparse_losa(W.bits(q2), W.bits(w.k_cache), W.bits(w.v_cache),
                                         w.n_ctx.numpy(), r.idx, r.cnt, W.bits(bk2), W.bits(bv2),
                                         np.ones((w.S, w.B), bool), np.zeros(W.bits(w.q1).shape, np.uint16),
                                         np.zeros(w.q1.shape[:3]))
    assert np.allclose(o2[0, 0, 0], g["losa_step2_o_row0"], rtol=1e-12, atol=1e-15)
    assert np.allclose(cl2.reshape(-1), g["losa_step2_cache_lse"], rtol=1e-13)
    q3, bk3, bv3 = w.step_inputs(3)
    o3, lse3, _, _ = oracle.sparse_losa(W.bits(q3), W.bits(w.k_cache), W.bits(w.v_cache),
                                        w.n_ctx.numpy(), r.idx, r.cnt, W.bits(bk3), W.bits(bv3),
                                        np.array(g["losa_step3_mask"], bool),
                                        W.bits(torch.from_numpy(co2).to(torch.bfloat16)), cl2)
    assert np.allclose(o3.reshape(-1)[:64], g["losa_step3_o"], rtol=1e-12, atol=1e-15)
    assert np.allclose(lse3.reshape(-1), g["losa_step3_lse"], rtol=1e-13)
