"""Exact step-1 output (prefix and block) from the selection pass's prefix-only
output and the block-only sparse pass, merged through their log-sum-exps
(dsa_merge_attn), against the oracle's dense attention over prefix + block; and
the row log-sum-exps of both passes against the oracle's."""
import numpy as np
import pytest
import torch

import oracle
import parity
from block_sparse_attention_27_b200 import workloads as W

pytestmark = pytest.mark.gpu

LSE_TOL = 2e-3   # fp32 log-sum-exp of bf16 logits over up to 128K keys


@pytest.mark.parametrize("name,kw", [("8k", dict(n=3000, topk=256)), ("tiny", {}),
                                     ("batched", dict(S=3, n_lo=100, n_hi=3000, B=8, Hq=8, Hkv=2,
                                                      topk_choices=(64, 128)))])
def test_exact_step1_and_lse(name, kw):
    from block_sparse_attention_27_b200 import dsa
    w = W.make(name, 0, **kw)
    dw = dsa.DeviceWorkload(w)
    rows = w.q1.shape[:3]
    lse_sel = torch.empty(rows, dtype=torch.float32, device="cuda")
    lse_blk = torch.empty_like(lse_sel)
    lse_all = torch.empty_like(lse_sel)
    idx, cnt, o_sel = dw.select(lse_out=lse_sel)
    o_sel = o_sel.clone()
    zero = torch.zeros_like(dw.cnt)
    o_blk = dw.sparse(dw.q1, dw.blk_k1, dw.blk_v1, cnt=zero, lse_out=lse_blk).clone()
    o_all = torch.empty_like(o_sel)
    dsa.dsa_merge_attn(o_sel, lse_sel, o_blk, lse_blk, o_all, lse_all)
    torch.cuda.synchronize()
    assert dw.ws_sel.status() == dsa.DSA_OK and dw.ws_sp.status() == dsa.DSA_OK

    pt = None if w.page_table is None else w.page_table.numpy()
    ref_sel = oracle.select(W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                            w.topk.numpy(), page_table=pt, max_pages=w.max_pages)
    assert np.max(np.abs(lse_sel.cpu().numpy() - ref_sel.lse)) < LSE_TOL
    idx_all, cnt_all = oracle.all_pages(w.n_ctx.numpy(), w.P, w.Hkv)
    dense_o, dense_lse = oracle.sparse(W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache),
                                       w.n_ctx.numpy(), idx_all, cnt_all, W.bits(w.blk_k1),
                                       W.bits(w.blk_v1), page_table=pt, max_pages=w.max_pages)
    parity.check_output(o_all, dense_o, f"{w.name} exact step-1 output")
    assert np.max(np.abs(lse_all.cpu().numpy() - dense_lse)) < LSE_TOL
    none = np.zeros_like(cnt_all)
    blk_o, blk_lse = oracle.sparse(W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache),
                                   w.n_ctx.numpy(), idx_all, none, W.bits(w.blk_k1),
                                   W.bits(w.blk_v1), page_table=pt, max_pages=w.max_pages)
    parity.check_output(o_blk, blk_o, f"{w.name} block-only attention")
    assert np.max(np.abs(lse_blk.cpu().numpy() - blk_lse)) < LSE_TOL
