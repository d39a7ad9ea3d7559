"""Reuse of the prefix part for stable tokens ("LoSA: Locality Aware Sparse
Attention for Block-Wise Diffusion Language Models", abstract), on the GPU against
the oracle's sparse_losa: step 2 with every token active fills the caches, step 3
reuses them for the stable tokens of a mask."""
import numpy as np
import pytest
import torch

import oracle
import parity
from block_sparse_attention_27_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa_mod():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    from block_sparse_attention_27_b200 import build, dsa
    build.build()
    dsa.load()
    return dsa


CASES = {
    "tiny": ("tiny", {}),
    "8k_small": ("8k", dict(n=3000, topk=256)),
    "ragged_paged": ("batched", dict(S=3, n_lo=1500, n_hi=5000, topk_choices=(512, 1024))),
}


def check_cache(got_o, got_lse, ref_o, ref_lse, rows, what):
    """The cache rows selected by `rows` ([S, B] bool) against the oracle's."""
    go = got_o.float().cpu().numpy()[rows]
    gl = got_lse.cpu().numpy().astype(np.float64)[rows]
    ro, rl = ref_o[rows], ref_lse[rows]
    assert np.all(np.isfinite(go)) and np.max(np.abs(go - ro)) <= parity.MAX_ABS, what
    assert np.mean(np.abs(go - ro)) <= parity.MEAN_ABS, what
    assert np.max(np.abs(gl - rl)) <= 1e-3, what


def run_losa_case(dsa_mod, w, active3):
    dw = dsa_mod.DeviceWorkload(w)
    dw.select()
    torch.cuda.synchronize()
    gidx, gcnt = dw.idx.cpu().numpy(), dw.cnt.cpu().numpy()
    pt = None if w.page_table is None else w.page_table.numpy()
    dev = dw.q1.device
    cache_o = torch.zeros(w.q1.shape, dtype=torch.bfloat16, device=dev)
    cache_lse = torch.zeros(w.q1.shape[:3], dtype=torch.float32, device=dev)

    def ref(q, bk, bv, active, co, cl):
        return oracle.sparse_losa(W.bits(q), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                                  gidx, gcnt, W.bits(bk), W.bits(bv), active, W.bits(co.cpu()),
                                  cl.cpu().numpy().astype(np.float64), page_table=pt,
                                  max_pages=w.max_pages)

    # step 2, every token active: the caches are written, the output is the plain sparse pass
    q, bk, bv = w.step_inputs(2)
    all_on = np.ones((w.S, w.B), bool)
    o = dw.sparse(q.to(dev), bk.to(dev), bv.to(dev), active=torch.ones((w.S, w.B), dtype=torch.uint8, device=dev),
                  cache=(cache_o, cache_lse))
    torch.cuda.synchronize()
    assert dw.ws_sp.status() == dsa_mod.DSA_OK
    r_o, _, r_co, r_cl = ref(q, bk, bv, all_on, torch.zeros_like(cache_o), torch.zeros_like(cache_lse))
    parity.check_output(o, r_o, f"{w.name} step 2 (all active)")
    rows = np.ones((w.S, w.B, w.Hq), bool)
    check_cache(cache_o, cache_lse, r_co, r_cl, rows, f"{w.name} step 2 cache")

    # step 3 with the mask: stable tokens reuse the step-2 caches
    prev_o, prev_l = cache_o.clone(), cache_lse.clone()
    q, bk, bv = w.step_inputs(3)
    o = dw.sparse(q.to(dev), bk.to(dev), bv.to(dev), active=torch.from_numpy(active3.astype(np.uint8)).to(dev),
                  cache=(cache_o, cache_lse))
    torch.cuda.synchronize()
    assert dw.ws_sp.status() == dsa_mod.DSA_OK
    r_o, _, r_co, r_cl = ref(q, bk, bv, active3, prev_o, prev_l)
    parity.check_output(o, r_o, f"{w.name} step 3 (mask)")
    act_rows = np.repeat(active3[:, :, None], w.Hq, axis=2)
    if act_rows.any():
        check_cache(cache_o, cache_lse, r_co, r_cl, act_rows, f"{w.name} step 3 cache, active rows")
    stable = torch.from_numpy(~act_rows).to(dev)
    assert torch.equal(cache_o[stable], prev_o[stable]), "a stable row's cache changed"
    assert torch.equal(cache_lse[stable], prev_l[stable]), "a stable row's cache changed"
    return dw


@pytest.mark.parametrize("case", list(CASES), ids=list(CASES))
@pytest.mark.parametrize("mask", ["mixed", "all_stable", "one_sequence_stable"])
def test_losa_parity(dsa_mod, case, mask):
    name, kw = CASES[case]
    w = W.make(name, 0, **kw)
    rng = np.random.default_rng(11)
    if mask == "mixed":
        active = rng.random((w.S, w.B)) < 0.3
        active[:, 0] = True
    elif mask == "all_stable":
        active = np.zeros((w.S, w.B), bool)
    else:
        active = rng.random((w.S, w.B)) < 0.5
        active[0] = False
        if w.S > 1:
            active[1:, 0] = True
    run_losa_case(dsa_mod, w, active)


def test_losa_rejects_missing_cache(dsa_mod):
    w = W.make("tiny", 0)
    dw = dsa_mod.DeviceWorkload(w)
    q, bk, bv = (x.cuda() for x in w.step_inputs(2))
    act = torch.ones((w.S, w.B), dtype=torch.uint8, device="cuda")
    with pytest.raises(TypeError):
        dw.sparse(q, bk, bv, active=act, cache=(None, None))
