"""Head-adaptive budget ("Step-dLLM: Adaptive Step-aware Sparse Attention for
Efficient Diffusion LLM Inference", abstract): one budget of Hkv * kp pages per
sequence shared by its KV heads.  The CUDA path against the oracle's
select_global, and the sparse pass on the resulting per-head counts."""
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
    "32k_small": ("32k", dict(n=6000)),
    "ragged_paged": ("batched", dict(S=3, n_lo=1500, n_hi=5000, topk_choices=(512, 1024))),
}


def kp_list(w):
    return [int(w.topk[s]) // w.P for s in range(w.S)]


def run_global_case(dsa_mod, w, steps=(2,)):
    dw = dsa_mod.DeviceWorkload(w, head_budget=1)
    dw.select()
    torch.cuda.synchronize()
    assert dw.ws_sel.status() == dsa_mod.DSA_OK
    pt = None if w.page_table is None else w.page_table.numpy()
    ref = oracle.select_global(W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                               w.topk.numpy(), kmax=dw.kmax, page_table=pt, max_pages=w.max_pages)
    gidx, gcnt = dw.idx.cpu().numpy(), dw.cnt.cpu().numpy()
    parity.check_global_selection(gidx, gcnt, ref, [w.n_pages(s) for s in range(w.S)], kp_list(w))
    parity.check_output(dw.o_sel, ref.o, f"{w.name} head-budget selection o_out")
    for t in steps:
        q, bk, bv = w.step_inputs(t)
        o = dw.sparse(q.cuda(), bk.cuda(), bv.cuda())
        torch.cuda.synchronize()
        assert dw.ws_sp.status() == dsa_mod.DSA_OK
        ref_o, _ = oracle.sparse(W.bits(q), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                                 gidx, gcnt, W.bits(bk), W.bits(bv), page_table=pt,
                                 max_pages=w.max_pages)
        parity.check_output(o, ref_o, f"{w.name} head-budget sparse step {t}")
    return dw, ref


@pytest.mark.parametrize("case", list(CASES), ids=list(CASES))
def test_head_budget_parity(dsa_mod, case):
    name, kw = CASES[case]
    dw, ref = run_global_case(dsa_mod, W.make(name, 0, **kw), steps=(2, 3))
    # the counts really differ between heads somewhere (else the test shows nothing)
    if case == "ragged_paged":
        assert len(set(dw.cnt.cpu().numpy().reshape(-1).tolist())) > 1


def test_head_budget_concentrated_head(dsa_mod):
    """A head whose attention sits on two planted pages keeps only those."""
    w = W.make("tiny", 7, n=2000, topk=128, B=4, Hq=4, Hkv=2, d=64, needle_count=0)
    q = w.q1.float().view(w.S, w.B, w.Hkv, w.G, w.d).mean(dim=(1, 3))[0]
    k = w.k_cache.float()
    for lp in (5, 40):
        k[lp, 0] += 8.0 * q[0]
    w.k_cache = k.to(torch.bfloat16)
    dw, ref = run_global_case(dsa_mod, w)
    c0 = int(dw.cnt[0, 0])
    assert dw.idx[0, 0, :c0].cpu().tolist() == [5, 40]
    assert int(dw.cnt[0, 1]) == 2 * (128 // w.P) - 2


def test_head_budget_full_size(dsa_mod):
    """128K workload: one budget of 8 * 64 pages shared by the 8 KV heads."""
    run_global_case(dsa_mod, W.make("128k", 0), steps=(2,))


def test_head_budget_launches(dsa_mod):
    w = W.make("8k", 0, n=3000, topk=256)
    dw = dsa_mod.DeviceWorkload(w, head_budget=1)
    assert dsa_mod.select_launches(dw.dims) == 2
    dw1 = dsa_mod.DeviceWorkload(w)
    assert dsa_mod.select_launches(dw1.dims) == 1


@pytest.mark.parametrize("n,Hkv,topk,path", [(1000, 2, 256, "head lists"), (20000, 8, 256, "head lists"),
                                              (40000, 8, 4096, "every pair, keys from L2")])
def test_head_budget_all_ties(dsa_mod, n, Hkv, topk, path):
    """All keys zero: every full page of every head has the same score, bit for bit,
    on both sides.  The shared budget then goes to the lowest (head, page) pairs:
    head 0 takes it all and the other heads keep nothing (the sparse pass then
    attends to the block alone for them).  The last case's head lists (8 x 2048)
    exceed the global kernel's staging area, so it ranks every pair, and with all
    keys equal no histogram narrows them: its radix passes read the keys from L2."""
    w = W.make("tiny", 3, n=n, topk=topk, B=4, Hq=2 * Hkv, Hkv=Hkv, d=64, needle_count=0)
    w.k_cache = torch.zeros_like(w.k_cache)
    dw, ref = run_global_case(dsa_mod, w)
    got = dw.idx.cpu().numpy()
    K = Hkv * (topk // w.P)
    assert int(dw.cnt[0, 0]) == K and got[0, 0, :K].tolist() == list(range(K))
    assert dw.cnt[0, 1:].sum().item() == 0
    assert np.array_equal(got, ref.idx) and np.array_equal(dw.cnt.cpu().numpy(), ref.cnt)


def test_head_budget_long_lists(dsa_mod):
    """Head lists longer than the global kernel's staging area (8 x 2048 > 8192
    candidates): it ranks every (head, page) pair instead, through the key range,
    histogram narrowing and compaction of the keys above the cut."""
    run_global_case(dsa_mod, W.make("tiny", 5, n=40000, topk=4096, B=4, Hq=16, Hkv=8, d=64,
                                    needle_count=16))
