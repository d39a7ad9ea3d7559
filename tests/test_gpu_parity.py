"""CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

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


# name -> (workload, overrides); sizes span several tiles and ragged tails
CASES = {
    "tiny": ("tiny", {}),
    "tiny_tail_d64": ("tiny", dict(n=1000, topk=96)),
    "8k": ("8k", {}),
    "32k_g7_p64": ("32k", {}),
    "small_g7_p64_tail": ("32k", dict(n=5000, topk=512)),
    "ragged_paged": ("batched", dict(S=3, n_lo=100, n_hi=3000, B=8, Hq=8, Hkv=2,
                                     topk_choices=(64, 128, 4096))),
    "b1": ("8k", dict(n=3000, B=1, topk=256)),
    "kp1": ("8k", dict(n=2000, topk=16)),
    "budget_covers_prefix": ("8k", dict(n=1500, topk=2048)),
    "p32": ("8k", dict(n=4000, P=32, topk=512)),
    "p64_d64": ("tiny", dict(n=3000, P=64, topk=256, B=8, Hq=8, Hkv=2)),
    # more selected pages than the all-keys-resident kernel's CTAs can hold: the
    # streaming kernel serves it
    "wide_budget": ("8k", dict(n=8000, topk=8192)),
}


def kp_list(w):
    return [int(w.topk[s]) // w.P for s in range(w.S)]


def run_case(dsa_mod, w, steps=(2,), sm_limit=0, early_gather=0):
    dw = dsa_mod.DeviceWorkload(w, sm_limit=sm_limit, early_gather=early_gather)
    dw.select()
    torch.cuda.synchronize()
    assert dw.ws_sel.status() == dsa_mod.DSA_OK
    pt = None if w.page_table is None else w.page_table.numpy()
    ref = oracle.select(W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                        w.topk.numpy(), page_table=pt, max_pages=w.max_pages)
    gidx, gcnt = dw.idx.cpu().numpy(), dw.cnt.cpu().numpy()
    parity.check_selection(gidx, gcnt, ref, [w.n_pages(s) for s in range(w.S)], kp_list(w))
    parity.check_output(dw.o_sel, ref.o, f"{w.name} selection o_out")
    for t in steps:
        q, bk, bv = w.step_inputs(t)
        o = dw.sparse(q.cuda(), bk.cuda(), bv.cuda())
        torch.cuda.synchronize()
        assert dw.ws_sp.status() == dsa_mod.DSA_OK
        ref_o, _ = oracle.sparse(W.bits(q), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                                 gidx, gcnt, W.bits(bk), W.bits(bv), page_table=pt,
                                 max_pages=w.max_pages)
        parity.check_output(o, ref_o, f"{w.name} sparse step {t}")
    return dw, ref


@pytest.mark.parametrize("case", list(CASES), ids=list(CASES))
def test_parity(dsa_mod, case):
    name, kw = CASES[case]
    run_case(dsa_mod, W.make(name, 0, **kw), steps=(2, 3))


@pytest.mark.parametrize("name,sm_limit", [("8k", 20), ("8k", 37), ("ragged_paged", 6)])
def test_parity_with_sm_limit(dsa_mod, name, sm_limit):
    """A selection pass held to fewer SMs (fewer splits) computes the same result."""
    wname, kw = CASES[name]
    run_case(dsa_mod, W.make(wname, 0, **kw), sm_limit=sm_limit)


@pytest.mark.parametrize("name", ["128k", "batched"])
def test_parity_full_size(dsa_mod, name):
    """Full-size workloads in the launch configuration the bench times."""
    run_case(dsa_mod, W.make(name, 0), steps=(2,), early_gather=1)


EARLY_CASES = ["tiny", "tiny_tail_d64", "8k", "32k_g7_p64", "ragged_paged", "kp1",
               "budget_covers_prefix", "p64_d64", "wide_budget"]


@pytest.mark.parametrize("case,resident", [("tiny", True), ("8k", True), ("32k_g7_p64", True),
                                           ("ragged_paged", True), ("p64_d64", True),
                                           ("wide_budget", False)])
def test_sparse_kernel_choice(dsa_mod, case, resident):
    """Which sparse kernel serves a shape (dsa_sparse_kernel): the all-keys-resident
    kernel for the workloads' budgets, the streaming one past 16 CTAs x 256 keys or
    with prefix-part reuse; the parity tests above then cover both."""
    name, kw = CASES[case]
    w = W.make(name, 0, **kw)
    dw = dsa_mod.DeviceWorkload(w)
    got = dsa_mod.sparse_kernel(dw.dims)
    assert (got > 1) == resident, got
    if resident:
        on = torch.ones((w.S, w.B), dtype=torch.uint8, device="cuda")
        d = dsa_mod.dsa_dims.from_buffer_copy(dw.dims)
        d.active = on.data_ptr()
        assert dsa_mod.sparse_kernel(d) == 1


@pytest.mark.parametrize("name", ["128k", "batched"])
def test_sparse_kernel_choice_full_size(dsa_mod, name):
    w = W.make(name, 0)
    dw = dsa_mod.DeviceWorkload(w)
    assert dsa_mod.sparse_kernel(dw.dims) > 1


@pytest.mark.parametrize("case", EARLY_CASES, ids=EARLY_CASES)
def test_parity_early_gather(dsa_mod, case):
    """dims.early_gather = 1: the pages are gathered before the dependency wait."""
    name, kw = CASES[case]
    run_case(dsa_mod, W.make(name, 0, **kw), steps=(2, 3), early_gather=1)


@pytest.mark.parametrize("case", ["8k", "ragged_paged", "128k", "batched"])
def test_early_gather_back_to_back(dsa_mod, case):
    """Sparse steps of two layers queued back to back on one stream (each kernel a
    programmatic dependent of the one before, so each gathers its pages while the
    previous step still runs), every output against the oracle."""
    name, kw = CASES.get(case, (case, {}))
    ws = [W.make(name, seed, **kw) for seed in (0, 1)]
    dws = [dsa_mod.DeviceWorkload(w, early_gather=1) for w in ws]
    for dw in dws:
        dw.select()
    torch.cuda.synchronize()
    steps = (2, 3, 4)
    inputs = [[tuple(x.cuda() for x in w.step_inputs(t)) for t in steps] for w in ws]
    outs = [[torch.empty_like(dw.q1) for _ in steps] for dw in dws]
    for i in range(len(steps)):
        for li, dw in enumerate(dws):
            dw.sparse(*inputs[li][i], out=outs[li][i])
    torch.cuda.synchronize()
    for li, (w, dw) in enumerate(zip(ws, dws)):
        assert dw.ws_sp.status() == dsa_mod.DSA_OK
        pt = None if w.page_table is None else w.page_table.numpy()
        gidx, gcnt = dw.idx.cpu().numpy(), dw.cnt.cpu().numpy()
        for i, t in enumerate(steps):
            q, bk, bv = w.step_inputs(t)
            ref_o, _ = oracle.sparse(W.bits(q), W.bits(w.k_cache), W.bits(w.v_cache),
                                     w.n_ctx.numpy(), gidx, gcnt, W.bits(bk), W.bits(bv),
                                     page_table=pt, max_pages=w.max_pages)
            parity.check_output(outs[li][i], ref_o, f"{w.name} layer {li} step {t}")


def test_planted_needles_selected(dsa_mod):
    w = W.make("tiny", 0)
    dw = dsa_mod.DeviceWorkload(w)
    dw.select()
    assert dw.idx[0, 0].cpu().tolist() == w.planted[(0, 0)]


def test_exact_ties_resolved_within_window(dsa_mod):
    w = W.make("8k", 1, n=2048, topk=256)
    for b, a in ((40, 3), (77, 10), (100, 64)):      # bit-identical page copies
        w.k_cache[b] = w.k_cache[a]
        w.v_cache[b] = w.v_cache[a]
    run_case(dsa_mod, w)


def test_dense_when_budget_covers_prefix(dsa_mod):
    """kp >= pages: the sparse pass is dense attention over prefix + block."""
    w = W.make("8k", 2, n=1200, topk=2048)
    dw, _ = run_case(dsa_mod, w)
    idx, cnt = oracle.all_pages(w.n_ctx.numpy(), w.P, w.Hkv, kmax=w.kmax)
    assert np.array_equal(dw.idx.cpu().numpy(), idx)


def test_bad_index_reported_not_faulting(dsa_mod):
    w = W.make("8k", 3, n=1000, topk=128)
    dw = dsa_mod.DeviceWorkload(w)
    dw.select()
    idx = dw.idx.clone()
    idx[0, 0, 0] = w.n_pages(0) + 5      # past the prefix
    idx[0, 1, 1] = -7
    q, bk, bv = w.step_inputs(2)
    dw.sparse(q.cuda(), bk.cuda(), bv.cuda(), idx=idx)
    torch.cuda.synchronize()
    assert dw.ws_sp.status() == dsa_mod.DSA_ERR_BAD_INDEX
    assert torch.isfinite(dw.o_sp.float()).all()


def test_nonfinite_input_reported(dsa_mod):
    w = W.make("8k", 4, n=1000, topk=128)
    w.q1[0, 0, 0, 0] = float("nan")
    dw = dsa_mod.DeviceWorkload(w)
    dw.select()
    torch.cuda.synchronize()
    assert dw.ws_sel.status() == dsa_mod.DSA_ERR_NONFINITE


def test_selection_on_second_stream(dsa_mod):
    """Selection on a side stream, gated to the sparse stream by an event, gives the
    same indices and outputs as running everything on one stream."""
    w = W.make("8k", 5, n=6000)
    dw = dsa_mod.DeviceWorkload(w)
    q, bk, bv = (x.cuda() for x in w.step_inputs(2))
    dw.select()
    o_ref = dw.sparse(q, bk, bv).clone()
    idx_ref = dw.idx.clone()
    dw.idx.fill_(-1)
    side = torch.cuda.Stream()
    ev = torch.cuda.Event()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        dw.select(stream=side)
        ev.record(side)
    torch.cuda.current_stream().wait_event(ev)
    o = dw.sparse(q, bk, bv)
    torch.cuda.synchronize()
    assert torch.equal(dw.idx, idx_ref)
    assert torch.equal(o, o_ref)


@pytest.mark.parametrize("case", ["8k", "ragged_paged"])
def test_selection_stream_overlap_against_oracle(dsa_mod, case):
    """The bench's step shape, checked against the oracle: for two layers, the
    selection of block n+1 runs on a side stream while block n's sparse steps run on
    the main stream (early gathering on, ping-pong index buffers); then block n+1's
    first sparse step waits for the selection's event.  Every selection and every
    sparse output is compared with the oracle."""
    name, kw = CASES[case]
    ws = [W.make(name, seed, **kw) for seed in (0, 1)]
    dws = [dsa_mod.DeviceWorkload(w, early_gather=1) for w in ws]
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    idx = [[torch.full_like(dw.idx, -1) for _ in range(2)] for dw in dws]
    cnt = [[torch.zeros_like(dw.cnt) for _ in range(2)] for dw in dws]
    o_sel = [torch.empty_like(dw.q1) for dw in dws]
    # block n's indices, then block n+1's queries (another step's draw stands in)
    q_next = [w.step_inputs(9)[0] for w in ws]
    for li, dw in enumerate(dws):
        dw.select()
        idx[li][0].copy_(dw.idx)
        cnt[li][0].copy_(dw.cnt)
    torch.cuda.synchronize()
    steps = (2, 3, 4)
    inputs = [[tuple(x.cuda() for x in w.step_inputs(t)) for t in steps] for w in ws]
    qn = [q.cuda() for q in q_next]
    outs = [[torch.empty_like(dw.q1) for _ in range(len(steps) + 1)] for dw in dws]
    side.wait_stream(main)
    with torch.cuda.stream(side):
        for li, dw in enumerate(dws):
            dsa_mod.dsa_select(qn[li], dw.k_cache, dw.v_cache, dw.n_ctx, dw.w.P, dw.topk,
                               idx[li][1], o_sel[li], side, dims=dw.dims, cnt_out=cnt[li][1],
                               workspace=dw.ws_sel)
    ev = torch.cuda.Event()
    ev.record(side)
    for i in range(len(steps)):
        for li, dw in enumerate(dws):
            dw.sparse(*inputs[li][i], idx=idx[li][0], cnt=cnt[li][0], out=outs[li][i])
    main.wait_event(ev)
    for li, dw in enumerate(dws):   # block n+1, its first later step
        dw.sparse(*inputs[li][0], idx=idx[li][1], cnt=cnt[li][1], out=outs[li][-1])
    torch.cuda.synchronize()
    for li, (w, dw) in enumerate(zip(ws, dws)):
        assert dw.ws_sel.status() == dsa_mod.DSA_OK and dw.ws_sp.status() == dsa_mod.DSA_OK
        pt = None if w.page_table is None else w.page_table.numpy()
        ref_n = oracle.select(W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                              w.topk.numpy(), page_table=pt, max_pages=w.max_pages)
        ref_n1 = oracle.select(W.bits(q_next[li]), W.bits(w.k_cache), W.bits(w.v_cache),
                               w.n_ctx.numpy(), w.topk.numpy(), page_table=pt,
                               max_pages=w.max_pages)
        npg = [w.n_pages(s) for s in range(w.S)]
        gi0, gc0 = idx[li][0].cpu().numpy(), cnt[li][0].cpu().numpy()
        gi1, gc1 = idx[li][1].cpu().numpy(), cnt[li][1].cpu().numpy()
        parity.check_selection(gi0, gc0, ref_n, npg, kp_list(w))
        parity.check_selection(gi1, gc1, ref_n1, npg, kp_list(w))
        parity.check_output(o_sel[li], ref_n1.o, f"{w.name} layer {li} side-stream selection")
        for i, t in enumerate(steps + (steps[0],)):
            gi, gc = (gi0, gc0) if i < len(steps) else (gi1, gc1)
            q, bk, bv = w.step_inputs(t)
            ref_o, _ = oracle.sparse(W.bits(q), W.bits(w.k_cache), W.bits(w.v_cache),
                                     w.n_ctx.numpy(), gi, gc, W.bits(bk), W.bits(bv),
                                     page_table=pt, max_pages=w.max_pages)
            parity.check_output(outs[li][i], ref_o, f"{w.name} layer {li} output {i}")


def test_deterministic(dsa_mod):
    w = W.make("8k", 6, n=5000)
    dw = dsa_mod.DeviceWorkload(w)
    q, bk, bv = (x.cuda() for x in w.step_inputs(2))
    dw.select()
    a = (dw.idx.clone(), dw.o_sel.clone(), dw.sparse(q, bk, bv).clone())
    dw.select()
    b = (dw.idx.clone(), dw.o_sel.clone(), dw.sparse(q, bk, bv).clone())
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def _poison(dsa_mod, ws):
    """Fill a workspace with 0xFF bytes (NaN as fp32), then zero its status header:
    a kernel that reads a word it did not write this call now sees NaN."""
    ws.buf.fill_(0xFF)
    rc = dsa_mod.load().dsa_workspace_init(dsa_mod._ptr(ws.buf), ws.nbytes, dsa_mod._stream(None))
    assert rc == dsa_mod.DSA_OK


def test_repeatable_on_poisoned_workspaces(dsa_mod):
    """Full-size 128K: four selection passes and four sparse steps, each on freshly
    poisoned workspaces, give finite results that are bitwise identical from run to
    run (catches reads of unwritten workspace and timing-dependent races)."""
    w = W.make("128k", 0)
    dw = dsa_mod.DeviceWorkload(w)
    q, bk, bv = (x.cuda() for x in w.step_inputs(2))
    first = None
    for _ in range(4):
        _poison(dsa_mod, dw.ws_sel)
        _poison(dsa_mod, dw.ws_sp)
        idx, cnt, o_sel = (t.clone() for t in dw.select())
        o_sp = dw.sparse(q, bk, bv).clone()
        torch.cuda.synchronize()
        assert dw.ws_sel.status() == dsa_mod.DSA_OK and dw.ws_sp.status() == dsa_mod.DSA_OK
        bad_sel = (~torch.isfinite(o_sel.float())).nonzero()
        bad_sp = (~torch.isfinite(o_sp.float())).nonzero()
        assert len(bad_sel) == 0, f"selection output: {len(bad_sel)} non-finite, first {bad_sel[:4].tolist()}"
        assert len(bad_sp) == 0, f"sparse output: {len(bad_sp)} non-finite, first {bad_sp[:4].tolist()}"
        got = (idx, cnt, o_sel, o_sp)
        if first is None:
            first = got
        else:
            for a, b in zip(first, got):
                assert torch.equal(a, b)


def test_empty_prefix(dsa_mod):
    """A sequence with an empty prefix (n_ctx = 0) beside a normal one: its selection
    keeps no page (idx -1, cnt 0, o_out 0, log-sum-exp -inf), its sparse step attends
    to the block alone (numpy softmax over the block), and the other sequence's results
    are bit for bit those of a run where the first sequence has its prefix."""
    w = W.make("batched", 0, S=2, n_lo=500, n_hi=1500, B=8, Hq=8, Hkv=2, topk_choices=(64,))
    base = dsa_mod.DeviceWorkload(w)
    base.select()
    q, bk, bv = (x.cuda() for x in w.step_inputs(2))
    o_base = base.sparse(q, bk, bv).clone()
    w.n_ctx[0] = 0
    dw = dsa_mod.DeviceWorkload(w)
    lse = torch.empty(w.q1.shape[:3], dtype=torch.float32, device="cuda")
    dw.select(lse_out=lse)
    o = dw.sparse(q, bk, bv)
    torch.cuda.synchronize()
    assert dw.ws_sel.status() == dsa_mod.DSA_OK and dw.ws_sp.status() == dsa_mod.DSA_OK
    assert int(dw.cnt[0].abs().sum()) == 0 and bool((dw.idx[0] == -1).all())
    assert bool((dw.o_sel[0] == 0).all()) and bool(torch.isneginf(lse[0]).all())
    # the block alone
    qf, kf, vf = (x.double().cpu().numpy() for x in (w.step_inputs(2)[0][0], w.step_inputs(2)[1][0],
                                                     w.step_inputs(2)[2][0]))
    c = 1.0 / np.sqrt(w.d)
    for j in range(w.Hq):
        h = j // w.G
        x = c * qf[:, j] @ kf[:, h].T
        p = np.exp(x - x.max(axis=1, keepdims=True))
        ref = (p / p.sum(axis=1, keepdims=True)) @ vf[:, h]
        got = o[0, :, j].double().cpu().numpy()
        assert np.max(np.abs(got - ref)) <= parity.MAX_ABS
    # the other sequence is untouched
    assert torch.equal(dw.idx[1], base.idx[1]) and torch.equal(dw.o_sel[1], base.o_sel[1])
    assert torch.equal(o[1], o_base[1])
