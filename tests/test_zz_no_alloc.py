"""dsa_select_static_scratch (selection pass on the library's static scratch array)
against dsa_select with a caller workspace, on the same inputs and stream.

Collected last on purpose: it must also pass after every other GPU test has run
in the same process (same module, same static array)."""
import pytest
import torch

from block_sparse_attention_27_b200 import dsa, workloads as W
from parity import MAX_ABS, MEAN_ABS

pytestmark = pytest.mark.gpu


def _static_select(dw, q, status):
    w = dw.w
    idx = torch.full_like(dw.idx, -7)
    cnt = torch.full_like(dw.cnt, -7)
    o = torch.full_like(dw.o_sel, float("nan"))
    dsa.dsa_select_static_scratch(q, dw.k_cache, dw.v_cache, dw.n_ctx, w.P, dw.topk, idx, o,
                                  dims=dw.dims, cnt_out=cnt, status=status)
    return idx, cnt, o


def _compare(dw, got, want):
    idx, cnt, o = got
    widx, wcnt, wo = want
    assert torch.equal(cnt, wcnt)
    assert torch.equal(idx, widx)
    err = (o.float() - wo.float()).abs()
    assert torch.isfinite(o.float()).all()
    assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS


@pytest.mark.parametrize("names", [("tiny", "8k"), ("32k", "tiny")])
def test_static_scratch_matches_workspace_path(names):
    """Two calls in a row (different shapes, so the second reuses the array that the
    first wrote), each equal to dsa_select run on the same inputs."""
    torch.cuda.init()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for name in names:
        dw = dsa.DeviceWorkload(W.make(name, 0))
        assert dsa.select_workspace_size(dw.dims) <= dsa.DSA_SELECT_STATIC_SCRATCH_BYTES
        q2 = dw.w.step_inputs(2)[0].cuda()
        for q in (dw.q1, q2):
            want = tuple(t.clone() for t in dw.select(q))
            got = _static_select(dw, q, status)
            torch.cuda.synchronize()
            _compare(dw, got, want)
        assert dw.ws_sel.status() == dsa.DSA_OK
    assert dsa.status_word(status) == dsa.DSA_OK
    assert int(status.item()) == 0


@pytest.mark.parametrize("kw", [dict(head_budget=1), dict(sm_limit=4)],
                         ids=["head_budget", "sm_limit"])
def test_static_scratch_variants(kw):
    """The head-adaptive budget (whose second kernel reads the page scores from the
    array) and a pass held to 4 SMs (two selection launches reusing the group
    counters of one call), each twice in a row, equal to dsa_select."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dw = dsa.DeviceWorkload(W.make("8k", 0), **kw)
    assert dsa.select_workspace_size(dw.dims) <= dsa.DSA_SELECT_STATIC_SCRATCH_BYTES
    q2 = dw.w.step_inputs(2)[0].cuda()
    for q in (dw.q1, q2, dw.q1):
        want = tuple(t.clone() for t in dw.select(q))
        got = _static_select(dw, q, status)
        torch.cuda.synchronize()
        _compare(dw, got, want)
    assert dw.ws_sel.status() == dsa.DSA_OK
    assert dsa.status_word(status) == dsa.DSA_OK


def test_static_scratch_reports_through_status_word():
    """A bad page-table entry is reported in the caller's status word, sticky, and
    cleared by writing 0."""
    w = W.make("tiny", 0)
    dw = dsa.DeviceWorkload(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    table = torch.arange(w.max_pages, dtype=torch.int32, device="cuda").reshape(1, -1)
    table[0, 3] = w.n_phys + 5          # outside the cache: skipped, reported
    dims = dsa.dims_for(dw.q1, dw.k_cache, w.max_pages, w.kmax, table)
    idx, cnt = torch.empty_like(dw.idx), torch.empty_like(dw.cnt)
    o = torch.empty_like(dw.o_sel)
    dsa.dsa_select_static_scratch(dw.q1, dw.k_cache, dw.v_cache, dw.n_ctx, w.P, dw.topk, idx, o,
                                  dims=dims, cnt_out=cnt, status=status)
    assert dsa.status_word(status) == dsa.DSA_ERR_BAD_INDEX
    status.zero_()
    _static_select(dw, dw.q1, status)
    assert dsa.status_word(status) == dsa.DSA_OK


def test_static_scratch_refuses_large_shapes():
    dims = dsa.make_dims(1, 32, 32, 8, 128, 16, 8192, 64, 8192)   # 128K prefix, 8 KV heads
    assert dsa.select_workspace_size(dims) > dsa.DSA_SELECT_STATIC_SCRATCH_BYTES
    dev = "cuda"
    q = torch.zeros((1, 32, 32, 128), dtype=torch.bfloat16, device=dev)
    kv = torch.zeros((16, 8, 16, 128), dtype=torch.bfloat16, device=dev)
    i32 = lambda *s: torch.zeros(s, dtype=torch.int32, device=dev)
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_select_static_scratch(q, kv, kv, i32(1), 16, i32(1), i32(1, 8, 64), q,
                                      dims=dims, cnt_out=i32(1, 8), status=i32(1))
    assert e.value.code == dsa.DSA_ERR_SCRATCH_LIMIT
