"""A device wait that runs out is reported, not hung, and leaves the library usable.

A test build of the library (-DDSA_TEST_TIMEOUT) shortens every bounded wait to
50 ms and makes the selection pass's group wait ask for one arrival more than a
group has, so that this wait, and only this one, runs out on every call.  Nothing
else changes: the GPU keeps answering, the call finishes, and the status word
carries the timeout with the site of the first wait that gave up."""
import ctypes
import os

import numpy as np
import pytest
import torch

import oracle
import parity
from block_sparse_attention_27_b200 import build, dsa, workloads as W

pytestmark = pytest.mark.gpu

TIMEOUT_LIB = os.path.join(os.path.dirname(build.LIB), "libdsa_timeout.so")


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    build.build()
    dsa.load()
    if not os.path.exists(TIMEOUT_LIB) or not build.up_to_date_at(TIMEOUT_LIB):
        build.build(defines=("DSA_TEST_TIMEOUT",), out=TIMEOUT_LIB)
    return dsa.open_library(TIMEOUT_LIB)


def _select(lib, dw, ws):
    w = dw.w
    rc = lib.dsa_select(dsa._ptr(dw.q1), dsa._ptr(dw.k_cache), dsa._ptr(dw.v_cache),
                        dsa._ptr(dw.n_ctx), w.P, dsa._ptr(dw.topk), dsa._ptr(dw.idx),
                        dsa._ptr(dw.o_sel), dsa._stream(None), ctypes.byref(dw.dims),
                        dsa._ptr(dw.cnt), dsa._ptr(ws.buf), ws.nbytes)
    assert rc == dsa.DSA_OK


def test_group_wait_timeout_reported_and_recovered(libs):
    w = W.make("tiny", 0)
    dw = dsa.DeviceWorkload(w)
    ws = dw.ws_sel
    dw.o_sel.fill_(float("nan"))
    _select(libs, dw, ws)
    torch.cuda.synchronize()
    assert libs.dsa_get_status(dsa._ptr(ws.buf), dsa._stream(None)) == dsa.DSA_ERR_DEVICE_TIMEOUT
    word = int(ws.buf[:4].view(torch.int32).item()) & 0xffffffff
    assert (word >> 16) & 0xff == 0xff          # site: the group wait of the selection pass
    # every partial was written before the wait gave up, so the pass still
    # finished with finite outputs, and the group counters are back at zero
    assert torch.isfinite(dw.o_sel.float()).all()
    counters = ws.buf[256:4096].view(torch.int32)
    assert int(counters.abs().sum().item()) == 0
    # the same workspace, its status cleared, serves a normal call of the library
    rc = dsa.load().dsa_workspace_init(dsa._ptr(ws.buf), ws.nbytes, dsa._stream(None))
    assert rc == dsa.DSA_OK
    dw.select()
    torch.cuda.synchronize()
    assert ws.status() == dsa.DSA_OK
    ref = oracle.select(W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                        w.topk.numpy(), max_pages=w.max_pages)
    parity.check_selection(dw.idx.cpu().numpy(), dw.cnt.cpu().numpy(), ref,
                           [w.n_pages(s) for s in range(w.S)],
                           [int(w.topk[s]) // w.P for s in range(w.S)])
    parity.check_output(dw.o_sel, ref.o, "selection after a timed-out call")
