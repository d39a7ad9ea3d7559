"""Thin ctypes binding of libdsa (include/dsa.h) with the same names.

Argument marshalling only: every step of both passes runs in the CUDA kernels
of libdsa.so.  Tensors are torch CUDA tensors; their data pointers and the
current CUDA stream are handed to the C ABI.  There is no fallback: if the
library is missing or no GPU is present, the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

DSA_OK = 0
DSA_ERR_INVALID_ARG = -1
DSA_ERR_UNSUPPORTED = -2
DSA_ERR_WORKSPACE_TOO_SMALL = -3
DSA_ERR_CUDA = -4
DSA_ERR_DEVICE_TIMEOUT = -5
DSA_ERR_BAD_INDEX = -6
DSA_ERR_NONFINITE = -7
DSA_ERR_SCRATCH_LIMIT = -8

# size of the library-held scratch array of dsa_select_static_scratch
DSA_SELECT_STATIC_SCRATCH_BYTES = 16 << 20

# every symbol include/dsa.h declares
EXPORTED = ("dsa_select", "dsa_sparse_attn", "dsa_select_workspace_size",
            "dsa_sparse_workspace_size", "dsa_workspace_init", "dsa_get_status",
            "dsa_strerror", "dsa_kernels_per_call", "dsa_select_launches", "dsa_version",
            "dsa_select_static_scratch",
            "dsa_merge_attn", "dsa_sparse_kernel")


class DsaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {strerror(code)} (code {code})")
        self.code = code


class dsa_dims(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int32), ("B", ctypes.c_int32), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32), ("page", ctypes.c_int32),
                ("max_pages", ctypes.c_int32), ("kmax", ctypes.c_int32),
                ("n_phys", ctypes.c_int64), ("page_table", ctypes.c_void_p),
                ("sm_limit", ctypes.c_int32), ("lse_out", ctypes.c_void_p),
                ("head_budget", ctypes.c_int32), ("active", ctypes.c_void_p),
                ("prefix_o_cache", ctypes.c_void_p), ("prefix_lse_cache", ctypes.c_void_p),
                ("early_gather", ctypes.c_int32)]


_lib = None


def load(path: str = LIB_PATH):
    """Load libdsa.so (raises if it has not been built); the binding's functions use
    the first library loaded."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = open_library(path)
    return _lib


def open_library(path: str):
    """A libdsa build at `path` with the C ABI's signatures declared, independent of
    the one the binding's functions use (e.g. a test build of the same sources)."""
    if not os.path.exists(path):
        raise RuntimeError(f"libdsa.so not built ({path}); run "
                           "`python -m block_sparse_attention_27_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz, ci = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    dims_p = ctypes.POINTER(dsa_dims)
    lib.dsa_select.restype = ci
    lib.dsa_select.argtypes = [vp, vp, vp, vp, ctypes.c_int32, vp, vp, vp, vp, dims_p, vp, vp, sz]
    lib.dsa_select_static_scratch.restype = ci
    lib.dsa_select_static_scratch.argtypes = [vp, vp, vp, vp, ctypes.c_int32, vp, vp, vp, vp,
                                              dims_p, vp, vp]
    lib.dsa_merge_attn.restype = ci
    lib.dsa_merge_attn.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int64, ctypes.c_int32, vp]
    lib.dsa_sparse_attn.restype = ci
    lib.dsa_sparse_attn.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, dims_p, vp, vp, vp, sz]
    lib.dsa_select_workspace_size.restype = sz
    lib.dsa_select_workspace_size.argtypes = [dims_p]
    lib.dsa_sparse_workspace_size.restype = sz
    lib.dsa_sparse_workspace_size.argtypes = [dims_p]
    lib.dsa_workspace_init.restype = ci
    lib.dsa_workspace_init.argtypes = [vp, sz, vp]
    lib.dsa_get_status.restype = ci
    lib.dsa_get_status.argtypes = [vp, vp]
    lib.dsa_strerror.restype = ctypes.c_char_p
    lib.dsa_strerror.argtypes = [ci]
    lib.dsa_version.restype = ci
    lib.dsa_version.argtypes = []
    lib.dsa_kernels_per_call.restype = ci
    lib.dsa_kernels_per_call.argtypes = [ci]
    lib.dsa_select_launches.restype = ci
    lib.dsa_select_launches.argtypes = [dims_p]
    lib.dsa_sparse_kernel.restype = ci
    lib.dsa_sparse_kernel.argtypes = [dims_p]
    return lib


def kernels_per_call(pass_: int) -> int:
    """Kernel launches per call: 0 = dsa_select (groups in one launch), 1 = dsa_sparse_attn,
    2 = dsa_merge_attn."""
    return int(load().dsa_kernels_per_call(int(pass_)))


def select_launches(dims: dsa_dims) -> int:
    """Kernel launches of one dsa_select call with these dims on the current device."""
    rc = int(load().dsa_select_launches(ctypes.byref(dims)))
    if rc < 0:
        raise DsaError(rc, "dsa_select_launches")
    return rc


def sparse_kernel(dims: dsa_dims) -> int:
    """1 = streaming sparse kernel, 1 + C = the all-keys-resident kernel in clusters of
    C CTAs, for these dims on the current device."""
    rc = int(load().dsa_sparse_kernel(ctypes.byref(dims)))
    if rc < 0:
        raise DsaError(rc, "dsa_sparse_kernel")
    return rc


def strerror(code: int) -> str:
    return load().dsa_strerror(int(code)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_dims(S, B, Hq, Hkv, d, page, max_pages, kmax, n_phys, page_table=None,
              sm_limit=0, head_budget=0, early_gather=0) -> dsa_dims:
    return dsa_dims(S, B, Hq, Hkv, d, page, max_pages, kmax, n_phys,
                    None if page_table is None else page_table.data_ptr(), int(sm_limit), None,
                    int(head_budget), None, None, None, int(early_gather))


def _with_lse(dims: dsa_dims, lse_out) -> dsa_dims:
    """dims for one call, with its optional log-sum-exp output (fp32 [S, B, Hq])."""
    if lse_out is None:
        return dims
    _check(lse_out, "lse_out", torch.float32)
    d = dsa_dims.from_buffer_copy(dims)
    d.lse_out = lse_out.data_ptr()
    return d


def dims_for(q_blk, k_cache, max_pages, kmax, page_table=None, sm_limit=0,
             head_budget=0, early_gather=0) -> dsa_dims:
    S, B, Hq, d = q_blk.shape
    n_phys, Hkv, page, d2 = k_cache.shape
    if d2 != d:
        raise ValueError("q_blk and k_cache disagree on the head dimension")
    return make_dims(S, B, Hq, Hkv, d, page, max_pages, kmax, n_phys, page_table, sm_limit,
                     head_budget, early_gather)


def _check(t, name, dtype, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")


class Workspace:
    """Device workspace for one stream of calls (zeroed header, sticky status word)."""

    def __init__(self, nbytes: int, device=None, stream=None):
        self.nbytes = int(nbytes)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device or "cuda")
        rc = load().dsa_workspace_init(_ptr(self.buf), self.nbytes, _stream(stream))
        if rc != DSA_OK:
            raise DsaError(rc, "dsa_workspace_init")

    def status(self, stream=None) -> int:
        return int(load().dsa_get_status(_ptr(self.buf), _stream(stream)))


def select_workspace_size(dims: dsa_dims) -> int:
    return int(load().dsa_select_workspace_size(ctypes.byref(dims)))


def sparse_workspace_size(dims: dsa_dims) -> int:
    return int(load().dsa_sparse_workspace_size(ctypes.byref(dims)))


def dsa_select(q_blk, k_cache, v_cache, n_ctx, page, topk, idx_out, o_out, stream=None, *,
               dims: dsa_dims, cnt_out, workspace: Workspace, lse_out=None):
    """Selection pass (see include/dsa.h).  All tensors on the GPU; raises DsaError."""
    _check(q_blk, "q_blk", torch.bfloat16, 4)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(n_ctx, "n_ctx", torch.int32)
    _check(topk, "topk", torch.int32)
    _check(idx_out, "idx_out", torch.int32)
    _check(o_out, "o_out", torch.bfloat16)
    _check(cnt_out, "cnt_out", torch.int32)
    dims = _with_lse(dims, lse_out)
    rc = load().dsa_select(_ptr(q_blk), _ptr(k_cache), _ptr(v_cache), _ptr(n_ctx), int(page),
                           _ptr(topk), _ptr(idx_out), _ptr(o_out), _stream(stream),
                           ctypes.byref(dims), _ptr(cnt_out), _ptr(workspace.buf), workspace.nbytes)
    if rc != DSA_OK:
        raise DsaError(rc, "dsa_select")


def dsa_select_static_scratch(q_blk, k_cache, v_cache, n_ctx, page, topk, idx_out, o_out,
                              stream=None, *, dims: dsa_dims, cnt_out, status):
    """Selection pass with the library's static scratch instead of a workspace (see
    include/dsa.h).  `status` is a device int32/uint32 tensor of one element that
    holds 0 before the first call; read it with status_word().  Raises DsaError."""
    _check(q_blk, "q_blk", torch.bfloat16, 4)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(n_ctx, "n_ctx", torch.int32)
    _check(topk, "topk", torch.int32)
    _check(idx_out, "idx_out", torch.int32)
    _check(o_out, "o_out", torch.bfloat16)
    _check(cnt_out, "cnt_out", torch.int32)
    if status.dtype == torch.uint32:  # the same 4-byte word either way
        status = status.view(torch.int32)
    _check(status, "status", torch.int32)
    rc = load().dsa_select_static_scratch(_ptr(q_blk), _ptr(k_cache), _ptr(v_cache), _ptr(n_ctx),
                                          int(page), _ptr(topk), _ptr(idx_out), _ptr(o_out),
                                          _stream(stream), ctypes.byref(dims), _ptr(cnt_out),
                                          _ptr(status))
    if rc != DSA_OK:
        raise DsaError(rc, "dsa_select_static_scratch")


def status_word(status, stream=None) -> int:
    """dsa_get_status() of a caller-owned status word (synchronises `stream`)."""
    return int(load().dsa_get_status(_ptr(status), _stream(stream)))


def dsa_sparse_attn(q_blk, k_cache, v_cache, idx, blk_k, blk_v, o_out, stream=None, *,
                    dims: dsa_dims, n_ctx, idx_cnt, workspace: Workspace, lse_out=None,
                    active=None, prefix_o_cache=None, prefix_lse_cache=None):
    """Sparse pass (see include/dsa.h).  All tensors on the GPU; raises DsaError.
    active (uint8 [S, B]) with prefix_o_cache (bf16 [S, B, Hq, d]) and prefix_lse_cache
    (fp32 [S, B, Hq]): reuse of the prefix part for stable tokens."""
    _check(q_blk, "q_blk", torch.bfloat16, 4)
    _check(k_cache, "k_cache", torch.bfloat16, 4)
    _check(v_cache, "v_cache", torch.bfloat16, 4)
    _check(idx, "idx", torch.int32)
    _check(blk_k, "blk_k", torch.bfloat16, 4)
    _check(blk_v, "blk_v", torch.bfloat16, 4)
    _check(o_out, "o_out", torch.bfloat16)
    _check(n_ctx, "n_ctx", torch.int32)
    _check(idx_cnt, "idx_cnt", torch.int32)
    dims = _with_lse(dims, lse_out)
    if active is not None:
        _check(active, "active", torch.uint8)
        _check(prefix_o_cache, "prefix_o_cache", torch.bfloat16)
        _check(prefix_lse_cache, "prefix_lse_cache", torch.float32)
        dims = dsa_dims.from_buffer_copy(dims)
        dims.active = active.data_ptr()
        dims.prefix_o_cache = prefix_o_cache.data_ptr()
        dims.prefix_lse_cache = prefix_lse_cache.data_ptr()
    rc = load().dsa_sparse_attn(_ptr(q_blk), _ptr(k_cache), _ptr(v_cache), _ptr(idx), _ptr(blk_k),
                                _ptr(blk_v), _ptr(o_out), _stream(stream), ctypes.byref(dims),
                                _ptr(n_ctx), _ptr(idx_cnt), _ptr(workspace.buf), workspace.nbytes)
    if rc != DSA_OK:
        raise DsaError(rc, "dsa_sparse_attn")


def dsa_merge_attn(o_a, lse_a, o_b, lse_b, o_out, lse_out=None, stream=None):
    """Merge of two attention results over disjoint key sets (see include/dsa.h).
    o_*: bf16 [..., d] with the same leading shape; lse_*: fp32 over the leading shape."""
    for t, n in ((o_a, "o_a"), (o_b, "o_b"), (o_out, "o_out")):
        _check(t, n, torch.bfloat16)
    for t, n in ((lse_a, "lse_a"), (lse_b, "lse_b")):
        _check(t, n, torch.float32)
    if lse_out is not None:
        _check(lse_out, "lse_out", torch.float32)
    d = o_a.shape[-1]
    rows = o_a.numel() // d
    if o_b.shape != o_a.shape or o_out.shape != o_a.shape or lse_a.numel() != rows or lse_b.numel() != rows:
        raise ValueError("dsa_merge_attn: shapes disagree")
    rc = load().dsa_merge_attn(_ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b), _ptr(o_out),
                               _ptr(lse_out), rows, d, _stream(stream))
    if rc != DSA_OK:
        raise DsaError(rc, "dsa_merge_attn")


class DeviceWorkload:
    """A workload's tensors on the GPU plus the dims, outputs and workspaces of both passes."""

    def __init__(self, w, device="cuda", sm_limit=0, head_budget=0, early_gather=0):
        """head_budget=1: one budget of Hkv*kp pages per sequence shared by its KV heads;
        idx rows then hold up to min(max_pages, Hkv*kp) pages.  early_gather=1: sparse steps
        gather their pages before waiting for the kernel ahead of them (include/dsa.h)."""
        self.w = w
        dev = torch.device(device)
        self.q1 = w.q1.to(dev)
        self.k_cache = w.k_cache.to(dev)
        self.v_cache = w.v_cache.to(dev)
        self.blk_k1 = w.blk_k1.to(dev)
        self.blk_v1 = w.blk_v1.to(dev)
        self.n_ctx = w.n_ctx.to(dev)
        self.topk = w.topk.to(dev)
        self.page_table = None if w.page_table is None else w.page_table.to(dev)
        kmax = min(w.max_pages, w.Hkv * w.kmax) if head_budget else w.kmax
        self.kmax = kmax
        self.dims = dims_for(self.q1, self.k_cache, w.max_pages, kmax, self.page_table, sm_limit,
                             head_budget, early_gather)
        S, Hkv = w.S, w.Hkv
        self.idx = torch.full((S, Hkv, kmax), -1, dtype=torch.int32, device=dev)
        self.cnt = torch.zeros((S, Hkv), dtype=torch.int32, device=dev)
        self.o_sel = torch.zeros_like(self.q1)
        self.o_sp = torch.zeros_like(self.q1)
        self.ws_sel = Workspace(select_workspace_size(self.dims), dev)
        self.ws_sp = Workspace(sparse_workspace_size(self.dims), dev)

    def select(self, q=None, stream=None, lse_out=None):
        dsa_select(self.q1 if q is None else q, self.k_cache, self.v_cache, self.n_ctx,
                   self.w.P, self.topk, self.idx, self.o_sel, stream, dims=self.dims,
                   cnt_out=self.cnt, workspace=self.ws_sel, lse_out=lse_out)
        return self.idx, self.cnt, self.o_sel

    def sparse(self, q, blk_k, blk_v, idx=None, cnt=None, stream=None, out=None, lse_out=None,
               active=None, cache=None):
        """cache = (prefix_o_cache, prefix_lse_cache), used with `active`."""
        o = self.o_sp if out is None else out
        dsa_sparse_attn(q, self.k_cache, self.v_cache, self.idx if idx is None else idx, blk_k,
                        blk_v, o, stream, dims=self.dims, n_ctx=self.n_ctx,
                        idx_cnt=self.cnt if cnt is None else cnt, workspace=self.ws_sp,
                        lse_out=lse_out, active=active,
                        prefix_o_cache=None if cache is None else cache[0],
                        prefix_lse_cache=None if cache is None else cache[1])
        return o
