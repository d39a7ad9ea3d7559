"""fp64 CPU oracle for shared-index top-k sparse KV attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It never touches the CUDA library and the
CUDA library never touches it; the two meet only through the seeded inputs of
``block_sparse_attention_27_b200.workloads``.

The arithmetic lives in ``oracle.c`` (plain C, double precision, OpenMP over
(sequence, KV head)); this module compiles it with gcc and marshals numpy arrays
through ctypes.  See ``oracle.c`` for what each function computes and which page
and section it follows.  ``Oracle(path)`` binds any build of that source (the
planted-mistake tests build altered copies); the module-level functions use the
default build.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")

ORACLE_OK, ORACLE_EINVAL, ORACLE_EPAGE, ORACLE_EINDEX, ORACLE_ENOMEM = 0, -1, -2, -3, -4


class OracleError(RuntimeError):
    pass


def compile_source(src: str, out: str) -> str:
    """Compile one C source of the oracle into a shared library (gcc, -O2, OpenMP)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile oracle.c into _build/liboracle.so unless it is up to date."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(SOURCE):
        return _LIB
    return compile_source(SOURCE, _LIB)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected bf16 bits as uint16, got {a.dtype}")
    return a


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a, ctype):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctype))


@dataclass
class SelectResult:
    idx: np.ndarray     # [S, Hkv, kmax] int32, ascending, -1 padded
    cnt: np.ndarray     # [S, Hkv] int32
    o: np.ndarray       # [S, B, Hq, d] float64, prefix-only output
    lse: np.ndarray     # [S, B, Hq] float64
    score: np.ndarray   # [S, Hkv, max_pages] float64
    mass: np.ndarray | None  # [S, Hkv, max_pages*P] float64


class Oracle:
    """ctypes binding of one build of oracle.c."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        i32p = ctypes.POINTER(ctypes.c_int32)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f64p = ctypes.POINTER(ctypes.c_double)
        ci, cl = ctypes.c_int, ctypes.c_long
        lib.oracle_select.restype = ci
        lib.oracle_select.argtypes = [u16p, u16p, u16p, i32p, i32p, i32p,
                                      ci, ci, ci, ci, ci, ci, ci, cl, ci,
                                      i32p, i32p, f64p, f64p, f64p, f64p]
        lib.oracle_sparse.restype = ci
        lib.oracle_sparse.argtypes = [u16p, u16p, u16p, i32p, i32p, i32p, i32p, ci, u16p, u16p,
                                      ci, ci, ci, ci, ci, ci, ci, cl, f64p, f64p]
        lib.oracle_select_global.restype = ci
        lib.oracle_select_global.argtypes = [f64p, i32p, i32p, ci, ci, ci, ci, ci, i32p, i32p]
        u8p = ctypes.POINTER(ctypes.c_uint8)
        lib.oracle_sparse_losa.restype = ci
        lib.oracle_sparse_losa.argtypes = [u16p, u16p, u16p, i32p, i32p, i32p, i32p, ci, u16p, u16p,
                                           u8p, u16p, f64p, ci, ci, ci, ci, ci, ci, ci, cl,
                                           f64p, f64p, f64p, f64p]
        lib.oracle_num_threads.restype = ci
        lib.oracle_num_threads.argtypes = []
        self.lib = lib
        self.path = path

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    @staticmethod
    def _max_pages(n_ctx, P, page_table, max_pages):
        if max_pages is not None:
            return int(max_pages)
        if page_table is not None:
            return int(page_table.shape[1])
        return int(np.max((n_ctx + P - 1) // P))

    def select(self, q, k, v, n_ctx, topk, *, page_table=None, max_pages=None, kmax=None,
               want_mass=False) -> SelectResult:
        """Selection pass.  q,k,v are bf16 bit patterns (uint16); topk is in tokens."""
        q, k, v = _u16(q), _u16(k), _u16(v)
        S, B, Hq, d = q.shape
        n_phys, Hkv, P, _ = k.shape
        n_ctx = _i32(n_ctx).reshape(S)
        topk = _i32(topk).reshape(S)
        max_pages = self._max_pages(n_ctx, P, page_table, max_pages)
        kmax = int(np.max(topk)) // P if kmax is None else int(kmax)
        pt = _i32(page_table) if page_table is not None else None
        idx = np.empty((S, Hkv, kmax), np.int32)
        cnt = np.empty((S, Hkv), np.int32)
        o = np.empty((S, B, Hq, d), np.float64)
        lse = np.empty((S, B, Hq), np.float64)
        score = np.empty((S, Hkv, max_pages), np.float64)
        mass = np.empty((S, Hkv, max_pages * P), np.float64) if want_mass else None
        I, F, U = ctypes.c_int32, ctypes.c_double, ctypes.c_uint16
        rc = self.lib.oracle_select(
            _p(q, U), _p(k, U), _p(v, U), _p(pt, I), _p(n_ctx, I), _p(topk, I),
            S, B, Hq, Hkv, d, P, max_pages, n_phys, kmax,
            _p(idx, I), _p(cnt, I), _p(o, F), _p(lse, F), _p(score, F), _p(mass, F))
        if rc != ORACLE_OK:
            raise OracleError(f"oracle_select failed with status {rc}")
        return SelectResult(idx, cnt, o, lse, score, mass)

    def select_global(self, q, k, v, n_ctx, topk, *, kmax, page_table=None, max_pages=None,
                      score=None) -> SelectResult:
        """Selection pass with the head-adaptive budget: one budget of Hkv * topk/P pages
        per sequence shared by its KV heads (see oracle_select_global).  The page scores
        and the prefix output are those of select(); `score` ([S, Hkv, max_pages]
        float64) skips recomputing them."""
        n_ctx_a = _i32(n_ctx).reshape(-1)
        topk_a = _i32(topk).reshape(-1)
        S = n_ctx_a.shape[0]
        Hkv, P = _u16(k).shape[1], _u16(k).shape[2]
        max_pages = self._max_pages(n_ctx_a, P, page_table, max_pages)
        base = None
        if score is None:
            base = self.select(q, k, v, n_ctx, topk, page_table=page_table, max_pages=max_pages)
            score = base.score
        score = np.ascontiguousarray(score, dtype=np.float64)
        idx = np.empty((S, Hkv, int(kmax)), np.int32)
        cnt = np.empty((S, Hkv), np.int32)
        I, F = ctypes.c_int32, ctypes.c_double
        rc = self.lib.oracle_select_global(_p(score, F), _p(n_ctx_a, I), _p(topk_a, I), S, Hkv, P,
                                           max_pages, int(kmax), _p(idx, I), _p(cnt, I))
        if rc != ORACLE_OK:
            raise OracleError(f"oracle_select_global failed with status {rc}")
        if base is None:
            return SelectResult(idx, cnt, None, None, score, None)
        return SelectResult(idx, cnt, base.o, base.lse, score, base.mass)

    def sparse(self, q, k, v, n_ctx, idx, cnt, blk_k, blk_v, *, page_table=None,
               max_pages=None):
        """Sparse pass; returns (o [S,B,Hq,d] float64, lse [S,B,Hq] float64)."""
        q, k, v = _u16(q), _u16(k), _u16(v)
        blk_k, blk_v = _u16(blk_k), _u16(blk_v)
        S, B, Hq, d = q.shape
        n_phys, Hkv, P, _ = k.shape
        n_ctx = _i32(n_ctx).reshape(S)
        max_pages = self._max_pages(n_ctx, P, page_table, max_pages)
        idx = _i32(idx)
        cnt = _i32(cnt).reshape(S, Hkv)
        kmax = idx.shape[-1]
        pt = _i32(page_table) if page_table is not None else None
        o = np.empty((S, B, Hq, d), np.float64)
        lse = np.empty((S, B, Hq), np.float64)
        I, F, U = ctypes.c_int32, ctypes.c_double, ctypes.c_uint16
        rc = self.lib.oracle_sparse(
            _p(q, U), _p(k, U), _p(v, U), _p(pt, I), _p(n_ctx, I), _p(idx, I), _p(cnt, I),
            kmax, _p(blk_k, U), _p(blk_v, U), S, B, Hq, Hkv, d, P, max_pages, n_phys,
            _p(o, F), _p(lse, F))
        if rc != ORACLE_OK:
            raise OracleError(f"oracle_sparse failed with status {rc}")
        return o, lse


    def sparse_losa(self, q, k, v, n_ctx, idx, cnt, blk_k, blk_v, active, cache_o, cache_lse, *,
              page_table=None, max_pages=None):
        """Sparse pass reusing the prefix part of stable tokens (see oracle_sparse_losa).
        active [S, B] bool; cache_o [S, B, Hq, d] bf16 bits; cache_lse [S, B, Hq] (natural log).
        Returns (o, lse, cache_o_new, cache_lse_new), all float64."""
        q, k, v = _u16(q), _u16(k), _u16(v)
        blk_k, blk_v = _u16(blk_k), _u16(blk_v)
        S, B, Hq, d = q.shape
        n_phys, Hkv, P, _ = k.shape
        n_ctx = _i32(n_ctx).reshape(S)
        max_pages = self._max_pages(n_ctx, P, page_table, max_pages)
        idx = _i32(idx)
        cnt = _i32(cnt).reshape(S, Hkv)
        kmax = idx.shape[-1]
        pt = _i32(page_table) if page_table is not None else None
        act = np.ascontiguousarray(np.asarray(active).reshape(S, B).astype(np.uint8))
        co = _u16(cache_o)
        cl = np.ascontiguousarray(np.asarray(cache_lse, dtype=np.float64).reshape(S, B, Hq))
        o = np.empty((S, B, Hq, d), np.float64)
        lse = np.empty((S, B, Hq), np.float64)
        co_new = np.empty((S, B, Hq, d), np.float64)
        cl_new = np.empty((S, B, Hq), np.float64)
        I, F, U, U8 = ctypes.c_int32, ctypes.c_double, ctypes.c_uint16, ctypes.c_uint8
        rc = self.lib.oracle_sparse_losa(
            _p(q, U), _p(k, U), _p(v, U), _p(pt, I), _p(n_ctx, I), _p(idx, I), _p(cnt, I), kmax,
            _p(blk_k, U), _p(blk_v, U), _p(act, U8), _p(co, U), _p(cl, F), S, B, Hq, Hkv, d, P,
            max_pages, n_phys, _p(o, F), _p(lse, F), _p(co_new, F), _p(cl_new, F))
        if rc != ORACLE_OK:
            raise OracleError(f"oracle_sparse_losa failed with status {rc}")
        return o, lse, co_new, cl_new


_default: Oracle | None = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def num_threads() -> int:
    return default().num_threads()


def select(*args, **kwargs) -> SelectResult:
    return default().select(*args, **kwargs)


def sparse(*args, **kwargs):
    return default().sparse(*args, **kwargs)


def select_global(*args, **kwargs) -> SelectResult:
    return default().select_global(*args, **kwargs)


def sparse_losa(*args, **kwargs):
    return default().sparse_losa(*args, **kwargs)


def all_pages(n_ctx, P, Hkv, kmax=None):
    """idx/cnt that select every page of every sequence (dense mode)."""
    n_ctx = np.asarray(n_ctx).reshape(-1)
    nps = (n_ctx + P - 1) // P
    kmax = int(nps.max()) if kmax is None else kmax
    S = n_ctx.shape[0]
    idx = np.full((S, Hkv, kmax), -1, np.int32)
    cnt = np.zeros((S, Hkv), np.int32)
    for s in range(S):
        idx[s, :, : nps[s]] = np.arange(nps[s], dtype=np.int32)
        cnt[s, :] = nps[s]
    return idx, cnt
