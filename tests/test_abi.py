"""The C-ABI library loads, exports every symbol include/dsa.h declares, and rejects
bad arguments on the host before touching a GPU (runs without a GPU)."""
import ctypes
import os
import re

import pytest
import torch

from block_sparse_attention_27_b200 import build as B
from block_sparse_attention_27_b200 import dsa

HEADER = os.path.join(B.ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return dsa.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(dsa.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_strerror_and_version(lib):
    assert lib.dsa_version() >= 100
    assert dsa.kernels_per_call(0) >= 1 and dsa.kernels_per_call(1) >= 1
    assert lib.dsa_kernels_per_call(7) == dsa.DSA_ERR_INVALID_ARG
    for code in range(0, -8, -1):
        assert dsa.strerror(code) and "unknown" not in dsa.strerror(code)
    assert "unknown" in dsa.strerror(-99)


def good_dims(**kw):
    base = dict(S=1, B=32, Hq=32, Hkv=8, d=128, page=16, max_pages=512, kmax=32, n_phys=512)
    base.update(kw)
    return dsa.make_dims(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=30), dsa.DSA_ERR_INVALID_ARG),      # Hq % Hkv != 0
    (dict(d=96), dsa.DSA_ERR_UNSUPPORTED),
    (dict(page=8), dsa.DSA_ERR_UNSUPPORTED),
    (dict(B=65, Hq=32, Hkv=8), dsa.DSA_ERR_UNSUPPORTED),  # B*G = 260 > 256
    (dict(kmax=0), dsa.DSA_ERR_INVALID_ARG),
    (dict(S=0), dsa.DSA_ERR_INVALID_ARG),
    (dict(head_budget=2), dsa.DSA_ERR_INVALID_ARG),
    (dict(head_budget=1, Hq=128, Hkv=128, B=1), dsa.DSA_ERR_UNSUPPORTED),  # more KV heads than supported
])
def test_bad_dims_rejected_on_host(lib, kw, code):
    dims = good_dims(**kw)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    rc = lib.dsa_select(fake, fake, fake, fake, dims.page, fake, fake, fake, None,
                        ctypes.byref(dims), fake, fake, 1 << 30)
    assert rc == code
    assert lib.dsa_select_workspace_size(ctypes.byref(dims)) == 0


def test_null_and_misaligned_pointers_rejected(lib):
    dims = good_dims()
    ok = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 2)
    rc = lib.dsa_select(None, ok, ok, ok, 16, ok, ok, ok, None, ctypes.byref(dims), ok, ok, 1 << 30)
    assert rc == dsa.DSA_ERR_INVALID_ARG
    rc = lib.dsa_select(bad, ok, ok, ok, 16, ok, ok, ok, None, ctypes.byref(dims), ok, ok, 1 << 30)
    assert rc == dsa.DSA_ERR_INVALID_ARG
    rc = lib.dsa_select(ok, ok, ok, ok, 32, ok, ok, ok, None, ctypes.byref(dims), ok, ok, 1 << 30)
    assert rc == dsa.DSA_ERR_INVALID_ARG  # page argument disagrees with dims
    rc = lib.dsa_sparse_attn(ok, ok, ok, ok, ok, bad, ok, None, ctypes.byref(dims), ok, ok, ok,
                             1 << 30)
    assert rc == dsa.DSA_ERR_INVALID_ARG


def test_workspace_too_small_rejected(lib):
    dims = good_dims()
    ok = ctypes.c_void_p(1 << 20)
    need = lib.dsa_sparse_workspace_size(ctypes.byref(dims))
    assert need >= 4096  # at least the status header
    rc = lib.dsa_sparse_attn(ok, ok, ok, ok, ok, ok, ok, None, ctypes.byref(dims), ok, ok, ok,
                             need - 1)
    assert rc == dsa.DSA_ERR_WORKSPACE_TOO_SMALL
    need = lib.dsa_select_workspace_size(ctypes.byref(dims))
    rc = lib.dsa_select(ok, ok, ok, ok, 16, ok, ok, ok, None, ctypes.byref(dims), ok, ok, need - 1)
    assert rc == dsa.DSA_ERR_WORKSPACE_TOO_SMALL


def test_library_has_no_oracle_dependency():
    """The product library is built from csrc/ only and never references the oracle."""
    for src in os.listdir(os.path.join(B.PKG, "csrc")):
        text = open(os.path.join(B.PKG, "csrc", src)).read()
        assert "oracle" not in text.lower(), src
    for py in ("dsa.py", "build.py", "__init__.py"):
        text = open(os.path.join(B.PKG, py)).read()
        assert "import oracle" not in text and "from oracle" not in text


def test_static_scratch_entry_checks_on_host(lib):
    """dsa_select_static_scratch: arguments checked like dsa_select, a status word is
    required, and shapes beyond the static array are refused before any launch."""
    ok = ctypes.c_void_p(1 << 20)
    dims = good_dims()
    rc = lib.dsa_select_static_scratch(ok, ok, ok, ok, 16, ok, ok, ok, None, ctypes.byref(dims),
                                       ok, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG
    rc = lib.dsa_select_static_scratch(ok, ok, ok, ok, 16, ok, ok, ok, None, ctypes.byref(dims),
                                       ok, ctypes.c_void_p((1 << 20) + 2))
    assert rc == dsa.DSA_ERR_INVALID_ARG
    big = good_dims(max_pages=8192, n_phys=8192, kmax=64)      # 128K prefix, 8 KV heads
    assert lib.dsa_select_workspace_size(ctypes.byref(big)) > dsa.DSA_SELECT_STATIC_SCRATCH_BYTES
    rc = lib.dsa_select_static_scratch(ok, ok, ok, ok, 16, ok, ok, ok, None, ctypes.byref(big),
                                       ok, ok)
    assert rc == dsa.DSA_ERR_SCRATCH_LIMIT
    assert "static" in dsa.strerror(dsa.DSA_ERR_SCRATCH_LIMIT)


def test_merge_entry_checks_on_host(lib):
    ok = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 2)
    assert lib.dsa_merge_attn(ok, ok, ok, ok, ok, None, 0, 128, None) == dsa.DSA_OK  # nothing to do
    assert lib.dsa_merge_attn(None, ok, ok, ok, ok, None, 4, 128, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_merge_attn(ok, ok, ok, ok, ok, None, 4, 12, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_merge_attn(ok, ok, bad, ok, ok, None, 4, 128, None) == dsa.DSA_ERR_INVALID_ARG
    assert dsa.kernels_per_call(2) == 1


def test_select_launches(lib):
    """The selection pass runs its (sequence, KV head) groups in co-resident
    launches: one for the bench shape, more when the groups outnumber the SMs
    (148 assumed without a GPU)."""
    if torch.cuda.is_available():
        pytest.skip("launch counts below assume 148 SMs")
    assert dsa.select_launches(good_dims()) == 1
    assert dsa.select_launches(good_dims(sm_limit=37)) == 1
    # 512 groups of one CTA: 148 per launch
    assert dsa.select_launches(good_dims(S=64)) == 4
    # 224 query rows per KV head: two 128-row tiles per group, 74 groups per launch
    assert dsa.select_launches(good_dims(S=100, Hq=28, Hkv=4)) == 6
    # the head-adaptive budget adds its per-sequence selection kernel
    assert dsa.select_launches(good_dims(head_budget=1)) == 2
    assert dsa.select_launches(good_dims(S=64, head_budget=1)) == 5
    with pytest.raises(dsa.DsaError):
        dsa.select_launches(good_dims(d=96))


def test_prefix_reuse_needs_both_caches(lib):
    """dims.active without the two prefix caches (or with a misaligned one) is rejected
    on the host, before anything is launched."""
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    for o_cache, lse_cache in ((None, None), (1 << 20, None), ((1 << 20) + 8, 1 << 20)):
        dims = good_dims()
        dims.active = 1 << 20
        dims.prefix_o_cache = o_cache
        dims.prefix_lse_cache = lse_cache
        rc = lib.dsa_sparse_attn(fake, fake, fake, fake, fake, fake, fake, None, ctypes.byref(dims),
                                 fake, fake, fake, 1 << 30)
        assert rc == dsa.DSA_ERR_INVALID_ARG
