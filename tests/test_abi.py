"""The C-ABI library: it loads, exports every entry point the header declares,
and rejects bad arguments on the host before touching the GPU (no compute
call runs here; these tests need no GPU)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import structured_sparse_attention_fibonacci_b200 as sa
from structured_sparse_attention_fibonacci_b200 import build as sa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    sa_build.build()
    return sa.lib()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(sparse_attn_\w+)\s*\(", text):
            names.add(m.group(1))
    return names


def test_header_declares_the_boundary():
    names = declared_functions()
    assert {"sparse_attn_fwd", "sparse_attn_bwd", "sparse_attn_workspace_size",
            "sparse_attn_status_string"} <= names


@pytest.mark.parametrize("path", [sa.LIB_PATH, sa.BOUNDS_LIB_PATH], ids=["library", "bounds"])
def test_every_declared_symbol_is_exported(lib, path):
    """Both builds (the library and its bounds-checking variant) export every
    function the header declares."""
    out = subprocess.check_output(["nm", "-D", "--defined-only", path]).decode()
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = declared_functions() - exported
    assert not missing, missing
    other = ctypes.CDLL(path)
    for name in declared_functions():
        assert getattr(lib, name) is not None
        assert getattr(other, name) is not None


def test_binding_lists_every_export():
    assert declared_functions() <= set(sa.EXPORTED)


def test_status_strings(lib):
    assert sa.status_string(sa.SA_OK) == "ok"
    assert "invalid" in sa.status_string(sa.SA_ERR_INVALID_ARG)
    assert "workspace" in sa.status_string(sa.SA_ERR_WORKSPACE)
    assert sa.status_string(99) == "unknown status"


def _p(**kw):
    base = dict(window=12, offsets=sa.FIB15, sinks=0)
    base.update(kw)
    shape = base.pop("shape", (16, 8, 8, 1024, 64))
    dtype = base.pop("dtype", torch.bfloat16)
    return sa.make_params(shape, dtype, **base)


def test_workspace_sizes(lib):
    f = lambda p, b: lib.sparse_attn_workspace_size(ctypes.byref(p), b)
    units, T = 16 * 8 * 8, 1024
    assert f(_p(), 0) == units * T * 64 * 2        # RoPE-rotated keys, 16-bit
    assert f(_p(dtype=torch.float32), 0) == 0      # the general forward needs none
    n = f(_p(), 1)
    assert n >= units * T * 4                      # D_i per query
    assert f(_p(sinks=4), 1) > n                   # sink partials
    assert f(_p(shape=(1, 1, 1, 1, 48)), 1) == 0   # unsupported D -> 0
    assert f(_p(window=0), 1) == 0


@pytest.mark.parametrize("bad,code", [
    (dict(window=0), sa.SA_ERR_INVALID_ARG),
    (dict(shape=(1, 1, 1, 0, 64)), sa.SA_ERR_INVALID_ARG),
    (dict(shape=(1, 1, 1, 64, 48)), sa.SA_ERR_UNSUPPORTED),
    (dict(offsets=(1, 0, 3)), sa.SA_ERR_INVALID_ARG),
    (dict(offsets=tuple(range(1, 40))), sa.SA_ERR_UNSUPPORTED),
    (dict(sinks=-1), sa.SA_ERR_INVALID_ARG),
    (dict(sinks=17), sa.SA_ERR_UNSUPPORTED),
    (dict(rope_base=0.0), sa.SA_ERR_INVALID_ARG),
    (dict(shape=(1, 1, 1, (1 << 24) + 1, 64)), sa.SA_ERR_UNSUPPORTED),   # beyond the position range
    (dict(shape=(4096, 64, 64, 1 << 20, 64)), sa.SA_ERR_UNSUPPORTED),     # grid beyond 2^31 CTAs
])
def test_bad_params_rejected_on_host(lib, bad, code):
    p = _p(**bad)
    dummy = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    st = lib.sparse_attn_fwd(ctypes.byref(p), dummy, dummy, dummy, dummy, dummy, dummy,
                             None, 0, None)
    assert st == code
    st = lib.sparse_attn_bwd(ctypes.byref(p), dummy, dummy, dummy, dummy, dummy, dummy, dummy,
                             dummy, dummy, dummy, dummy, None, 0, None)
    assert st == code


def test_null_and_misaligned_pointers_rejected(lib):
    p = _p(shape=(1, 1, 1, 64, 64))
    ok = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert lib.sparse_attn_fwd(ctypes.byref(p), None, ok, ok, ok, ok, None, None, 0, None) == 1
    assert lib.sparse_attn_fwd(ctypes.byref(p), odd, ok, ok, ok, ok, None, None, 0, None) == 1
    # backward: workspace too small is reported as such
    st = lib.sparse_attn_bwd(ctypes.byref(p), ok, ok, ok, ok, ok, ok, ok, ok, ok, ok, ok,
                             ok, 16, None)
    assert st == sa.SA_ERR_WORKSPACE


def test_python_binding_refuses_cpu_tensors(lib):
    q = torch.zeros((1, 1, 1, 8, 16))
    with pytest.raises((ValueError, RuntimeError)):
        sa.fwd(q, q, q, torch.ones(1), window=2)


def test_context_size_and_validation(lib):
    """The training context exists only for the staged configurations, and
    the training calls reject a missing or short context before any GPU work."""
    f = lambda p: lib.sparse_attn_context_size(ctypes.byref(p))
    units, T = 16 * 8 * 8, 1024
    n = f(_p())
    assert n >= units * T * (2 * 64 * 2 + 4 * (12 + 15 + 15))
    assert f(_p(dtype=torch.float32)) == 0
    assert f(_p(shape=(1, 1, 1, 64, 32))) == 0
    dummy = ctypes.c_void_p(1 << 20)     # never dereferenced: validation comes first
    p32 = _p(dtype=torch.float32, shape=(1, 1, 1, 64, 64))
    alpha = ctypes.c_void_p(1 << 20)
    st = lib.sparse_attn_fwd_train(ctypes.byref(p32), dummy, dummy, dummy, alpha, dummy, None,
                                   dummy, 1 << 30, None)
    assert st == sa.SA_ERR_UNSUPPORTED
    p16 = _p(shape=(1, 1, 1, 64, 64))
    st = lib.sparse_attn_fwd_train(ctypes.byref(p16), dummy, dummy, dummy, alpha, dummy, None,
                                   dummy, 16, None)
    assert st == sa.SA_ERR_WORKSPACE
    st = lib.sparse_attn_bwd_ctx(ctypes.byref(p16), dummy, dummy, dummy, dummy, None, dummy,
                                 alpha, None, dummy, dummy, dummy, alpha, dummy, 1 << 30, None)
    assert st == sa.SA_ERR_INVALID_ARG
