"""The log-prior on the offset members against the oracle.

The prior comes from "pi-Attention: Periodic Sparse Transformers for
Efficient Long-Context Modeling" (Core components: the local and skip logits
are fused in one softmax through a log-prior). Query i's beta_i is added to
the score of each of its offset members, and dbeta_i is the sum of those
members' dscores. The calls are sparse_attn_fwd_prior and
sparse_attn_bwd_prior through the C ABI.

Paths covered:
- the general kernels: fp32, and bf16 with D != 64;
- the staged kernels: bf16, D = 64, both forwards (CUDA-core and
  tensor-core) and the backward;
- the training pair with a context;
- the general kernels forced on a staged configuration.

Tolerances are those of tests/parity.py. dbeta uses the gradient tolerances:
fp32 max abs 1e-5, bf16 relative norm 5e-2.
"""
import zlib

import numpy as np
import pytest
import torch

import structured_sparse_attention_fibonacci_b200 as sa
from structured_sparse_attention_fibonacci_b200.inputs import (FIB15, WORKLOADS, make_inputs,
                                                                make_prior)
from parity import TOL, check_bwd, check_fwd, oracle_bwd, oracle_fwd, rel_norm, to_np

DEV = "cuda"

# (name, dtype, (L, B, H, T, D), window, sinks, alphas, offsets, beta scale)
CASES = [
    ("fp32_d16_fib", torch.float32, (2, 1, 2, 80, 16), 6, 0, [1.0, 0.77], FIB15, 1.0),
    ("fp32_d32_sinks", torch.float32, (1, 2, 1, 130, 32), 4, 3, [1.37], FIB15, 2.0),
    ("fp32_d64_tail", torch.float32, (1, 1, 2, 45, 64), 3, 0, [1.5], FIB15, 1.0),
    ("bf16_d128", torch.bfloat16, (1, 1, 2, 90, 128), 7, 1, [0.61], FIB15, 1.0),
    ("bf16_d64_stagger", torch.bfloat16, (3, 1, 2, 300, 64), 12, 0, [0.5, 0.9666667, 1.5], FIB15,
     1.0),
    ("bf16_d64_past_987", torch.bfloat16, (2, 1, 2, 1100, 64), 12, 0, [1.0, 1.1234], FIB15, 1.0),
    ("bf16_d64_w64_sinks", torch.bfloat16, (1, 1, 2, 700, 64), 64, 4, [1.0], FIB15, 1.0),
    ("bf16_d64_pi_skip", torch.bfloat16, (2, 1, 2, 260, 64), 5, 0, [1.0, 1.0], (16,), 1.5),
    ("bf16_d64_t1", torch.bfloat16, (1, 1, 2, 1, 64), 12, 2, [1.0], FIB15, 1.0),
]


def _inputs(shape, dtype, seed, scale):
    g = torch.Generator(device="cpu").manual_seed(seed)
    q, k, v, do = (torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)
                   for _ in range(4))
    beta = scale * torch.randn(shape[:4], generator=g, dtype=torch.float32)
    return [t.to(DEV) for t in (q, k, v, do, beta)]


def check_dbeta(dbeta_gpu, dbeta_ref, dtype, what):
    g, r = to_np(dbeta_gpu), np.asarray(dbeta_ref, np.float64)
    assert np.array_equal(np.isnan(g), np.isnan(r)), f"{what}: NaN pattern of dbeta"
    fin = ~np.isnan(r)
    if dtype == torch.float32:
        e = np.abs(g - r)[fin].max(initial=0.0)
        assert e <= TOL[dtype]["grad_abs"], f"{what}: dbeta max abs err {e:.3e}"
    else:
        e = rel_norm(g[fin], r[fin])
        assert e <= TOL[dtype]["grad_rel"], f"{what}: dbeta rel-norm err {e:.3e}"


def _ref(q, k, v, do, alpha, beta, **kw):
    o_ref, lse_ref = oracle_fwd(q, k, v, alpha, beta=to_np(beta), **kw)
    g_ref = oracle_bwd(q, k, v, do, alpha, beta=to_np(beta), **kw)
    return o_ref, lse_ref, g_ref


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_prior_fwd_bwd(case):
    name, dtype, shape, W, S, alphas, offs, bscale = case
    q, k, v, do, beta = _inputs(shape, dtype, zlib.crc32(name.encode()) % 10000, bscale)
    alpha = torch.tensor(alphas, dtype=torch.float32, device=DEV)
    kw = dict(window=W, sinks=S, offsets=offs)
    o, lse = sa.fwd(q, k, v, alpha, beta=beta, **kw)
    dq, dk, dv, dal, dbeta = sa.bwd(q, k, v, o, lse, do, alpha, beta=beta, **kw)
    torch.cuda.synchronize()
    o_ref, lse_ref, g_ref = _ref(q, k, v, do, alpha, beta, **kw)
    check_fwd(o, lse, o_ref, lse_ref, dtype, name)
    check_bwd((dq, dk, dv, dal), g_ref, dtype, name)
    check_dbeta(dbeta, g_ref[4], dtype, name)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["bf16_d64_stagger", "bf16_d64_w64_sinks", "bf16_d64_pi_skip"])
def test_prior_training_pair(name):
    """The training forward saves probabilities that include the prior; the
    context backward returns dbeta. The context is filled with NaN bytes
    first, so an unwritten entry would show."""
    _, dtype, shape, W, S, alphas, offs, bscale = next(c for c in CASES if c[0] == name)
    q, k, v, do, beta = _inputs(shape, dtype, zlib.crc32(name.encode()) % 10000, bscale)
    alpha = torch.tensor(alphas, dtype=torch.float32, device=DEV)
    kw = dict(window=W, sinks=S, offsets=offs)
    ctx = torch.full((sa.context_size(shape, dtype, **kw),), 0xFF, dtype=torch.uint8, device=DEV)
    o, lse = sa.fwd(q, k, v, alpha, beta=beta, context=ctx, **kw)
    dq, dk, dv, dal, dbeta = sa.bwd(q, k, v, o, lse, do, alpha, beta=beta, context=ctx, **kw)
    torch.cuda.synchronize()
    o_ref, lse_ref, g_ref = _ref(q, k, v, do, alpha, beta, **kw)
    check_fwd(o, lse, o_ref, lse_ref, dtype, name + " training")
    check_bwd((dq, dk, dv, dal), g_ref, dtype, name + " training")
    check_dbeta(dbeta, g_ref[4], dtype, name + " training")
    assert sa.device_error() == 0


@pytest.mark.gpu
def test_prior_general_kernels_forced():
    name = "bf16_d64_stagger"
    _, dtype, shape, W, S, alphas, offs, bscale = next(c for c in CASES if c[0] == name)
    q, k, v, do, beta = _inputs(shape, dtype, 77, bscale)
    alpha = torch.tensor(alphas, dtype=torch.float32, device=DEV)
    kw = dict(window=W, sinks=S, offsets=offs)
    sa.force_general(True)
    try:
        sa.trace_enable(True)
        sa.trace_read()
        o, lse = sa.fwd(q, k, v, alpha, beta=beta, **kw)
        dq, dk, dv, dal, dbeta = sa.bwd(q, k, v, o, lse, do, alpha, beta=beta, **kw)
        torch.cuda.synchronize()
        names = set(sa.trace_read())
        sa.trace_enable(False)
    finally:
        sa.force_general(False)
    assert names == {"fwd_general", "bwd_q_general", "bwd_kv_general", "reduce_dalpha"}, names
    o_ref, lse_ref, g_ref = _ref(q, k, v, do, alpha, beta, **kw)
    check_fwd(o, lse, o_ref, lse_ref, dtype, "forced general")
    check_bwd((dq, dk, dv, dal), g_ref, dtype, "forced general")
    check_dbeta(dbeta, g_ref[4], dtype, "forced general")


@pytest.mark.gpu
@pytest.mark.parametrize("kernel", [1, 2, 3])
def test_prior_on_both_staged_forwards(kernel):
    """W = 64 with sinks: the tensor-core forward (the default there) and the
    CUDA-core forward both carry the prior; each is dispatched as selected and
    matches the oracle."""
    q, k, v, do, beta = _inputs((1, 1, 2, 300, 64), torch.bfloat16, 5, 1.0)
    alpha = torch.tensor([1.1], device=DEV)
    kw = dict(window=64, sinks=4)
    sa.select_forward(kernel)
    try:
        sa.trace_enable(True)
        sa.trace_read()
        o, lse = sa.fwd(q, k, v, alpha, beta=beta, **kw)
        torch.cuda.synchronize()
        names = set(sa.trace_read())
        sa.trace_enable(False)
    finally:
        sa.select_forward(0)
    assert {1: "fwd_fast", 2: "fwd_tc", 3: "fwd_umma"}[kernel] in names, names
    o_ref, lse_ref = oracle_fwd(q, k, v, alpha, beta=to_np(beta), **kw)
    check_fwd(o, lse, o_ref, lse_ref, torch.bfloat16, f"prior forward kernel {kernel}")


@pytest.mark.gpu
def test_prior_limits_on_the_gpu():
    """beta = -1e4 (every e^beta underflows to 0) gives the attention without
    offsets and dbeta = 0; beta = 0 gives the plain call's results exactly."""
    shape = (2, 1, 2, 200, 64)
    q, k, v, do, _ = _inputs(shape, torch.bfloat16, 9, 1.0)
    alpha = torch.tensor([0.83, 1.21], device=DEV)
    kw = dict(window=12, sinks=1)
    far = torch.full(shape[:4], -1e4, device=DEV)
    o, lse = sa.fwd(q, k, v, alpha, beta=far, **kw)
    o0, lse0 = sa.fwd(q, k, v, alpha, offsets=(), **kw)
    g = sa.bwd(q, k, v, o, lse, do, alpha, beta=far, **kw)
    g0 = sa.bwd(q, k, v, o0, lse0, do, alpha, offsets=(), **kw)
    torch.cuda.synchronize()
    assert (o.float() - o0.float()).abs().max().item() <= 1e-2
    assert (lse - lse0).abs().max().item() <= 1e-3
    for a, b in zip(g[:3], g0[:3]):
        assert rel_norm(to_np(a), to_np(b)) <= 1e-2
    assert (g[4] == 0).all()
    zero = torch.zeros(shape[:4], device=DEV)
    o1, lse1 = sa.fwd(q, k, v, alpha, beta=zero, **kw)
    o2, lse2 = sa.fwd(q, k, v, alpha, **kw)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(lse1, lse2)


@pytest.mark.gpu
def test_prior_nan_alpha_layer():
    q, k, v, do, beta = _inputs((2, 1, 2, 64, 64), torch.bfloat16, 13, 1.0)
    alpha = torch.tensor([float("nan"), 1.0], device=DEV)
    o, lse = sa.fwd(q, k, v, alpha, beta=beta, window=6)
    g = sa.bwd(q, k, v, o, lse, do, alpha, beta=beta, window=6)
    torch.cuda.synchronize()
    assert torch.isnan(g[4][0]).all() and torch.isfinite(g[4][1]).all()
    o_ref, lse_ref, g_ref = _ref(q, k, v, do, alpha, beta, window=6)
    check_fwd(o, lse, o_ref, lse_ref, torch.bfloat16, "nan alpha prior")
    check_dbeta(g[4], g_ref[4], torch.bfloat16, "nan alpha prior")


@pytest.mark.gpu
def test_prior_workload_full_size():
    """The benchmark's prior workload (16 layers, B=8, H=8, T=1024) in its
    launch configuration: the training pair. Two whole layers are checked
    against the oracle. O, LSE and dbeta are compared on every unit of those
    layers; dQ, dK, dV on the same units; dalpha per layer."""
    wl = WORKLOADS["pi_gate_train"]
    q, k, v, do = make_inputs(wl, device=DEV)
    beta = make_prior(wl, device=DEV)
    alpha = wl.alpha().to(DEV)
    kw = dict(window=wl.window, sinks=wl.sinks, offsets=wl.offsets, rope_base=wl.rope_base)
    ctx = torch.empty(sa.context_size(tuple(q.shape), q.dtype, **kw), dtype=torch.uint8,
                      device=DEV)
    o, lse = sa.fwd(q, k, v, alpha, beta=beta, context=ctx, **kw)
    dq, dk, dv, dal, dbeta = sa.bwd(q, k, v, o, lse, do, alpha, beta=beta, context=ctx, **kw)
    torch.cuda.synchronize()
    for l in (0, wl.L - 1):
        s = slice(l, l + 1)
        o_ref, lse_ref, g_ref = _ref(q[s], k[s], v[s], do[s], alpha[s], beta[s], **kw)
        check_fwd(o[s], lse[s], o_ref, lse_ref, wl.dtype, f"pi_gate layer {l}")
        check_bwd((dq[s], dk[s], dv[s], dal[s]), g_ref, wl.dtype, f"pi_gate layer {l}")
        check_dbeta(dbeta[s], g_ref[4], wl.dtype, f"pi_gate layer {l}")


def test_prior_calls_reject_missing_beta():
    import ctypes
    p = sa.make_params((1, 1, 1, 64, 64), torch.bfloat16, window=12)
    dummy = ctypes.c_void_p(1 << 20)     # never dereferenced: validation comes first
    L = sa.lib()
    assert L.sparse_attn_fwd_prior(ctypes.byref(p), dummy, dummy, dummy, dummy, None, dummy,
                                   None, None, 0, None, 0, None) == sa.SA_ERR_INVALID_ARG
    assert L.sparse_attn_bwd_prior(ctypes.byref(p), dummy, dummy, dummy, dummy, dummy, dummy,
                                   dummy, dummy, None, dummy, dummy, dummy, dummy, None, None, 0,
                                   None) == sa.SA_ERR_INVALID_ARG
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert L.sparse_attn_fwd_prior(ctypes.byref(p), dummy, dummy, dummy, dummy, odd, dummy,
                                   None, None, 0, None, 0, None) == sa.SA_ERR_INVALID_ARG
