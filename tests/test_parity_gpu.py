"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Tolerances are in tests/parity.py."""
import zlib

import numpy as np
import pytest
import torch

import structured_sparse_attention_fibonacci_b200 as sa
from structured_sparse_attention_fibonacci_b200.inputs import (FIB15, POW2_4096, WORKLOADS,
                                                                make_dout, make_inputs)
from parity import (check_bwd, check_dalpha, check_fwd, half_ulp_bf16, oracle_bwd, oracle_fwd,
                    run_gpu_fwd, to_np)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(shape, dtype, seed, with_dout=True):
    g = torch.Generator(device="cpu").manual_seed(seed)
    ts = [torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)
          for _ in range(4 if with_dout else 3)]
    return [t.to(DEV) for t in ts]


# The largest offset table the library takes (32 entries): the Fibonacci and
# power-of-2 ladders together, unsorted, with duplicates (1, 2 and 8 appear in
# both), and entries whose distance at alpha = 1.5 exceeds T = 4096 (3000).
OFF32 = (2048, 1, 3000, 2, 3, 5, 8, 13, 100, 21, 34, 55, 89, 144, 233, 377, 610, 987, 1, 2, 4,
         8, 16, 32, 64, 128, 256, 512, 1024, 50, 7, 11)
assert len(OFF32) == 32

# (name, dtype, (L, B, H, T, D), window, sinks, alphas, offsets)
SMALL = [
    ("tiny_fp32_cfg", torch.float32, (1, 1, 2, 64, 16), 6, 0, [1.0], FIB15),
    ("stagger_ragged_bf16", torch.bfloat16, (3, 1, 2, 300, 64), 12, 0, [0.5, 0.9666667, 1.5], FIB15),
    ("past_987_bf16", torch.bfloat16, (2, 1, 2, 1100, 64), 12, 0, [1.0, 1.1234], FIB15),
    ("window64_sinks_bf16", torch.bfloat16, (1, 1, 2, 700, 64), 64, 4, [1.0], FIB15),
    ("d32_fp32", torch.float32, (2, 1, 2, 77, 32), 3, 2, [0.77, 1.33], FIB15),
    ("d128_fp32", torch.float32, (1, 2, 1, 50, 128), 5, 1, [1.2], FIB15),
    ("d128_bf16", torch.bfloat16, (1, 1, 2, 90, 128), 7, 3, [0.61], FIB15),
    ("d16_w1_bf16", torch.bfloat16, (1, 1, 3, 17, 16), 1, 0, [0.93], FIB15),
    ("t1_fp32", torch.float32, (2, 1, 1, 1, 64), 12, 4, [1.0, 0.5], FIB15),
    ("t2_fp32", torch.float32, (1, 1, 1, 2, 64), 12, 4, [0.5], FIB15),
    ("w_ge_t_fp32", torch.float32, (1, 1, 2, 33, 64), 40, 0, [1.0], FIB15),
    ("no_offsets_fp32", torch.float32, (1, 1, 2, 45, 64), 4, 2, [1.0], ()),
    ("offsets_beyond_t_fp32", torch.float32, (1, 1, 1, 40, 64), 2, 0, [1.5], FIB15),
    ("custom_pow2_bf16", torch.bfloat16, (1, 1, 2, 260, 64), 8, 0, [1.0],
     (1, 2, 4, 8, 16, 32, 64, 128, 256)),
    # the power-of-2 ladder at the 4x evaluation length: offsets up to 2048,
    # reaching 3072 + 1 rows back at alpha = 1.5
    ("pow2_ladder_t4096_bf16", torch.bfloat16, (2, 1, 1, 4096, 64), 12, 0, [1.0, 1.5], POW2_4096),
    ("offsets32_t4096_bf16", torch.bfloat16, (1, 1, 1, 4096, 64), 12, 2, [1.5], OFF32),
    ("offsets32_fp32", torch.float32, (1, 1, 1, 700, 32), 5, 1, [0.77], OFF32),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_fwd_bwd_small(case):
    name, dtype, shape, W, S, alphas, offs = case
    q, k, v, do = _inputs(shape, dtype, seed=zlib.crc32(name.encode()) % 10000)
    alpha = torch.tensor(alphas, dtype=torch.float32, device=DEV)
    kw = dict(window=W, sinks=S, offsets=offs)
    o, lse = run_gpu_fwd(q, k, v, alpha, **kw)
    o_ref, lse_ref = oracle_fwd(q, k, v, alpha, **kw)
    check_fwd(o, lse, o_ref, lse_ref, dtype, name)
    grads = sa.bwd(q, k, v, o, lse, do, alpha, **kw)
    torch.cuda.synchronize()
    ref = oracle_bwd(q, k, v, do, alpha, **kw)
    check_bwd(grads, ref, dtype, name)


def test_nan_alpha_poisons_only_its_layer():
    q, k, v, do = _inputs((2, 1, 2, 40, 64), torch.float32, seed=3)
    alpha = torch.tensor([float("nan"), 1.0], device=DEV)
    o, lse = run_gpu_fwd(q, k, v, alpha, window=4)
    assert torch.isnan(o[0]).all() and torch.isnan(lse[0]).all()
    o_ref, lse_ref = oracle_fwd(q, k, v, alpha, window=4)
    check_fwd(o, lse, o_ref, lse_ref, torch.float32, "nan alpha")
    grads = sa.bwd(q, k, v, o, lse, do, alpha, window=4)
    check_bwd(grads, oracle_bwd(q, k, v, do, alpha, window=4), torch.float32, "nan alpha bwd")


def test_backward_is_deterministic():
    q, k, v, do = _inputs((2, 2, 2, 513, 64), torch.bfloat16, seed=11)
    alpha = torch.tensor([0.71, 1.29], device=DEV)
    o, lse = run_gpu_fwd(q, k, v, alpha, window=12, sinks=2)
    a = [t.clone() for t in sa.bwd(q, k, v, o, lse, do, alpha, window=12, sinks=2)]
    b = sa.bwd(q, k, v, o, lse, do, alpha, window=12, sinks=2)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_streams_are_respected():
    q, k, v, _ = _inputs((1, 1, 2, 200, 64), torch.bfloat16, seed=12)
    alpha = torch.tensor([1.1], device=DEV)
    ref, _ = run_gpu_fwd(q, k, v, alpha, window=12)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, _ = sa.fwd(q, k, v, alpha, window=12)
    s.synchronize()
    assert torch.equal(o, ref)


# ---- full-size workloads, the launch the benchmark times; sampled units ------

def _sample_units(wl, n):
    rng = np.random.default_rng(123)
    units = {(0, 0, 0), (wl.L - 1, wl.B - 1, wl.H - 1)}
    while len(units) < min(n, wl.L * wl.B * wl.H):
        units.add((int(rng.integers(wl.L)), int(rng.integers(wl.B)), int(rng.integers(wl.H))))
    return sorted(units)


FULL = [(n, "plain") for n in WORKLOADS if not WORKLOADS[n].decode] + \
    [(n, "training") for n in WORKLOADS if WORKLOADS[n].backward and not WORKLOADS[n].prior]


@pytest.mark.parametrize("name,mode", FULL, ids=[f"{n}-{m}" for n, m in FULL])
def test_full_workload_sampled(name, mode):
    """Every non-decode workload at full size.  "plain": sparse_attn_fwd /
    sparse_attn_bwd.  "training": the launch the benchmark times for a
    training workload -- the forward saving its context into a buffer, then
    the backward reading it (with the forward's LSE).  O, LSE, dQ, dK, dV are
    compared on sampled (layer, batch, head) units; dalpha on every layer."""
    wl = WORKLOADS[name]
    ts = make_inputs(wl, device=DEV)
    q, k, v = ts[:3]
    alpha = wl.alpha().to(DEV)
    kw = dict(window=wl.window, sinks=wl.sinks, offsets=wl.offsets, rope_base=wl.rope_base)
    ctx = None
    if mode == "training":
        ctx = torch.full((sa.context_size(tuple(q.shape), q.dtype, **kw),), 0xFF,
                         dtype=torch.uint8, device=DEV)
    o, lse = sa.fwd(q, k, v, alpha, context=ctx, **kw)
    torch.cuda.synchronize()
    for (l, b, h) in _sample_units(wl, 4):
        sl = (slice(l, l + 1), slice(b, b + 1), slice(h, h + 1))
        o_ref, lse_ref = oracle_fwd(q[sl], k[sl], v[sl], alpha[l:l + 1], **kw)
        check_fwd(o[sl], lse[sl], o_ref, lse_ref, wl.dtype, f"{name} {mode} unit {(l, b, h)}")
    if not wl.backward:
        return
    do = ts[3]
    grads = sa.bwd(q, k, v, o, lse, do, alpha, context=ctx, **kw)
    torch.cuda.synchronize()
    assert sa.device_error() == 0
    for (l, b, h) in _sample_units(wl, 3):
        sl = (slice(l, l + 1), slice(b, b + 1), slice(h, h + 1))
        ref = oracle_bwd(q[sl], k[sl], v[sl], do[sl], alpha[l:l + 1], **kw)
        # one unit's dalpha is not the layer sum: compare dQ/dK/dV here
        g = tuple(x[sl] for x in grads[:3]) + (torch.tensor(ref[3]),)
        check_bwd(g, ref, wl.dtype, f"{name} {mode} bwd unit {(l, b, h)}")
    # dalpha: every layer, each against its own per-layer bound
    ref = oracle_bwd(q, k, v, do, alpha, **kw)
    check_dalpha(grads[3], ref[3], wl.dtype, f"{name} {mode} dalpha", units=ref.units)


@pytest.mark.parametrize("name", ["long_sinks", "window_64_stagger", "paper_fwd"])
def test_tcgen05_forward_full_size(name):
    """The fifth-generation tensor-core forward (selected explicitly; the
    default dispatch does not take it) at full size, sampled units."""
    wl = WORKLOADS[name]
    q, k, v = make_inputs(wl, device=DEV)[:3]
    alpha = wl.alpha().to(DEV)
    kw = dict(window=wl.window, sinks=wl.sinks, offsets=wl.offsets, rope_base=wl.rope_base)
    sa.select_forward(3)
    sa.trace_enable(True)
    try:
        o, lse = sa.fwd(q, k, v, alpha, **kw)
        torch.cuda.synchronize()
        names = set(sa.trace_read())
    finally:
        sa.trace_enable(False)
        sa.select_forward(0)
    assert "fwd_umma" in names, names
    assert sa.device_error() == 0
    for (l, b, h) in _sample_units(wl, 4):
        sl = (slice(l, l + 1), slice(b, b + 1), slice(h, h + 1))
        o_ref, lse_ref = oracle_fwd(q[sl], k[sl], v[sl], alpha[l:l + 1], **kw)
        check_fwd(o[sl], lse[sl], o_ref, lse_ref, wl.dtype, f"{name} tcgen05 unit {(l, b, h)}")


# ---- the staged bf16 d=64 forward and the general kernels on the same inputs ----
FAST = [
    ("fast_tail_129", (2, 1, 2, 129, 64), 12, 0, [0.5, 1.5], FIB15),
    ("fast_t257_sinks", (1, 2, 1, 257, 64), 12, 4, [1.1], FIB15),
    ("fast_t1", (1, 1, 2, 1, 64), 12, 4, [1.0], FIB15),
    ("fast_t3_s16", (1, 1, 1, 3, 64), 2, 16, [0.7], FIB15),
    ("fast_w64_s16", (1, 1, 2, 600, 64), 64, 16, [1.0], FIB15),
    ("fast_unsorted_dups", (1, 1, 2, 400, 64), 5, 1, [0.83], (34, 1, 5, 5, 233, 2, 89, 13)),
    ("fast_alpha0", (1, 1, 1, 70, 64), 3, 0, [0.0], FIB15),
    ("fast_w1", (1, 1, 2, 200, 64), 1, 0, [1.37], FIB15),
    ("fast_w7_odd", (2, 1, 1, 300, 64), 7, 3, [0.61, 1.44], FIB15),
    ("fast_long_1500", (1, 1, 1, 1700, 64), 12, 0, [1.5], FIB15),
    ("fast_pi_skip", (2, 1, 2, 300, 64), 5, 0, [1.0, 1.0], (16,)),
    ("fast_pow2_t4096", (2, 1, 1, 4096, 64), 12, 0, [1.0, 1.5], POW2_4096),
    ("fast_off32_t4096", (1, 1, 1, 4096, 64), 12, 2, [1.5], OFF32),
    ("fast_off32_w64", (1, 1, 1, 2000, 64), 64, 4, [1.0], OFF32),
    # rings of staged rows that are not a power of two (the mma.sync forward
    # sizes its ring for CTAs per SM: 224 rows here, 272 at W = 128)
    ("fast_w64_s4_ring224", (1, 1, 2, 700, 64), 64, 4, [1.37], FIB15),
    ("fast_w128_ring272", (1, 1, 1, 1100, 64), 128, 0, [0.77], FIB15),
]


@pytest.mark.parametrize("kernel", [1, 2, 3], ids=["cuda_core", "tensor_core", "tcgen05"])
@pytest.mark.parametrize("case", FAST, ids=[c[0] for c in FAST])
def test_fast_and_general_forward(case, kernel):
    name, shape, W, S, alphas, offs = case
    q, k, v, _ = _inputs(shape, torch.bfloat16, seed=zlib.crc32(name.encode()) % 10000)
    alpha = torch.tensor(alphas, dtype=torch.float32, device=DEV)
    kw = dict(window=W, sinks=S, offsets=offs)
    o_ref, lse_ref = oracle_fwd(q, k, v, alpha, **kw)
    sa.select_forward(kernel)
    try:
        o_fast, lse_fast = run_gpu_fwd(q, k, v, alpha, **kw)
    finally:
        sa.select_forward(0)
    check_fwd(o_fast, lse_fast, o_ref, lse_ref, torch.bfloat16, f"{name} (staged {kernel})")
    sa.force_general(True)
    try:
        o_gen, lse_gen = run_gpu_fwd(q, k, v, alpha, **kw)
    finally:
        sa.force_general(False)
    check_fwd(o_gen, lse_gen, o_ref, lse_ref, torch.bfloat16, name + " (general)")
    # the two paths differ by summation order and the 16-bit rounding of the
    # staged operands; each output is then rounded to bf16 on its own, so two
    # values on either side of a rounding boundary may differ by one bf16 ulp
    # on top of that
    og = o_gen.float().cpu().numpy()
    diff = np.abs(o_fast.float().cpu().numpy() - og) - 2 * half_ulp_bf16(og)
    assert diff.max() <= 1e-2
    assert (lse_fast - lse_gen).abs().max().item() <= 1e-2


def test_fast_path_is_the_one_dispatched():
    q, k, v, _ = _inputs((1, 1, 1, 300, 64), torch.bfloat16, seed=5)
    alpha = torch.tensor([1.0], device=DEV)
    sa.trace_enable(True)
    try:
        run_gpu_fwd(q, k, v, alpha, window=12)
        names = set(sa.trace_read())
    finally:
        sa.trace_enable(False)
    assert names == {"rope_keys", "fwd_fast"}, names     # W = 12: the CUDA-core kernel
    sa.select_forward(2)
    sa.trace_enable(True)
    try:
        run_gpu_fwd(q, k, v, alpha, window=12)
        names = set(sa.trace_read())
    finally:
        sa.trace_enable(False)
        sa.select_forward(0)
    assert names == {"rope_keys", "fwd_tc"}, names
    sa.select_forward(3)
    sa.trace_enable(True)
    try:
        run_gpu_fwd(q, k, v, alpha, window=12)
        names = set(sa.trace_read())
    finally:
        sa.trace_enable(False)
        sa.select_forward(0)
    assert names == {"rope_keys", "fwd_umma"}, names


@pytest.mark.parametrize("case", FAST, ids=[c[0] for c in FAST])
def test_fast_and_general_backward(case):
    name, shape, W, S, alphas, offs = case
    q, k, v, do = _inputs(shape, torch.bfloat16, seed=zlib.crc32(name.encode()) % 10000 + 1)
    alpha = torch.tensor(alphas, dtype=torch.float32, device=DEV)
    kw = dict(window=W, sinks=S, offsets=offs)
    ref = oracle_bwd(q, k, v, do, alpha, **kw)
    o, lse = run_gpu_fwd(q, k, v, alpha, **kw)
    g_fast = [t.clone() for t in sa.bwd(q, k, v, o, lse, do, alpha, **kw)]
    torch.cuda.synchronize()
    check_bwd(g_fast, ref, torch.bfloat16, name + " (staged)")
    sa.force_general(True)
    try:
        o, lse = run_gpu_fwd(q, k, v, alpha, **kw)
        g_gen = sa.bwd(q, k, v, o, lse, do, alpha, **kw)
        torch.cuda.synchronize()
    finally:
        sa.force_general(False)
    check_bwd(g_gen, ref, torch.bfloat16, name + " (general)")


@pytest.mark.parametrize("case", FAST, ids=[c[0] for c in FAST])
def test_training_context_forward_and_backward(case):
    """sparse_attn_fwd_train + sparse_attn_bwd_ctx against the oracle (the
    backward reuses the forward's probabilities, row-score differences and
    rotated keys instead of recomputing them)."""
    name, shape, W, S, alphas, offs = case
    q, k, v, do = _inputs(shape, torch.bfloat16, seed=zlib.crc32(name.encode()) % 10000 + 1)
    alpha = torch.tensor(alphas, dtype=torch.float32, device=DEV)
    kw = dict(window=W, sinks=S, offsets=offs)
    n_ctx = sa.context_size(shape, torch.bfloat16, **kw)
    assert n_ctx > 0
    ctx = torch.full((n_ctx,), 0xFF, dtype=torch.uint8, device=DEV)   # NaN-filled on purpose
    o, lse = sa.fwd(q, k, v, alpha, context=ctx, **kw)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle_fwd(q, k, v, alpha, **kw)
    check_fwd(o, lse, o_ref, lse_ref, torch.bfloat16, name + " (training forward)")
    g = sa.bwd(q, k, v, o, None, do, alpha, context=ctx, **kw)
    torch.cuda.synchronize()
    ref = oracle_bwd(q, k, v, do, alpha, **kw)
    check_bwd(g, ref, torch.bfloat16, name + " (context backward)")


def test_training_context_dispatch_skips_the_score_pass():
    q, k, v, do = _inputs((1, 1, 1, 300, 64), torch.bfloat16, seed=7)
    alpha = torch.tensor([1.1], device=DEV)
    ctx = torch.empty(sa.context_size(tuple(q.shape), q.dtype, window=12), dtype=torch.uint8,
                      device=DEV)
    sa.trace_enable(True)
    try:
        o, lse = sa.fwd(q, k, v, alpha, window=12, context=ctx)
        sa.bwd(q, k, v, o, lse, do, alpha, window=12, context=ctx)
        names = set(sa.trace_read())
    finally:
        sa.trace_enable(False)
    # one key rotation (the forward's); the queries come rotated from the forward
    assert names == {"rope_keys", "fwd_fast", "bwd_q_fast", "bwd_kv_fast", "reduce_dalpha"}, names
    assert sa.device_error() == 0


def test_fast_backward_is_the_one_dispatched():
    q, k, v, do = _inputs((1, 1, 1, 300, 64), torch.bfloat16, seed=6)
    alpha = torch.tensor([1.0], device=DEV)
    o, lse = run_gpu_fwd(q, k, v, alpha, window=12)
    sa.trace_enable(True)
    try:
        sa.bwd(q, k, v, o, lse, do, alpha, window=12)
        names = set(sa.trace_read())
    finally:
        sa.trace_enable(False)
    assert names == {"rope_keys", "rope_queries", "bwd_q_fast", "bwd_kv_fast",
                     "reduce_dalpha"}, names


def test_tensors_beyond_2_31_elements():
    """Maximum sizes: 520 (layer, batch, head) units of T = 65536 rows of 64
    (2.2e9 elements per tensor, 4.4 GB in bf16). The last unit starts past
    element 2^31, so any 32-bit index arithmetic would show. Units 0 and 519
    hold N(0, 1) data; every other unit is zero. Zero units contribute nothing
    to any output or to dalpha: q = k = v = dO = 0 there. So the oracle on the
    two data units gives the whole expected result. That covers O and LSE,
    dQ, dK and dV of those units, and the layer's dalpha, through the staged
    forward and backward."""
    L, B, H, T, D = 1, 1, 520, 65536, 64
    shape = (L, B, H, T, D)
    assert L * B * H * T * D > 2 ** 31
    data_units = (0, H - 1)
    g = torch.Generator(device="cpu").manual_seed(2031)
    host = {u: [torch.randn((T, D), generator=g, dtype=torch.float32).to(torch.bfloat16)
                for _ in range(4)] for u in data_units}
    q, k, v, do = (torch.zeros(shape, dtype=torch.bfloat16, device=DEV) for _ in range(4))
    for u in data_units:
        for t, x in zip((q, k, v, do), host[u]):
            t[0, 0, u].copy_(x)
    alpha = torch.tensor([1.1234], device=DEV)
    kw = dict(window=12, sinks=0, offsets=FIB15)
    o, lse = sa.fwd(q, k, v, alpha, **kw)
    dq, dk, dv, dal = sa.bwd(q, k, v, o, lse, do, alpha, **kw)
    torch.cuda.synchronize()
    assert sa.device_error() == 0
    sel = lambda t: t[:, :, list(data_units)].contiguous()
    o_ref, lse_ref = oracle_fwd(sel(q), sel(k), sel(v), alpha, **kw)
    check_fwd(sel(o), sel(lse), o_ref, lse_ref, torch.bfloat16, "beyond 2^31 forward")
    ref = oracle_bwd(sel(q), sel(k), sel(v), sel(do), alpha, **kw)
    check_bwd((sel(dq), sel(dk), sel(dv), dal), ref, torch.bfloat16, "beyond 2^31 backward")
    # a zero unit in between: zero outputs and gradients
    mid = H // 2
    for t in (o, dq, dk, dv):
        assert t[0, 0, mid].float().abs().max().item() == 0.0


# ---- input magnitude: Q and K scaled up --------------------------------------
# Scores grow with the square of the scale; a peaked softmax turns a score's
# rounding into an output error.  The staged kernels round the rotated keys to
# fp16 (2^-12 relative, reading 18), which keeps O within its bound up to about
# x2 (measured on B200: x2 at 0.82 of the bound, x4 at 1.3x on the CUDA-core
# kernel); the general kernels (fp32 throughout) keep the forward within it at
# x100 and x10000, where only the fp32 LSE's relative rounding grows.

def _scaled_inputs(shape, c, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    q, k, v, do = (torch.randn(shape, generator=g, dtype=torch.float32) for _ in range(4))
    return [t.to(torch.bfloat16).to(DEV) for t in (q * c, k * c, v, do)]


@pytest.mark.parametrize("kernel", [1, 2, 3], ids=["cuda_core", "tensor_core", "tcgen05"])
def test_staged_path_at_twice_the_input_scale(kernel):
    shape = (2, 1, 2, 600, 64)
    q, k, v, do = _scaled_inputs(shape, 2.0, seed=505)
    alpha = torch.tensor([0.77, 1.23], device=DEV)
    for W, S in ((12, 2), (64, 4)):
        kw = dict(window=W, sinks=S)
        sa.select_forward(kernel)
        try:
            o, lse = run_gpu_fwd(q, k, v, alpha, **kw)
        finally:
            sa.select_forward(0)
        o_ref, lse_ref = oracle_fwd(q, k, v, alpha, **kw)
        check_fwd(o, lse, o_ref, lse_ref, torch.bfloat16, f"x2 inputs W={W} (staged {kernel})")
        if kernel == 1:
            grads = sa.bwd(q, k, v, o, lse, do, alpha, **kw)
            torch.cuda.synchronize()
            check_bwd(grads, oracle_bwd(q, k, v, do, alpha, **kw), torch.bfloat16,
                      f"x2 inputs W={W} backward")


@pytest.mark.parametrize("c", [1e2, 1e4])
def test_general_forward_at_large_input_scales(c):
    shape = (1, 1, 2, 300, 64)
    q, k, v, _ = _scaled_inputs(shape, c, seed=506)
    alpha = torch.tensor([1.1234], device=DEV)
    kw = dict(window=12, sinks=2)
    sa.force_general(True)
    try:
        o, lse = run_gpu_fwd(q, k, v, alpha, **kw)
    finally:
        sa.force_general(False)
    o_ref, lse_ref = oracle_fwd(q, k, v, alpha, **kw)
    from parity import o_bound
    err = np.abs(to_np(o) - o_ref) / o_bound(o_ref, torch.bfloat16)
    assert err.max() <= 1.0, f"x{c:g} inputs: O err {err.max():.3f} x its bound"
    # LSE of scores near c^2: each score is a 64-term fp32 dot product of
    # c^2-sized products, rounded to about sqrt(64) * 2^-24 of itself
    rel = np.abs(to_np(lse) - lse_ref) / np.maximum(np.abs(lse_ref), 1.0)
    assert rel.max() <= 1e-5, f"x{c:g} inputs: LSE rel err {rel.max():.2e}"
