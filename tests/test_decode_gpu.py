"""Single-token decode (sparse_attn_decode) against the oracle.

Decode is row `pos` of the forward on the first pos + 1 rows ("Depth-Staggered
Fibonacci Spacing for Sparse Attention", Methodology: the attended set of
query pos).  The oracle therefore runs its forward on a sequence whose row pos
is the decode query and whose other query rows are arbitrary, and the test
takes row pos of O and LSE.  Cache rows after pos are filled with NaN: a read
of any of them would show in the result.
"""
import zlib

import numpy as np
import pytest
import torch

import structured_sparse_attention_fibonacci_b200 as sa
from structured_sparse_attention_fibonacci_b200.inputs import FIB15, WORKLOADS, make_decode_inputs

import oracle
from parity import check_fwd, oracle_fwd, to_np

DEV = "cuda"

# (name, dtype, (L, B, H, T_cache, D), window, sinks, alphas, offsets, positions)
CASES = [
    ("fp32_d16", torch.float32, (1, 1, 2, 80, 16), 6, 0, [1.0], FIB15, [0, 1, 5, 37, 79]),
    ("bf16_d64_stagger", torch.bfloat16, (3, 2, 2, 1200, 64), 12, 0, [0.5, 1.0, 1.5], FIB15,
     [0, 11, 12, 300, 987, 1199]),
    ("bf16_d64_sinks", torch.bfloat16, (1, 1, 4, 700, 64), 64, 4, [1.0], FIB15, [2, 63, 64, 699]),
    ("fp32_d32_learned", torch.float32, (2, 1, 2, 300, 32), 5, 2, [0.83, 1.37], FIB15, [3, 150, 299]),
    ("bf16_d128", torch.bfloat16, (1, 2, 1, 200, 128), 8, 1, [1.1], (34, 1, 5, 5, 2, 89, 13),
     [0, 100, 199]),
]


def _caches(shape, dtype, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    L, B, H, T, D = shape
    q = torch.randn((L, B, H, D), generator=g, dtype=torch.float32).to(dtype)
    k = torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)
    v = torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)
    return q, k, v


def _oracle_row(q, k, v, alpha, pos, **kw):
    """Row pos of the oracle forward on rows 0..pos, query row pos = q."""
    L, B, H, T, D = k.shape
    g = torch.Generator(device="cpu").manual_seed(pos + 1)
    qf = torch.randn((L, B, H, pos + 1, D), generator=g, dtype=torch.float32).to(q.dtype)
    qf[:, :, :, pos, :] = q
    o, lse = oracle_fwd(qf, k[:, :, :, :pos + 1].contiguous(), v[:, :, :, :pos + 1].contiguous(),
                        alpha, **kw)
    return o[:, :, :, pos, :], lse[:, :, :, pos]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_decode_matches_the_oracle(case):
    name, dtype, shape, W, S, alphas, offs, positions = case
    q, k, v = _caches(shape, dtype, zlib.crc32(name.encode()) % 10000)
    alpha = torch.tensor(alphas, dtype=torch.float32)
    kw = dict(window=W, sinks=S, offsets=offs)
    for pos in positions:
        kd, vd = k.clone(), v.clone()
        kd[:, :, :, pos + 1:] = float("nan")            # rows after pos must not be read
        vd[:, :, :, pos + 1:] = float("nan")
        o, lse = sa.decode(q.to(DEV), kd.to(DEV), vd.to(DEV), alpha.to(DEV), pos, **kw)
        torch.cuda.synchronize()
        o_ref, lse_ref = _oracle_row(q, k, v, alpha, pos, **kw)
        check_fwd(o, lse, o_ref, lse_ref, dtype, f"{name} pos={pos}")


@pytest.mark.gpu
def test_decode_nan_alpha_layer():
    q, k, v = _caches((2, 1, 1, 64, 64), torch.bfloat16, 5)
    alpha = torch.tensor([float("nan"), 1.0], device=DEV)
    o, lse = sa.decode(q.to(DEV), k.to(DEV), v.to(DEV), alpha, 40, window=12)
    torch.cuda.synchronize()
    assert torch.isnan(o[0].float()).all() and torch.isnan(lse[0]).all()
    assert torch.isfinite(o[1].float()).all() and torch.isfinite(lse[1]).all()


@pytest.mark.gpu
def test_decode_equals_the_forward_row_for_the_last_position():
    """The same kernel family end to end: decode at pos = T - 1 equals row
    T - 1 of sparse_attn_fwd on the same tensors (general path, fp32)."""
    L, B, H, T, D = 2, 2, 2, 150, 32
    g = torch.Generator(device="cpu").manual_seed(9)
    Q, K, V = (torch.randn((L, B, H, T, D), generator=g).to(DEV) for _ in range(3))
    alpha = torch.tensor([0.7, 1.3], device=DEV)
    o_f, lse_f = sa.fwd(Q, K, V, alpha, window=7)
    o_d, lse_d = sa.decode(Q[:, :, :, T - 1].contiguous(), K, V, alpha, T - 1, window=7)
    torch.cuda.synchronize()
    assert (o_d - o_f[:, :, :, T - 1]).abs().max().item() <= 1e-5
    assert (lse_d - lse_f[:, :, :, T - 1]).abs().max().item() <= 1e-5


def test_decode_rejects_windows_it_cannot_hold():
    import ctypes
    p = sa.make_params((1, 1, 1, 1024, 64), torch.bfloat16, window=257)
    dummy = ctypes.c_void_p(1 << 20)     # never dereferenced: validation comes first
    st = sa.lib().sparse_attn_decode(ctypes.byref(p), 600, dummy, dummy, dummy, dummy, dummy,
                                     None, None)
    assert st == sa.SA_ERR_UNSUPPORTED


def test_decode_rejects_positions_outside_the_cache():
    import ctypes
    p = sa.make_params((1, 1, 1, 64, 64), torch.bfloat16, window=12)
    dummy = ctypes.c_void_p(1 << 20)     # never dereferenced: validation comes first
    for pos in (-1, 64, 1000):
        st = sa.lib().sparse_attn_decode(ctypes.byref(p), pos, dummy, dummy, dummy, dummy, dummy,
                                         None, None)
        assert st == sa.SA_ERR_INVALID_ARG


@pytest.mark.gpu
def test_decode_workload_full_size():
    """The benchmark's decode workload (16 layers, B=8, H=8, 4096-row caches,
    position 4095), in its launch configuration; two whole layers (128 units)
    against the oracle's decode."""
    wl = WORKLOADS["decode_4k"]
    q1, kc, vc = make_decode_inputs(wl)
    alpha = wl.alpha()
    kw = dict(window=wl.window, sinks=wl.sinks, offsets=wl.offsets, rope_base=wl.rope_base)
    o, lse = sa.decode(q1.to(DEV), kc.to(DEV), vc.to(DEV), alpha.to(DEV), wl.T - 1, **kw)
    torch.cuda.synchronize()
    for l in (0, wl.L - 1):
        o_ref, lse_ref = oracle.decode(to_np(q1[l:l + 1]), to_np(kc[l:l + 1]), to_np(vc[l:l + 1]),
                                       alpha[l:l + 1].numpy(), wl.T - 1, **kw)
        check_fwd(o[l:l + 1], lse[l:l + 1], o_ref, lse_ref, wl.dtype, f"decode_4k layer {l}")


@pytest.mark.gpu
@pytest.mark.parametrize("case", [c for c in CASES if c[0] in ("bf16_d64_stagger", "fp32_d32_learned")],
                         ids=lambda c: c[0])
def test_decode_with_a_prior(case):
    """sparse_attn_decode_prior: the new queries' log-prior on their offset
    members, against the oracle's decode with the same prior."""
    name, dtype, shape, W, S, alphas, offs, positions = case
    q, k, v = _caches(shape, dtype, zlib.crc32(name.encode()) % 10000 + 1)
    g = torch.Generator(device="cpu").manual_seed(44)
    beta = 1.5 * torch.randn(shape[:3], generator=g)
    alpha = torch.tensor(alphas, dtype=torch.float32)
    kw = dict(window=W, sinks=S, offsets=offs)
    for pos in positions:
        o, lse = sa.decode(q.to(DEV), k.to(DEV), v.to(DEV), alpha.to(DEV), pos, beta=beta.to(DEV),
                           **kw)
        torch.cuda.synchronize()
        o_ref, lse_ref = oracle.decode(to_np(q), to_np(k), to_np(v), alpha.numpy(), pos,
                                       beta=beta.numpy(), **kw)
        check_fwd(o, lse, o_ref, lse_ref, dtype, f"{name} prior pos={pos}")
