"""Failure paths of the staged kernels, made to happen without a GPU fault.

Bounded waits.  Every staging round waits on an mbarrier for at most a
limit of SM clocks.  With sparse_attn_plant_stall(1) each CTA of the staged
launches expects 16 bytes more in its first round than its copies deliver,
so that wait must give up: the kernel sets bit 0 of the device error word,
waits (again bounded) for its real copies, and returns.  The tests lower the
limit to 2e5 clocks (about 0.1 ms) so that the run stays short, then check
that the word reports it, that the process and the context stay usable, and
that the next call, without the stall, matches the oracle.

Range.  Rotated keys (and the backward's scaled queries) are staged as fp16
of the value / 256; values at or beyond 65520 * 256 would become infinite.
The RoPE pre-pass reports such an input in bit 2 of the error word; just
inside the limit nothing is reported and the output matches the oracle.
"""
import numpy as np
import pytest
import torch

import structured_sparse_attention_fibonacci_b200 as sa
from parity import check_bwd, check_fwd, o_bound, oracle_bwd, oracle_fwd, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.device_error_expected]

DEV = "cuda"
KW = dict(window=12, sinks=2)


def _inputs(shape, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return [torch.randn(shape, generator=g).to(torch.bfloat16).to(DEV) for _ in range(4)]


@pytest.fixture
def stalled():
    sa.device_error(clear=True)
    sa.set_wait_limit(200000)
    sa.plant_stall(True)
    try:
        yield
    finally:
        sa.plant_stall(False)
        sa.set_wait_limit(0)
        sa.device_error(clear=True)


@pytest.mark.parametrize("kernel", [1, 2, 3], ids=["cuda_core", "tensor_core", "tcgen05"])
def test_forward_wait_gives_up_and_reports(stalled, kernel):
    q, k, v, _ = _inputs((1, 1, 2, 300, 64), seed=21)
    alpha = torch.tensor([1.1234], device=DEV)
    sa.select_forward(kernel)
    try:
        sa.fwd(q, k, v, alpha, **KW)
        torch.cuda.synchronize()
        assert sa.device_error(clear=True) & sa.ERR_WAIT
        sa.plant_stall(False)
        o, lse = sa.fwd(q, k, v, alpha, **KW)
        torch.cuda.synchronize()
    finally:
        sa.select_forward(0)
    assert sa.device_error(clear=True) == 0
    o_ref, lse_ref = oracle_fwd(q, k, v, alpha, **KW)
    check_fwd(o, lse, o_ref, lse_ref, torch.bfloat16, "after a stalled forward")


@pytest.mark.parametrize("context", [False, True], ids=["plain", "training"])
def test_backward_wait_gives_up_and_reports(stalled, context):
    q, k, v, do = _inputs((1, 1, 2, 300, 64), seed=22)
    alpha = torch.tensor([0.8765], device=DEV)
    ctx = None
    if context:
        ctx = torch.empty(sa.context_size(tuple(q.shape), q.dtype, **KW), dtype=torch.uint8,
                          device=DEV)
    sa.plant_stall(False)
    o, lse = sa.fwd(q, k, v, alpha, context=ctx, **KW)
    sa.plant_stall(True)
    sa.bwd(q, k, v, o, lse, do, alpha, context=ctx, **KW)
    torch.cuda.synchronize()
    assert sa.device_error(clear=True) & sa.ERR_WAIT
    sa.plant_stall(False)
    g = sa.bwd(q, k, v, o, lse, do, alpha, context=ctx, **KW)
    torch.cuda.synchronize()
    assert sa.device_error(clear=True) == 0
    check_bwd(g, oracle_bwd(q, k, v, do, alpha, **KW), torch.bfloat16, "after a stalled backward")


def test_range_limit_of_the_staged_keys():
    """One key element per unit set to a large value, its RoPE partner 0:
    the rotated pair has that magnitude, split between its two dims by the
    angle at row 77.  1.6e7 (at most 62500 after / 256) is inside the fp16
    range: nothing is reported and O matches the oracle (the member's scores
    are about 2e6, so LSE carries fp16's 2^-12 relative rounding of them and
    is only required finite).  2.5e7 puts at least one rotated dim at 1.77e7
    (69000 after / 256) and is reported in bit 2."""
    q, k, v, _ = _inputs((1, 1, 2, 200, 64), seed=23)
    alpha = torch.tensor([1.0], device=DEV)
    kw = dict(window=12)
    sa.device_error(clear=True)
    k_in = k.clone()
    k_in[0, 0, :, 77, 5] = 1.6e7
    k_in[0, 0, :, 77, 37] = 0.0
    o, lse = sa.fwd(q, k_in, v, alpha, **kw)
    torch.cuda.synchronize()
    assert sa.device_error(clear=True) == 0
    assert torch.isfinite(lse).all() and torch.isfinite(o.float()).all()
    o_ref, _ = oracle_fwd(q, k_in, v, alpha, **kw)
    err = np.abs(to_np(o) - o_ref) / o_bound(o_ref, torch.bfloat16)
    assert err.max() <= 1.0, f"O err {err.max():.3f} x its bound with a key at 1.6e7"
    k_out = k.clone()
    k_out[0, 0, :, 77, 5] = 2.5e7
    k_out[0, 0, :, 77, 37] = 0.0
    sa.fwd(q, k_out, v, alpha, **kw)
    torch.cuda.synchronize()
    assert sa.device_error(clear=True) & sa.ERR_RANGE
