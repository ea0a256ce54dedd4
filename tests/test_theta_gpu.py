"""Learned-alpha map on the GPU (sparse_attn_alpha_from_theta / _dtheta)
against the oracle: alpha = 0.5 + sigmoid(theta) and its gradient."""
import numpy as np
import pytest
import torch

import structured_sparse_attention_fibonacci_b200 as sa

import oracle
from parity import check_dalpha, oracle_bwd, to_np

DEV = "cuda"


@pytest.mark.gpu
def test_alpha_and_dtheta_match_the_oracle():
    g = torch.Generator(device="cpu").manual_seed(3)
    theta = torch.cat([torch.tensor([0.0, 20.0, -20.0, np.log(3.0)]),
                       3 * torch.randn(60, generator=g)]).float()
    dalpha = torch.randn(theta.numel(), generator=g).float()
    a = sa.alpha_from_theta(theta.to(DEV))
    dth = sa.dtheta(theta.to(DEV), dalpha.to(DEV))
    torch.cuda.synchronize()
    orc = oracle.default()
    a_ref = orc.alpha_from_theta(theta.numpy().astype(np.float64))
    d_ref = orc.dtheta(theta.numpy().astype(np.float64), dalpha.numpy().astype(np.float64))
    assert np.abs(to_np(a) - a_ref).max() <= 2e-7
    assert (to_np(a) >= 0.5).all() and (to_np(a) <= 1.5).all()
    assert float(a[0]) == 1.0
    assert np.abs(to_np(dth) - d_ref).max() <= 1e-6 * max(1.0, np.abs(d_ref).max())


@pytest.mark.gpu
def test_learned_step_through_theta():
    """theta -> alpha -> forward + backward -> dalpha -> dtheta, against the
    oracle's backward at the same alpha and the oracle's chain rule."""
    L, B, H, T, D = 3, 1, 2, 300, 64
    g = torch.Generator(device="cpu").manual_seed(11)
    q, k, v, do = (torch.randn((L, B, H, T, D), generator=g).to(torch.bfloat16).to(DEV)
                   for _ in range(4))
    theta = torch.tensor([0.0, -0.8, 1.1], device=DEV)
    alpha = sa.alpha_from_theta(theta)
    o, lse = sa.fwd(q, k, v, alpha, window=12)
    dq, dk, dv, dal = sa.bwd(q, k, v, o, lse, do, alpha, window=12)
    dth = sa.dtheta(theta, dal)
    torch.cuda.synchronize()
    ref = oracle_bwd(q, k, v, do, alpha, window=12)
    check_dalpha(dal, ref[3], torch.bfloat16, "dalpha at alpha(theta)", units=ref.units)
    dth_ref = oracle.default().dtheta(to_np(theta), ref[3])
    # each unit's share of dtheta: its dalpha share times the same chain-rule factor
    th = to_np(theta)
    sig = 1.0 / (1.0 + np.exp(-th))
    units_th = ref.units * (sig * (1.0 - sig)).reshape(-1, 1, 1)
    check_dalpha(dth, dth_ref, torch.bfloat16, "dtheta", units=units_th)
