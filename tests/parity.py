"""Shared helpers for the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare with the stated tolerances.

Tolerances (written here, used by every parity test):
  fp32 inputs : max |GPU - oracle| <= 1e-5 on O, LSE, dQ, dK, dV;
                d-alpha per layer: |GPU - oracle| <= 1e-5 * max(1, A_l).
  bf16 inputs : |GPU - oracle| <= max(1e-2, ulp_bf16(oracle) / 2) elementwise
                on O: the 1e-2 max-abs bound, except where storing the exact
                value in bf16 alone moves it further (|O| >= 4, where half a
                bf16 ulp is 0.0156), in which case a correctly rounded result
                must pass;
                max |GPU - oracle| <= 1e-2 on LSE (fp32);
                relative Frobenius norm <= 5e-2 on dQ, dK, dV;
                d-alpha per layer: |GPU - oracle| <= 5e-2 * A_l + 1e-6.
  A_l = sum over the layer's (batch, head) units of |unit's d-alpha| (the
  oracle's per-unit shares).  A layer's d-alpha sums per-unit terms of both
  signs that can cancel far below their size (the learned-alpha workload's
  layer 0: -72.7 from units of about 1e4), so the error a correct computation
  makes is proportional to A_l, not to the total; every layer is checked.
  The LSE bound follows from the staged kernels keeping rotated K rows in fp16
  (relative rounding 2^-12 per element, score errors of a few 1e-4 for N(0,1)
  inputs, up to ~1e-3 at the worst of ~1e5 queries).
The oracle is the fp64 build, fed the exact values the GPU reads (bf16 inputs
upcast), so the comparison measures only the GPU path's rounding.
"""
import numpy as np
import torch

import oracle
import structured_sparse_attention_fibonacci_b200 as sa

TOL = {
    torch.float32: dict(o_abs=1e-5, lse_abs=1e-5, grad_abs=1e-5, grad_rel=None, dal_rel=1e-5),
    torch.bfloat16: dict(o_abs=1e-2, lse_abs=1e-2, grad_abs=None, grad_rel=5e-2, dal_rel=5e-2),
}


class BwdRef(tuple):
    """The oracle's backward outputs (dQ, dK, dV, dalpha[, dbeta]) with each
    (layer, batch, head) unit's share of dalpha as ``units`` [L, B, H]."""
    units = None


def rel_norm(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def run_gpu_fwd(q, k, v, alpha, **kw):
    o, lse = sa.fwd(q, k, v, alpha, **kw)
    torch.cuda.synchronize()
    return o, lse


def half_ulp_bf16(x):
    """Half a bf16 unit in the last place of |x| (8 significant bits)."""
    ax = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8), 0.0)


def o_bound(o_ref, dtype):
    """Elementwise bound on |O_gpu - O_oracle|: the dtype's max-abs tolerance,
    or for bf16 outputs half a bf16 ulp of the exact value where that is larger
    (a correctly rounded bf16 result always passes)."""
    tol = TOL[dtype]["o_abs"]
    if dtype != torch.bfloat16:
        return tol
    return np.maximum(tol, half_ulp_bf16(o_ref))


def check_fwd(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what=""):
    """Returns (worst |dO| / bound, worst |dLSE|); asserts both within bounds."""
    tol = TOL[dtype]
    o_gpu, lse_gpu = to_np(o_gpu), to_np(lse_gpu)
    assert np.array_equal(np.isnan(o_gpu), np.isnan(o_ref)), f"{what}: NaN pattern of O"
    fin = ~np.isnan(o_ref)
    err = np.abs(o_gpu - o_ref)
    ratio = (err / o_bound(o_ref, dtype))[fin]
    worst = ratio.max(initial=0.0)
    err_l = np.abs(lse_gpu - lse_ref)[~np.isnan(lse_ref)].max(initial=0.0)
    if worst > 1.0:
        at = np.unravel_index(np.argmax(np.where(fin, err / o_bound(o_ref, dtype), -1)), err.shape)
        raise AssertionError(f"{what}: O err {err[at]:.3e} at {at} (oracle {o_ref[at]:.5f}, "
                             f"gpu {o_gpu[at]:.5f}) beyond its bound ({worst:.3f} x)")
    assert err_l <= tol["lse_abs"], f"{what}: LSE max abs err {err_l:.3e}"
    return worst, err_l


def check_bwd(gpu, ref, dtype, what="", units=None):
    """gpu, ref: (dQ, dK, dV, dalpha, ...); the dalpha check uses the oracle's
    per-unit shares (``units``, else ``ref.units``)."""
    tol = TOL[dtype]
    out = {}
    for name, g, r in zip(("dQ", "dK", "dV"), gpu[:3], ref[:3]):
        g = to_np(g)
        assert np.array_equal(np.isnan(g), np.isnan(r)), f"{what}: NaN pattern of {name}"
        fin = ~np.isnan(r)
        if tol["grad_abs"] is not None:
            e = np.abs(g - r)[fin].max(initial=0.0)
            assert e <= tol["grad_abs"], f"{what}: {name} max abs err {e:.3e}"
        else:
            e = rel_norm(g[fin], r[fin])
            assert e <= tol["grad_rel"], f"{what}: {name} rel-norm err {e:.3e}"
        out[name] = e
    if units is None:
        units = getattr(ref, "units", None)
    out["dalpha"] = check_dalpha(gpu[3], ref[3], dtype, what, units=units)
    return out


def dalpha_scale(dal_ref, units):
    """A_l per layer: sum over the layer's units of |unit's d-alpha| (|dalpha_l|
    itself when the per-unit shares are not given)."""
    dal_ref = np.asarray(dal_ref, np.float64).reshape(-1)
    if units is None:
        return np.abs(dal_ref)
    u = np.abs(np.asarray(units, np.float64)).reshape(dal_ref.shape[0], -1)
    return u.sum(axis=1)


def check_dalpha(dal_gpu, dal_ref, dtype, what="", units=None):
    """Every layer: |GPU - oracle| <= tol * A_l (+ a floor), A_l from
    dalpha_scale.  Returns the worst |error| / bound over the layers."""
    tol = TOL[dtype]["dal_rel"]
    dal_g = to_np(dal_gpu).reshape(-1)
    dal_r = np.asarray(dal_ref, np.float64).reshape(-1)
    fin = ~np.isnan(dal_r)
    assert np.array_equal(np.isnan(dal_g), ~fin), f"{what}: NaN pattern of dalpha"
    if not fin.any():
        return 0.0
    scale = dalpha_scale(dal_r, units)
    if dtype == torch.float32:
        bound = tol * np.maximum(scale, 1.0)
    else:
        bound = tol * scale + 1e-6
    ratio = np.abs(dal_g - dal_r)[fin] / bound[fin]
    worst = float(ratio.max())
    assert worst <= 1.0, (f"{what}: dalpha beyond its per-layer bound ({worst:.3f} x): "
                          f"gpu {dal_g} vs oracle {dal_r}, A_l {scale}")
    return worst


def oracle_fwd(q, k, v, alpha, **kw):
    return oracle.fwd(to_np(q), to_np(k), to_np(v), to_np(alpha).astype(np.float32), **kw)


def oracle_bwd(q, k, v, dout, alpha, **kw):
    out = oracle.bwd(to_np(q), to_np(k), to_np(v), to_np(dout),
                     to_np(alpha).astype(np.float32), dalpha_units=True, **kw)
    ref = BwdRef(out[:-1])
    ref.units = out[-1]
    return ref
