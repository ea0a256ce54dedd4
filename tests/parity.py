"""Shared helpers for the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare with the stated tolerances.

Tolerances (written here, used by every parity test):
  fp32 inputs : max |GPU - oracle| <= 1e-5 on O, LSE, dQ, dK, dV;
                relative norm <= 1e-5 on the per-layer d-alpha vector.
  bf16 inputs : |GPU - oracle| <= 1e-2 + ulp_bf16(oracle)/2 elementwise on O
                -- the 1e-2 bound applies to the computation, and O is stored
                in bf16, whose rounding alone reaches 0.0078 for |O| in [2, 4)
                and 0.0156 in [4, 8); max |GPU - oracle| <= 1e-2 on LSE (fp32); relative Frobenius norm <= 5e-2 on dQ, dK, dV and
                on the per-layer d-alpha vector.  The LSE bound follows from
                the staged kernels keeping rotated K rows in bf16: a relative
                rounding of 2^-9 per element gives score errors of about
                2^-9/sqrt(3) * |q_hat o k| ~ 1e-3 for N(0,1) inputs, a few 1e-3
                at the worst of ~1e5 queries.
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


def check_fwd(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what=""):
    tol = TOL[dtype]
    o_gpu, lse_gpu = to_np(o_gpu), to_np(lse_gpu)
    assert np.array_equal(np.isnan(o_gpu), np.isnan(o_ref)), f"{what}: NaN pattern of O"
    fin = ~np.isnan(o_ref)
    store = half_ulp_bf16(o_ref) if dtype == torch.bfloat16 else 0.0
    excess = (np.abs(o_gpu - o_ref) - store)[fin]
    err_o = excess.max(initial=0.0)
    err_l = np.abs(lse_gpu - lse_ref)[~np.isnan(lse_ref)].max(initial=0.0)
    assert err_o <= tol["o_abs"], f"{what}: O max abs err beyond bf16 storage {err_o:.3e}"
    assert err_l <= tol["lse_abs"], f"{what}: LSE max abs err {err_l:.3e}"
    return err_o, err_l


def check_bwd(gpu, ref, dtype, what=""):
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
    out["dalpha"] = check_dalpha(gpu[3], ref[3], dtype, what)
    return out


def check_dalpha(dal_gpu, dal_ref, dtype, what=""):
    """Relative norm of the per-layer d-alpha vector.  Each layer's value is a
    sum of per-(batch, head) terms that are large (about 1e4 for the learned-
    alpha workload) and of both signs, so a single layer's total can cancel to
    a value far below its terms (layer 0 of that workload: -72.7, next to
    1e5-scale layers); the norm over layers is the well-conditioned measure."""
    tol = TOL[dtype]
    dal_g, dal_r = to_np(dal_gpu), np.asarray(dal_ref, np.float64)
    fin = ~np.isnan(dal_r)
    assert np.array_equal(np.isnan(dal_g), ~fin), f"{what}: NaN pattern of dalpha"
    if not fin.any():
        return 0.0
    e = float(np.linalg.norm(dal_g[fin] - dal_r[fin]) / max(np.linalg.norm(dal_r[fin]), 1e-3))
    assert e <= tol["dal_rel"], f"{what}: dalpha rel-norm err {e:.3e} ({dal_g} vs {dal_r})"
    return e


def oracle_fwd(q, k, v, alpha, **kw):
    return oracle.fwd(to_np(q), to_np(k), to_np(v), to_np(alpha).astype(np.float32), **kw)


def oracle_bwd(q, k, v, dout, alpha, **kw):
    return oracle.bwd(to_np(q), to_np(k), to_np(v), to_np(dout),
                      to_np(alpha).astype(np.float32), **kw)
