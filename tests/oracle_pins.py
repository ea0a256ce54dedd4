"""Pins of the CPU oracle against what the page and the mathematics fix.

Every pin takes an ``Oracle`` instance, so the same checks run on the default
build (tests/test_oracle_pins.py) and on deliberately mutated copies of the
oracle's source (tests/test_oracle_mutants.py), which must each fail one pin.

Page: "Depth-Staggered Fibonacci Spacing for Sparse Attention" (C. A. Capps),
technical summary, Methodology ("Attended set", "Scaling", "Implementation")
and "Experimental variables".
"""
import os

import numpy as np

from independent import dense_causal, integer_gather, multiset_bias, prior_bias, rope_complex

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden_offsets():
    with open(os.path.join(GOLDEN, "fibonacci_offsets.txt")) as f:
        rows = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    return tuple(int(x) for x in rows[0].split())


def golden_alpha_schedules():
    out = []
    with open(os.path.join(GOLDEN, "alpha_schedules.txt")) as f:
        for ln in f:
            if ln.strip() and not ln.startswith("#"):
                l, a, src = ln.split()
                out.append((int(l), float(a), int(src)))
    return out


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _close(a, b, atol, rtol=0.0, what=""):
    a, b = np.asarray(a), np.asarray(b)
    err = np.abs(a - b)
    lim = atol + rtol * np.abs(b)
    assert np.all(err <= lim), f"{what}: max err {err.max():.3e} (limit {lim.max():.3e})"


FIB = golden_offsets()


# -- geometry ("Scaling": d_k = alpha f_k; interpolation and drop readings) ----

def pin_geometry(orc):
    for f in FIB:                       # integer alpha: no interpolation
        assert orc.geometry(1.0, f) == (True, f, 0.0, f)
        assert orc.geometry(2.0, f) == (True, 2 * f, 0.0, 2 * f)
    assert orc.geometry(0.5, 1) == (True, 0, 0.5, 1)      # d = 0.5: rows i, i-1
    assert orc.geometry(0.5, 2) == (True, 1, 0.0, 1)
    assert orc.geometry(0.5, 3) == (True, 1, 0.5, 2)
    assert orc.geometry(1.5, 987) == (True, 1480, 0.5, 1481)
    assert orc.geometry(0.0, 5) == (True, 0, 0.0, 0)
    for a in (np.float32(0.5 + 1 / 15), np.float32(1.1), np.float32(1.0333334)):
        for f in FIB:                   # d is one fp32 product
            d = np.float32(a) * np.float32(f)
            lo = int(np.floor(d))
            ok, glo, gw, gc = orc.geometry(float(a), f)
            assert ok and glo == lo and gc == int(np.ceil(d))
            assert gw == float(d - np.float32(lo))
    for bad in (float("nan"), -1.0, 1e30):
        assert not orc.geometry(bad, 3)[0]


def pin_schedules():
    """The golden schedule table against its stated closed forms."""
    sched = golden_alpha_schedules()
    assert [s[0] for s in sched] == list(range(16))
    assert abs(sched[0][1] - 0.5) < 1e-15 and abs(sched[15][1] - 1.5) < 1e-15
    for l, a, _ in sched:
        assert abs(a - (0.5 + l / 15)) < 1e-15
    src = [s[2] for s in sched]
    assert sorted(src) == list(range(16))            # a permutation
    assert all(src[src[l]] == l for l in range(16))  # 7*7 = 49 = 1 mod 16: self-inverse
    assert FIB[:4] == (1, 2, 3, 5) and FIB[-1] == 987 and len(FIB) == 15
    assert all(FIB[k + 1] == FIB[k] + FIB[k - 1] for k in range(1, 14))


# -- RoPE ("RoPE before the gather") -------------------------------------------

def pin_rope(orc):
    x = _rand((16,), 1)
    assert np.allclose(orc.rope(x, 0), x, atol=0, rtol=0)
    for pos in (1, 7, 1000, 32767):
        r = orc.rope(x, pos)
        assert abs(np.linalg.norm(r) - np.linalg.norm(x)) < 1e-12
        ref = rope_complex(np.stack([x] * (pos + 1)))[pos] if pos < 2000 else None
        if ref is not None:
            _close(r, ref, 1e-12, what="rope vs complex form")
    # relative-position property: <R(q,i), R(k,j)> depends on i - j only
    q, k = _rand((16,), 2), _rand((16,), 3)
    base = orc.rope(q, 9) @ orc.rope(k, 4)
    for s in (1, 50, 999):
        assert abs(orc.rope(q, 9 + s) @ orc.rope(k, 4 + s) - base) < 1e-10
    # frequencies: D=4, unit vector on dim 1 turns at theta_1 = base^(-1/2) = 0.01
    e1 = np.array([0.0, 1.0, 0.0, 0.0])
    for pos in (1, 3, 100):
        r = orc.rope(e1, pos)
        _close(r, [0.0, np.cos(0.01 * pos), 0.0, np.sin(0.01 * pos)], 1e-14, what="rope freq")


# -- forward special cases -----------------------------------------------------

def pin_dense_limit(orc):
    """W >= T, no offsets, no sinks: plain dense causal attention."""
    q, k, v = (_rand((1, 1, 2, 37, 8), s) for s in (10, 11, 12))
    o, lse = orc.fwd(q, k, v, [1.0], window=37, offsets=())
    o_ref, lse_ref = dense_causal(q, k, v)
    _close(o, o_ref, 1e-12, what="dense O")
    _close(lse, lse_ref, 1e-12, what="dense LSE")
    o2, _ = orc.fwd(q, k, v, [1.0], window=50, offsets=(), scale=0.3)
    _close(o2, dense_causal(q, k, v, scale=0.3)[0], 1e-12, what="dense O, scale")


def pin_integer_gather(orc):
    """alpha = 1 (and 2): the interpolated gather equals an exact integer gather."""
    q, k, v = (_rand((1, 1, 2, 64, 16), s) for s in (20, 21, 22))
    for alpha, sinks, window in ((1.0, 0, 6), (1.0, 4, 5), (2.0, 2, 3)):
        o, lse = orc.fwd(q, k, v, [alpha], window=window, sinks=sinks, offsets=FIB)
        o_ref, lse_ref = integer_gather(q, k, v, window=window, sinks=sinks,
                                        dists=[int(alpha) * f for f in FIB])
        _close(o, o_ref, 1e-12, what=f"integer gather O alpha={alpha}")
        _close(lse, lse_ref, 1e-12, what=f"integer gather LSE alpha={alpha}")


def pin_multiset(orc):
    """Integer distances: the sparse set equals dense causal attention with a
    log-multiplicity bias (duplicates from window/offset/sink overlaps kept)."""
    T = 50
    q, k, v = (_rand((1, 1, 1, T, 8), s) for s in (30, 31, 32))
    for alpha, window, sinks in ((1.0, 4, 3), (1.0, 12, 0), (3.0, 2, 5)):
        dists = [int(alpha) * f for f in FIB]
        o, lse = orc.fwd(q, k, v, [alpha], window=window, sinks=sinks)
        bias = multiset_bias(T, window=window, dists=dists, sinks=sinks)
        o_ref, lse_ref = dense_causal(q, k, v, bias=bias)
        _close(o, o_ref, 1e-12, what="multiset O")
        _close(lse, lse_ref, 1e-12, what="multiset LSE")


def pin_softmax(orc):
    """Weights are >= 0 and sum to 1; members that do not exist weigh 0."""
    q, k, v = (_rand((3, 1, 2, 40, 8), s) for s in (40, 41, 42))
    alpha = np.float32([0.5, 1.0, 1.37])
    W, S = 5, 2
    _, _, p = orc.fwd(q, k, v, alpha, window=W, sinks=S, want_probs=True)
    assert np.all(p >= 0)
    _close(p.sum(-1), np.ones(p.shape[:-1]), 1e-12, what="sum p")
    for i in range(40):
        for t in range(W):                      # window slot t exists iff i-t >= 0
            assert (p[..., i, t] > 0).all() == (i - t >= 0)
        for s in range(S):
            assert (p[..., i, W + s] > 0).all() == (s <= i)
    # worked example, alpha = 1, query 2: offsets 1 and 2 exist, 3 is dropped
    assert (p[1, ..., 2, W + S + 0] > 0).all() and (p[1, ..., 2, W + S + 1] > 0).all()
    assert (p[1, ..., 2, W + S + 2:] == 0).all()
    # alpha = 0.5: f=1 -> d=0.5 needs rows i and i-1, so it exists from i = 1
    assert (p[0, ..., 0, W + S + 0] == 0).all() and (p[0, ..., 1, W + S + 0] > 0).all()


def pin_constant_v(orc):
    """Every V row equal to c: O = c, interpolated members included."""
    q, k = (_rand((4, 1, 1, 60, 8), s) for s in (50, 51))
    c = _rand((8,), 52)
    v = np.broadcast_to(c, (4, 1, 1, 60, 8))
    o, _ = orc.fwd(q, k, v, np.float32([0.5, 0.77, 1.21, 1.5]), window=3, sinks=1)
    _close(o, np.broadcast_to(c, o.shape), 1e-12, what="constant V")


def pin_interp_continuity(orc):
    """As alpha*f approaches an integer n, the interpolated member approaches
    the integer gather at distance n.  From below (lo = n-1, w -> 1) the weight
    moves onto row i-n and the member exists from i = n, as in the integer
    gather.  From above (lo = n, w -> 0) it needs row i-n-1, so by the drop
    rule it exists only from i = n+1; at i = n the query sees the window alone.
    Together these fix the direction of interpolation and the drop rule."""
    q, k, v = (_rand((1, 1, 2, 30, 8), s) for s in (60, 61, 62))
    f, n = 5, 7
    o_int, _ = integer_gather(q, k, v, window=2, dists=[n])
    o_win, _ = integer_gather(q, k, v, window=2, dists=[])
    ref = {-1: o_int, 1: o_int.copy()}
    ref[1][..., n, :] = o_win[..., n, :]
    errs = {}
    for eps in (1e-3, 1e-4):
        for side in (-1, 1):
            a = np.float32(n / f + side * eps)
            o, _ = orc.fwd(q, k, v, [a], window=2, offsets=(f,))
            errs[(eps, side)] = np.abs(o - ref[side]).max()
    for side in (-1, 1):
        assert errs[(1e-3, side)] < 0.05, errs
        assert errs[(1e-4, side)] < errs[(1e-3, side)] / 4, errs   # O(eps) convergence


def pin_nan_geometry(orc):
    q, k, v = (_rand((2, 1, 1, 20, 8), s) for s in (70, 71, 72))
    o, lse = orc.fwd(q, k, v, np.float32([np.nan, 1.0]), window=3)
    assert np.isnan(o[0]).all() and np.isnan(lse[0]).all()
    assert np.isfinite(o[1]).all() and np.isfinite(lse[1]).all()
    o, _ = orc.fwd(q, k, v, np.float32([-1.0, 1.0]), window=3)
    assert np.isnan(o[0]).all() and np.isfinite(o[1]).all()
    dq, dk, dv, dal = orc.bwd(q, k, v, q, np.float32([np.nan, 1.0]), window=3)
    assert np.isnan(dq[0]).all() and np.isnan(dk[0]).all() and np.isnan(dv[0]).all()
    assert np.isnan(dal[0]) and np.isfinite(dal[1])


def pin_fp32_build(orc):
    """The fp32 build computes the same function to fp32 accuracy."""
    q, k, v = (_rand((2, 1, 2, 64, 16), s) for s in (80, 81, 82))
    al = np.float32([0.63, 1.47])
    o64, l64 = orc.fwd(q, k, v, al, window=6, sinks=2)
    o32, l32 = orc.fwd(q, k, v, al, window=6, sinks=2, precision="f32")
    _close(o32, o64, 2e-6, what="fp32 O")
    _close(l32, l64, 2e-6, what="fp32 LSE")
    d64 = orc.bwd(q, k, v, o64, al, window=6, sinks=2)
    d32 = orc.bwd(q, k, v, o64, al, window=6, sinks=2, precision="f32")
    for a, b, name in zip(d32, d64, ("dq", "dk", "dv", "dalpha")):
        _close(a, b, 5e-5, 1e-5, what=f"fp32 {name}")


# -- backward (finite differences of sum(dO * O), fp64) ------------------------

FD_ALPHA = np.float32([1.1234, 0.6789])   # every alpha*f (f*alpha <= 40) is >= 1e-2 from an integer
FD_KW = dict(window=3, sinks=1)


def _fd_problem():
    shape = (2, 1, 2, 40, 8)
    q, k, v, do = (_rand(shape, s) for s in (90, 91, 92, 93))
    return q, k, v, do


def pin_fd_inputs(orc):
    q, k, v, do = _fd_problem()
    dq, dk, dv, _ = orc.bwd(q, k, v, do, FD_ALPHA, **FD_KW)
    h = 1e-6

    def loss(qq, kk, vv):
        return float((orc.fwd(qq, kk, vv, FD_ALPHA, **FD_KW)[0] * do).sum())

    rng = np.random.default_rng(5)
    for name, grad, which in (("dQ", dq, 0), ("dK", dk, 1), ("dV", dv, 2)):
        idxs = [tuple(rng.integers(0, s) for s in q.shape) for _ in range(60)]
        idxs += [(0, 0, 0, 0, 0), (1, 0, 1, 39, 7), (0, 0, 1, 1, 3)]
        for idx in idxs:
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 + 1e-6 * abs(fd), (name, idx, fd, grad[idx])


def pin_fd_alpha(orc):
    """dalpha per layer, and each (layer, batch, head) unit's share of it,
    against central finite differences of sum(dO * O) (the unit's share: of
    that unit's part of the sum alone)."""
    q, k, v, do = _fd_problem()
    _, _, _, dal, dun = orc.bwd(q, k, v, do, FD_ALPHA, dalpha_units=True, **FD_KW)
    for l in range(2):
        for h in (3e-4,):
            ap, am = FD_ALPHA.copy(), FD_ALPHA.copy()
            ap[l] = np.float32(FD_ALPHA[l] + h)
            am[l] = np.float32(FD_ALPHA[l] - h)
            op = orc.fwd(q, k, v, ap, **FD_KW)[0] * do
            om = orc.fwd(q, k, v, am, **FD_KW)[0] * do
            da = float(ap[l]) - float(am[l])
            fd = (float(op.sum()) - float(om.sum())) / da
            assert abs(fd - dal[l]) <= 2e-3 * abs(fd) + 1e-6, (l, fd, dal[l])
            for b in range(q.shape[1]):
                for hh in range(q.shape[2]):
                    fu = (float(op[l, b, hh].sum()) - float(om[l, b, hh].sum())) / da
                    assert abs(fu - dun[l, b, hh]) <= 2e-3 * abs(fu) + 1e-6, (l, b, hh, fu)


# -- learned-alpha map ---------------------------------------------------------

def pin_theta_map(orc):
    """alpha = 0.5 + sigmoid(theta): theta = 0 is the initialisation alpha = 1,
    theta = +-ln 3 gives 1.25 / 0.75 (sigmoid = 3/4, 1/4), alpha stays inside
    [0.5, 1.5] and increases with theta; dtheta = dalpha * s (1 - s) equals a
    central finite difference of the oracle's loss through alpha(theta)."""
    th = np.array([0.0, np.log(3.0), -np.log(3.0), 40.0, -40.0, 0.3])
    a = orc.alpha_from_theta(th)
    _close(a[:3], [1.0, 1.25, 0.75], 1e-15, what="alpha(theta) closed forms")
    assert (a >= 0.5).all() and (a <= 1.5).all()
    grid = np.linspace(-8, 8, 101)
    assert (np.diff(orc.alpha_from_theta(grid)) > 0).all()
    # chain rule through the whole forward: theta chosen so alpha(theta) = FD_ALPHA
    q, k, v, do = _fd_problem()
    theta = -np.log(1.0 / (FD_ALPHA.astype(np.float64) - 0.5) - 1.0)
    alpha = orc.alpha_from_theta(theta).astype(np.float32)
    _close(alpha, FD_ALPHA, 1e-7, what="alpha(theta) round trip")
    _, _, _, dal = orc.bwd(q, k, v, do, alpha, **FD_KW)
    dth = orc.dtheta(theta, dal)
    for l in range(2):
        h = 1e-3
        tp, tm = theta.copy(), theta.copy()
        tp[l] += h
        tm[l] -= h
        ap = orc.alpha_from_theta(tp).astype(np.float32)
        am = orc.alpha_from_theta(tm).astype(np.float32)
        lp = float((orc.fwd(q, k, v, ap, **FD_KW)[0] * do).sum())
        lm = float((orc.fwd(q, k, v, am, **FD_KW)[0] * do).sum())
        # the fp32 rounding of alpha moves the step slightly: divide by the
        # theta step that the rounded alphas correspond to
        s = lambda x: 1.0 / (1.0 + np.exp(-x))
        fd = (lp - lm) / (float(ap[l]) - float(am[l])) * (s(tp[l]) - s(tm[l])) / (2 * h)
        assert abs(fd - dth[l]) <= 2e-3 * abs(fd) + 1e-6, (l, fd, dth[l])


# -- single-token decode ------------------------------------------------------

def pin_decode_dense_and_gather(orc):
    """Decode at pos = the attended set of query pos: with W > pos and no
    offsets it is row pos of plain dense causal attention; at alpha = 1 it is
    row pos of the exact integer gather; rows after pos (NaN here) are never
    read; and it matches row pos of the oracle forward with interpolation."""
    L, B, H, T, D = 1, 1, 2, 70, 16
    q, k, v = (_rand((L, B, H, T, D), s) for s in (70, 71, 72))
    for pos in (0, 9, 40, 69):
        kc, vc = k.copy(), v.copy()
        kc[..., pos + 1:, :] = np.nan
        vc[..., pos + 1:, :] = np.nan
        q1 = q[..., pos, :]
        o, lse = orc.decode(q1, kc, vc, [1.0], pos, window=T + 5, offsets=())
        o_ref, lse_ref = dense_causal(q[..., :pos + 1, :], k[..., :pos + 1, :], v[..., :pos + 1, :])
        _close(o, o_ref[..., pos, :], 1e-12, what=f"decode dense O pos={pos}")
        _close(lse, lse_ref[..., pos], 1e-12, what=f"decode dense LSE pos={pos}")
        o, lse = orc.decode(q1, kc, vc, [1.0], pos, window=6, sinks=2, offsets=FIB)
        o_ref, lse_ref = integer_gather(q[..., :pos + 1, :], k[..., :pos + 1, :],
                                        v[..., :pos + 1, :], window=6, sinks=2, dists=list(FIB))
        _close(o, o_ref[..., pos, :], 1e-12, what=f"decode gather O pos={pos}")
        _close(lse, lse_ref[..., pos], 1e-12, what=f"decode gather LSE pos={pos}")
        for alpha in (0.63, 1.37):
            o, lse = orc.decode(q1, kc, vc, [alpha], pos, window=5, sinks=1, offsets=FIB)
            of, lf = orc.fwd(q[..., :pos + 1, :], k[..., :pos + 1, :], v[..., :pos + 1, :],
                             [alpha], window=5, sinks=1, offsets=FIB)
            _close(o, of[..., pos, :], 1e-12, what=f"decode vs forward alpha={alpha}")
            _close(lse, lf[..., pos], 1e-12, what=f"decode vs forward LSE alpha={alpha}")
        # with a log-prior: row pos of the forward whose query pos has that prior
        beta = _rand((L, B, H, pos + 1), 73 + pos)
        o, lse = orc.decode(q1, kc, vc, [0.91], pos, window=4, offsets=FIB, beta=beta[..., pos])
        of, lf = orc.fwd(q[..., :pos + 1, :], k[..., :pos + 1, :], v[..., :pos + 1, :], [0.91],
                         window=4, offsets=FIB, beta=beta)
        _close(o, of[..., pos, :], 1e-12, what=f"decode with a prior pos={pos}")
        _close(lse, lf[..., pos], 1e-12, what=f"decode with a prior, LSE pos={pos}")


# -- log-prior on the offset members (pi-Attention's fusion in one softmax) ---

def pin_log_prior_dense(orc):
    """Integer distances with a per-query log-prior beta on the offset members:
    dense causal attention whose bias gives key j of query i the weight
    (local multiplicity) + (offset multiplicity) * e^beta_i."""
    T = 60
    q, k, v = (_rand((1, 1, 2, T, 8), s) for s in (130, 131, 132))
    beta = 1.5 * _rand((1, 1, 2, T), 133)
    for alpha, window, sinks in ((1.0, 4, 2), (2.0, 3, 0)):
        dists = [int(alpha) * f for f in FIB]
        o, lse = orc.fwd(q, k, v, [alpha], window=window, sinks=sinks, beta=beta)
        bias = prior_bias(beta, window=window, dists=dists, sinks=sinks)
        o_ref, lse_ref = dense_causal(q, k, v, bias=bias)
        _close(o, o_ref, 1e-12, what=f"log-prior O alpha={alpha}")
        _close(lse, lse_ref, 1e-12, what=f"log-prior LSE alpha={alpha}")


def pin_log_prior_limits(orc):
    """beta = ln 2 counts every offset member twice (the offset list given
    twice, duplicates kept); beta = -800 (e^beta = 0 in fp64) removes the
    offsets: forward and backward equal the oracle without offsets, and dbeta
    is 0.  Interpolated alphas."""
    q, k, v, do = (_rand((2, 1, 1, 45, 8), s) for s in (140, 141, 142, 143))
    alpha = np.float32([0.73, 1.41])
    kw = dict(window=4, sinks=1)
    ln2 = np.full((2, 1, 1, 45), np.log(2.0))
    o, lse = orc.fwd(q, k, v, alpha, beta=ln2, **kw)
    o2, lse2 = orc.fwd(q, k, v, alpha, offsets=FIB + FIB, **kw)
    _close(o, o2, 1e-12, what="beta = ln 2 vs doubled offsets, O")
    _close(lse, lse2, 1e-12, what="beta = ln 2 vs doubled offsets, LSE")
    g = orc.bwd(q, k, v, do, alpha, beta=ln2, **kw)
    g2 = orc.bwd(q, k, v, do, alpha, offsets=FIB + FIB, **kw)
    for name, a, b in zip(("dQ", "dK", "dV", "dalpha"), g[:4], g2):
        _close(a, b, 1e-11, 1e-11, what=f"beta = ln 2 vs doubled offsets, {name}")
    off = np.full((2, 1, 1, 45), -800.0)
    o, lse = orc.fwd(q, k, v, alpha, beta=off, **kw)
    o0, lse0 = orc.fwd(q, k, v, alpha, offsets=(), **kw)
    _close(o, o0, 1e-12, what="beta = -800 vs no offsets, O")
    _close(lse, lse0, 1e-12, what="beta = -800 vs no offsets, LSE")
    g = orc.bwd(q, k, v, do, alpha, beta=off, **kw)
    g0 = orc.bwd(q, k, v, do, alpha, offsets=(), **kw)
    for name, a, b in zip(("dQ", "dK", "dV", "dalpha"), g[:4], g0):
        _close(a, b, 1e-12, what=f"beta = -800 vs no offsets, {name}")
    assert np.all(g[4] == 0.0), "dbeta with vanishing offset weights"


def pin_fd_beta(orc):
    """Central finite differences of sum(dO * O) for dbeta and, with the prior
    present, for dQ, dK, dV and dalpha (interpolated alphas)."""
    q, k, v, do = _fd_problem()
    beta = 0.8 * _rand((2, 1, 2, 40), 150)
    dq, dk, dv, dal, dbeta = orc.bwd(q, k, v, do, FD_ALPHA, beta=beta, **FD_KW)

    def loss(qq, kk, vv, bb, al=FD_ALPHA):
        return float((orc.fwd(qq, kk, vv, al, beta=bb, **FD_KW)[0] * do).sum())

    h = 1e-6
    rng = np.random.default_rng(6)
    idxs = [tuple(rng.integers(0, s) for s in beta.shape) for _ in range(40)]
    idxs += [(0, 0, 0, 0), (1, 0, 1, 39), (0, 0, 1, 2)]
    for idx in idxs:
        bp, bm = beta.copy(), beta.copy()
        bp[idx] += h
        bm[idx] -= h
        fd = (loss(q, k, v, bp) - loss(q, k, v, bm)) / (2 * h)
        assert abs(fd - dbeta[idx]) <= 1e-6 + 1e-6 * abs(fd), ("dbeta", idx, fd, dbeta[idx])
    for name, grad, which in (("dQ", dq, 0), ("dK", dk, 1), ("dV", dv, 2)):
        for idx in [tuple(rng.integers(0, s) for s in q.shape) for _ in range(20)]:
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            fd = (loss(*args_p, beta) - loss(*args_m, beta)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 + 1e-6 * abs(fd), (name, idx, fd, grad[idx])
    for l in range(2):
        ap, am = FD_ALPHA.copy(), FD_ALPHA.copy()
        ap[l] = np.float32(FD_ALPHA[l] + 3e-4)
        am[l] = np.float32(FD_ALPHA[l] - 3e-4)
        fd = (loss(q, k, v, beta, ap) - loss(q, k, v, beta, am)) / (float(ap[l]) - float(am[l]))
        assert abs(fd - dal[l]) <= 2e-3 * abs(fd) + 1e-6, ("dalpha", l, fd, dal[l])


ALL_PINS = [pin_geometry, pin_rope, pin_dense_limit, pin_integer_gather, pin_multiset,
            pin_softmax, pin_constant_v, pin_interp_continuity, pin_nan_geometry,
            pin_fp32_build, pin_fd_inputs, pin_fd_alpha, pin_theta_map,
            pin_decode_dense_and_gather, pin_log_prior_dense, pin_log_prior_limits,
            pin_fd_beta]
