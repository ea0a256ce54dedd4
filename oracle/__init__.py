"""CPU oracle for structured sparse causal attention with Fibonacci offsets.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg import this package; the library's product path
never does, and it shares no code with the CUDA library.

The arithmetic lives in ``oracle_attn.c`` (plain loops, see its header for the
passages of "Depth-Staggered Fibonacci Spacing for Sparse Attention" it
follows and the readings it takes).  This module only marshals numpy arrays.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
except the RoPE pairing convention (rotate-half versus interleaved pairs),
which the page does not fix: parity unpinned for that choice alone.
"""
import ctypes
import os

import numpy as np

from .build import build as _build

FIB15 = (1, 2, 3, 5, 8, 13, 21, 34, 55, 89, 144, 233, 377, 610, 987)


def _np_dtype(precision):
    if precision == "f64":
        return np.float64, ctypes.c_double
    if precision == "f32":
        return np.float32, ctypes.c_float
    raise ValueError(precision)


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _prep(x, dt):
    return np.ascontiguousarray(np.asarray(x, dtype=dt))


class Oracle:
    """ctypes view of one build of oracle_attn.c (the default build, or a
    deliberately mutated copy that the mutation tests compile)."""

    def __init__(self, path):
        lib = ctypes.CDLL(path)
        for suffix, ctype in (("_f64", ctypes.c_double), ("_f32", ctypes.c_float)):
            P = ctypes.POINTER(ctype)
            head = [ctypes.c_int] * 7 + [ctypes.POINTER(ctypes.c_int32), ctypes.c_int,
                                         ctypes.c_double, ctypes.c_double,
                                         ctypes.POINTER(ctypes.c_float)]
            fwd = getattr(lib, "oracle_fwd" + suffix)
            fwd.restype = ctypes.c_int
            fwd.argtypes = head + [P] * 7
            bwd = getattr(lib, "oracle_bwd" + suffix)
            bwd.restype = ctypes.c_int
            bwd.argtypes = head + [P] * 11
            geo = getattr(lib, "oracle_geometry" + suffix)
            geo.restype = ctypes.c_int
            geo.argtypes = [ctypes.c_float, ctypes.c_int32, ctypes.POINTER(ctypes.c_int64),
                            ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]
            dec = getattr(lib, "oracle_decode" + suffix)
            dec.restype = ctypes.c_int
            dec.argtypes = head + [ctypes.c_int64] + [P] * 6
            a_th = getattr(lib, "oracle_alpha_from_theta" + suffix)
            a_th.restype = None
            a_th.argtypes = [ctypes.c_int, P, P]
            d_th = getattr(lib, "oracle_dtheta" + suffix)
            d_th.restype = None
            d_th.argtypes = [ctypes.c_int, P, P, P]
            rope = getattr(lib, "oracle_rope" + suffix)
            rope.restype = None
            rope.argtypes = [P, ctypes.c_int64, ctypes.c_int, ctypes.c_double, P]
        self.lib = lib
        self.path = path

    def fwd(self, q, k, v, alpha, *, window, offsets=FIB15, sinks=0, rope_base=10000.0,
            scale=0.0, precision="f64", want_probs=False, beta=None):
        """Forward.  q, k, v: [L, B, H, T, D] (upcast); alpha: [L] fp32 values;
        beta: optional [L, B, H, T] log-prior added to every offset member's
        score of each query (None: no prior).

        Returns (O, LSE) or (O, LSE, P), P [L, B, H, T, W+S+n_off] holding each
        member's softmax weight in a fixed slot (window t, sink s, offset k),
        0 where the member does not exist.
        """
        dt, ct = _np_dtype(precision)
        q, k, v = (_prep(x, dt) for x in (q, k, v))
        L, B, H, T, D = q.shape
        assert k.shape == q.shape and v.shape == q.shape
        al = _prep(alpha, np.float32).reshape(-1)
        assert al.shape == (L,)
        offs = np.ascontiguousarray(np.asarray(offsets, dtype=np.int32).reshape(-1))
        o = np.empty_like(q)
        lse = np.empty((L, B, H, T), dtype=dt)
        n_slots = window + sinks + len(offs)
        p = np.empty((L, B, H, T, n_slots), dtype=dt) if want_probs else None
        bt = _prep(beta, dt).reshape(L, B, H, T) if beta is not None else None
        fn = getattr(self.lib, "oracle_fwd_" + precision)
        rc = fn(L, B, H, T, D, int(window), len(offs), _ptr(offs, ctypes.c_int32), int(sinks),
                float(rope_base), float(scale), _ptr(al, ctypes.c_float),
                _ptr(q, ct), _ptr(k, ct), _ptr(v, ct), _ptr(o, ct), _ptr(lse, ct),
                _ptr(p, ct) if p is not None else None,
                _ptr(bt, ct) if bt is not None else None)
        if rc != 0:
            raise ValueError(f"oracle_fwd rejected its arguments (rc={rc})")
        return (o, lse, p) if want_probs else (o, lse)

    def bwd(self, q, k, v, dout, alpha, *, window, offsets=FIB15, sinks=0,
            rope_base=10000.0, scale=0.0, precision="f64", beta=None, dalpha_units=False):
        """Backward for upstream dO: returns (dQ, dK, dV, dalpha[L]), and with
        a log-prior beta [L, B, H, T] also dbeta: (dQ, dK, dV, dalpha, dbeta).
        With dalpha_units=True one more element follows: each (layer, batch,
        head) unit's share of dalpha, [L, B, H] (dalpha[l] is their sum)."""
        dt, ct = _np_dtype(precision)
        q, k, v, dout = (_prep(x, dt) for x in (q, k, v, dout))
        L, B, H, T, D = q.shape
        al = _prep(alpha, np.float32).reshape(-1)
        assert al.shape == (L,)
        offs = np.ascontiguousarray(np.asarray(offsets, dtype=np.int32).reshape(-1))
        dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
        dal = np.empty((L,), dtype=dt)
        bt = _prep(beta, dt).reshape(L, B, H, T) if beta is not None else None
        dbt = np.empty((L, B, H, T), dtype=dt) if beta is not None else None
        dun = np.empty((L, B, H), dtype=dt) if dalpha_units else None
        fn = getattr(self.lib, "oracle_bwd_" + precision)
        rc = fn(L, B, H, T, D, int(window), len(offs), _ptr(offs, ctypes.c_int32), int(sinks),
                float(rope_base), float(scale), _ptr(al, ctypes.c_float),
                _ptr(q, ct), _ptr(k, ct), _ptr(v, ct), _ptr(dout, ct),
                _ptr(dq, ct), _ptr(dk, ct), _ptr(dv, ct), _ptr(dal, ct),
                _ptr(bt, ct) if bt is not None else None,
                _ptr(dbt, ct) if dbt is not None else None,
                _ptr(dun, ct) if dun is not None else None)
        if rc != 0:
            raise ValueError(f"oracle_bwd rejected its arguments (rc={rc})")
        out = (dq, dk, dv, dal, dbt) if beta is not None else (dq, dk, dv, dal)
        return out + (dun,) if dalpha_units else out

    def decode(self, q1, k, v, alpha, pos, *, window, offsets=FIB15, sinks=0,
               rope_base=10000.0, scale=0.0, precision="f64", beta=None):
        """Single-token decode: q1 [L, B, H, D] at position pos against the
        caches k, v [L, B, H, T, D] (rows 0..pos used).  beta: optional
        [L, B, H] log-prior on the new query's offset members.
        Returns (O1, LSE1)."""
        dt, ct = _np_dtype(precision)
        q1, k, v = (_prep(x, dt) for x in (q1, k, v))
        L, B, H, T, D = k.shape
        assert v.shape == k.shape and q1.shape == (L, B, H, D)
        al = _prep(alpha, np.float32).reshape(-1)
        assert al.shape == (L,)
        offs = np.ascontiguousarray(np.asarray(offsets, dtype=np.int32).reshape(-1))
        o = np.empty_like(q1)
        lse = np.empty((L, B, H), dtype=dt)
        bt = _prep(beta, dt).reshape(L, B, H) if beta is not None else None
        fn = getattr(self.lib, "oracle_decode_" + precision)
        rc = fn(L, B, H, T, D, int(window), len(offs), _ptr(offs, ctypes.c_int32), int(sinks),
                float(rope_base), float(scale), _ptr(al, ctypes.c_float), int(pos),
                _ptr(q1, ct), _ptr(k, ct), _ptr(v, ct), _ptr(o, ct), _ptr(lse, ct),
                _ptr(bt, ct) if bt is not None else None)
        if rc != 0:
            raise ValueError(f"oracle_decode rejected its arguments (rc={rc})")
        return o, lse

    def alpha_from_theta(self, theta, precision="f64"):
        """alpha = 0.5 + sigmoid(theta) per layer (the learned-alpha map)."""
        dt, ct = _np_dtype(precision)
        th = _prep(theta, dt).reshape(-1)
        out = np.empty_like(th)
        getattr(self.lib, "oracle_alpha_from_theta_" + precision)(th.shape[0], _ptr(th, ct),
                                                                  _ptr(out, ct))
        return out

    def dtheta(self, theta, dalpha, precision="f64"):
        """Gradient to theta through alpha = 0.5 + sigmoid(theta)."""
        dt, ct = _np_dtype(precision)
        th, da = _prep(theta, dt).reshape(-1), _prep(dalpha, dt).reshape(-1)
        out = np.empty_like(th)
        getattr(self.lib, "oracle_dtheta_" + precision)(th.shape[0], _ptr(th, ct), _ptr(da, ct),
                                                        _ptr(out, ct))
        return out

    def geometry(self, alpha, f):
        """(ok, lo, w, c) of one offset under the oracle's reading."""
        lo, w, c = ctypes.c_int64(), ctypes.c_double(), ctypes.c_int64()
        ok = self.lib.oracle_geometry_f64(ctypes.c_float(alpha), int(f), ctypes.byref(lo),
                                          ctypes.byref(w), ctypes.byref(c))
        return bool(ok), lo.value, w.value, c.value

    def rope(self, x, pos, rope_base=10000.0):
        """RoPE of one row x[D] at integer position pos (fp64)."""
        x = _prep(x, np.float64)
        out = np.empty_like(x)
        self.lib.oracle_rope_f64(_ptr(x, ctypes.c_double), int(pos), x.shape[0],
                                 float(rope_base), _ptr(out, ctypes.c_double))
        return out


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(_build())
    return _default


def fwd(*a, **kw):
    return default().fwd(*a, **kw)


def bwd(*a, **kw):
    return default().bwd(*a, **kw)


def decode(*a, **kw):
    return default().decode(*a, **kw)


def geometry(alpha, f):
    return default().geometry(alpha, f)


def rope(x, pos, rope_base=10000.0):
    return default().rope(x, pos, rope_base)
