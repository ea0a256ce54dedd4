"""Independent restatements used to pin the oracle (numpy, fp64).

None of this shares code with the oracle: each function computes a special
case of the method through a different formulation, so that a mistake in the
oracle's loops (a dropped term, a wrong sign or index, a swapped operand)
shows up as a disagreement.

  rope_complex      -- RoPE as multiplication of complex pairs by e^{i*pos*theta}
                       (the textbook rotary form; rotate-half pairing).
  dense_causal      -- matrix-form causal softmax attention with an optional
                       additive score bias (the textbook routine).
  integer_gather    -- the attended set written as a list of integer row
                       indices per query, no interpolation.
  multiset_bias     -- log-multiplicity bias that turns dense causal attention
                       into the sparse attended set when every distance is an
                       integer (duplicates counted).
  prior_bias        -- the same with a per-query log-prior on the offset
                       members: key j of query i weighs
                       (local multiplicity) + (offset multiplicity) * e^beta_i.
"""
import numpy as np


def rope_complex(x, base=10000.0):
    """x: [..., T, D]; row t is rotated by angle t * theta_j on pair (j, j+D/2)."""
    x = np.asarray(x, dtype=np.float64)
    T, D = x.shape[-2], x.shape[-1]
    h = D // 2
    theta = base ** (-np.arange(h, dtype=np.float64) * 2.0 / D)
    ang = np.arange(T, dtype=np.float64)[:, None] * theta[None, :]
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * ang)
    return np.concatenate([z.real, z.imag], axis=-1)


def _scale(D, scale):
    return scale if scale and scale > 0 else 1.0 / np.sqrt(D)


def dense_causal(q, k, v, *, base=10000.0, scale=0.0, bias=None):
    """Causal softmax attention over all keys j <= i. q,k,v: [..., T, D].

    bias: optional [T, T] additive score bias (-inf removes a key).
    Returns (O, LSE) in fp64.
    """
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    T, D = q.shape[-2], q.shape[-1]
    s = _scale(D, scale)
    qr = rope_complex(q, base) * s
    kr = rope_complex(k, base)
    scores = qr @ np.swapaxes(kr, -1, -2)
    mask = np.tril(np.ones((T, T), dtype=bool))
    scores = np.where(mask, scores, -np.inf)
    if bias is not None:
        scores = scores + bias
    m = scores.max(axis=-1, keepdims=True)
    e = np.exp(scores - m)
    z = e.sum(axis=-1, keepdims=True)
    return (e / z) @ v, (m + np.log(z))[..., 0]


def integer_gather(q, k, v, *, window, dists, sinks=0, base=10000.0, scale=0.0):
    """Attended set with integer distances: rows i..i-W+1, sinks 0..S-1 (<= i),
    and i - n for each distance n (dropped when i - n < 0).  [..., T, D]."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    lead = q.shape[:-2]
    T, D = q.shape[-2], q.shape[-1]
    s = _scale(D, scale)
    qr = rope_complex(q, base) * s
    kr = rope_complex(k, base)
    O = np.zeros_like(q)
    LSE = np.zeros(lead + (T,))
    for idx in np.ndindex(*lead):
        for i in range(T):
            rows = [i - t for t in range(window) if i - t >= 0]
            rows += [j for j in range(sinks) if j <= i]
            rows += [i - n for n in dists if i - n >= 0]
            sc = kr[idx][rows] @ qr[idx][i]
            m = sc.max()
            e = np.exp(sc - m)
            O[idx + (i,)] = (e / e.sum()) @ v[idx][rows]
            LSE[idx + (i,)] = m + np.log(e.sum())
    return O, LSE


def multiset_bias(T, *, window, dists, sinks=0):
    """[T, T] bias log(count_ij), count = multiplicity of key j in query i's set
    (window, sinks, integer distances; duplicates counted); -inf where 0."""
    cnt = np.zeros((T, T))
    for i in range(T):
        for t in range(window):
            if i - t >= 0:
                cnt[i, i - t] += 1
        for j in range(sinks):
            if j <= i:
                cnt[i, j] += 1
        for n in dists:
            if i - n >= 0:
                cnt[i, i - n] += 1
    with np.errstate(divide="ignore"):
        return np.log(cnt)


def prior_bias(beta, *, window, dists, sinks=0):
    """[..., T, T] bias log(c_local_ij + c_offset_ij * exp(beta_i)) for
    beta [..., T]: local = window and sinks, offset = integer distances
    (duplicates counted); -inf where key j is not attended."""
    beta = np.asarray(beta, dtype=np.float64)
    T = beta.shape[-1]
    loc = np.zeros((T, T))
    off = np.zeros((T, T))
    for i in range(T):
        for t in range(window):
            if i - t >= 0:
                loc[i, i - t] += 1
        for j in range(sinks):
            if j <= i:
                loc[i, j] += 1
        for n in dists:
            if i - n >= 0:
                off[i, i - n] += 1
    w = loc + off * np.exp(beta)[..., :, None]
    with np.errstate(divide="ignore"):
        return np.log(w)
