"""Structured sparse causal attention with depth-staggered Fibonacci offsets,
for B200 (sm_100a).

Thin ctypes binding over the C ABI in ``include/sparse_attn.h`` (library
``libsparse_attn.so`` built in-tree by ``build.py``).  This module only
marshals arguments: every step of the computation runs in the library's CUDA
kernels.  There is no CPU fallback; if the library is missing or no GPU is
present, the calls raise.

    O, lse = fwd(q, k, v, alpha, window=12)                 # [L, B, H, T, D]
    dq, dk, dv, dalpha = bwd(q, k, v, O, lse, dO, alpha, window=12)

Method: "Depth-Staggered Fibonacci Spacing for Sparse Attention" (C. A.
Capps), technical summary, Methodology -- "Attended set", "Scaling",
"Implementation".
"""
import ctypes
import os

import torch

FIB15 = (1, 2, 3, 5, 8, 13, 21, 34, 55, 89, 144, 233, 377, 610, 987)

_HERE = os.path.dirname(os.path.abspath(__file__))
# The library; SPARSE_ATTN_LIBRARY may name another build of the same sources
# (build.py also writes libsparse_attn_bounds.so, the bounds-checking build).
LIB_PATH = os.environ.get("SPARSE_ATTN_LIBRARY") or os.path.join(_HERE, "libsparse_attn.so")
BOUNDS_LIB_PATH = os.path.join(_HERE, "libsparse_attn_bounds.so")

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE, SA_ERR_CUDA, SA_ERR_INTERNAL = range(6)
SA_DTYPE_F32, SA_DTYPE_BF16 = 0, 1
MAX_OFFSETS = 32
MAX_SINKS = 16

EXPORTED = ("sparse_attn_fwd", "sparse_attn_bwd", "sparse_attn_workspace_size",
            "sparse_attn_status_string", "sparse_attn_last_launch_count",
            "sparse_attn_trace_enable", "sparse_attn_trace_read", "sparse_attn_force_general",
            "sparse_attn_fwd_noalloc", "sparse_attn_device_error", "sparse_attn_select_forward",
            "sparse_attn_context_size", "sparse_attn_fwd_train", "sparse_attn_bwd_ctx",
            "sparse_attn_decode", "sparse_attn_alpha_from_theta", "sparse_attn_dtheta",
            "sparse_attn_fwd_prior", "sparse_attn_bwd_prior", "sparse_attn_decode_prior",
            "sparse_attn_set_wait_limit", "sparse_attn_plant_stall", "sparse_attn_diag_fma_probe")

# Device error word bits (sparse_attn_device_error)
ERR_WAIT, ERR_BOUNDS, ERR_RANGE = 1, 2, 4


class SaParams(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int32), ("B", ctypes.c_int32), ("H", ctypes.c_int32),
                ("T", ctypes.c_int32), ("D", ctypes.c_int32), ("window", ctypes.c_int32),
                ("n_offsets", ctypes.c_int32), ("offsets", ctypes.POINTER(ctypes.c_int32)),
                ("n_sinks", ctypes.c_int32), ("rope_base", ctypes.c_float),
                ("scale", ctypes.c_float), ("dtype", ctypes.c_int32)]


class SparseAttnError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


_lib = None


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m structured_sparse_attention_fibonacci_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(SaParams)
        vp, fp = ctypes.c_void_p, ctypes.c_void_p
        L.sparse_attn_workspace_size.restype = ctypes.c_size_t
        L.sparse_attn_workspace_size.argtypes = [P, ctypes.c_int]
        L.sparse_attn_fwd.restype = ctypes.c_int
        L.sparse_attn_fwd.argtypes = [P, vp, vp, vp, fp, vp, fp, vp, ctypes.c_size_t, vp]
        L.sparse_attn_bwd.restype = ctypes.c_int
        L.sparse_attn_bwd.argtypes = [P, vp, vp, vp, vp, fp, vp, fp, vp, vp, vp, fp, vp,
                                      ctypes.c_size_t, vp]
        L.sparse_attn_fwd_noalloc.restype = ctypes.c_int
        L.sparse_attn_fwd_noalloc.argtypes = [P, vp, vp, vp, fp, vp, fp, vp]
        L.sparse_attn_status_string.restype = ctypes.c_char_p
        L.sparse_attn_status_string.argtypes = [ctypes.c_int]
        L.sparse_attn_last_launch_count.restype = ctypes.c_int32
        L.sparse_attn_last_launch_count.argtypes = []
        L.sparse_attn_force_general.restype = None
        L.sparse_attn_force_general.argtypes = [ctypes.c_int]
        L.sparse_attn_alpha_from_theta.restype = ctypes.c_int
        L.sparse_attn_alpha_from_theta.argtypes = [ctypes.c_int32, fp, fp, vp]
        L.sparse_attn_dtheta.restype = ctypes.c_int
        L.sparse_attn_dtheta.argtypes = [ctypes.c_int32, fp, fp, fp, vp]
        L.sparse_attn_decode.restype = ctypes.c_int
        L.sparse_attn_decode.argtypes = [P, ctypes.c_int32, vp, vp, vp, fp, vp, fp, vp]
        L.sparse_attn_decode_prior.restype = ctypes.c_int
        L.sparse_attn_decode_prior.argtypes = [P, ctypes.c_int32, vp, vp, vp, fp, fp, vp, fp, vp]
        L.sparse_attn_context_size.restype = ctypes.c_size_t
        L.sparse_attn_context_size.argtypes = [P]
        L.sparse_attn_fwd_train.restype = ctypes.c_int
        L.sparse_attn_fwd_train.argtypes = [P, vp, vp, vp, fp, vp, fp, vp, ctypes.c_size_t, vp]
        L.sparse_attn_bwd_ctx.restype = ctypes.c_int
        L.sparse_attn_bwd_ctx.argtypes = [P, vp, vp, vp, vp, fp, vp, fp, vp, vp, vp, vp, fp, vp,
                                          ctypes.c_size_t, vp]
        L.sparse_attn_fwd_prior.restype = ctypes.c_int
        L.sparse_attn_fwd_prior.argtypes = [P, vp, vp, vp, fp, fp, vp, fp, vp, ctypes.c_size_t,
                                            vp, ctypes.c_size_t, vp]
        L.sparse_attn_bwd_prior.restype = ctypes.c_int
        L.sparse_attn_bwd_prior.argtypes = [P, vp, vp, vp, vp, fp, vp, fp, fp, vp, vp, vp, vp, fp,
                                            fp, vp, ctypes.c_size_t, vp]
        L.sparse_attn_select_forward.restype = None
        L.sparse_attn_select_forward.argtypes = [ctypes.c_int]
        L.sparse_attn_device_error.restype = ctypes.c_int32
        L.sparse_attn_device_error.argtypes = [ctypes.c_int]
        L.sparse_attn_set_wait_limit.restype = None
        L.sparse_attn_set_wait_limit.argtypes = [ctypes.c_longlong]
        L.sparse_attn_plant_stall.restype = None
        L.sparse_attn_plant_stall.argtypes = [ctypes.c_int]
        L.sparse_attn_diag_fma_probe.restype = ctypes.c_int
        L.sparse_attn_diag_fma_probe.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                 ctypes.c_int32, fp, vp]
        L.sparse_attn_trace_enable.restype = None
        L.sparse_attn_trace_enable.argtypes = [ctypes.c_int]
        L.sparse_attn_trace_read.restype = ctypes.c_int32
        L.sparse_attn_trace_read.argtypes = [ctypes.c_int32, ctypes.POINTER(ctypes.c_char_p),
                                             ctypes.POINTER(ctypes.c_double),
                                             ctypes.POINTER(ctypes.c_int32)]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().sparse_attn_status_string(status).decode()


def _check(fn, status):
    if status != SA_OK:
        raise SparseAttnError(fn, status, status_string(status))


def make_params(shape, dtype, *, window, offsets=FIB15, sinks=0, rope_base=10000.0, scale=0.0):
    """Build the C parameter block (the offsets array is kept alive on it)."""
    L_, B, H, T, D = shape
    offs = (ctypes.c_int32 * max(1, len(offsets)))(*[int(x) for x in offsets])
    if dtype == torch.float32:
        dt = SA_DTYPE_F32
    elif dtype == torch.bfloat16:
        dt = SA_DTYPE_BF16
    else:
        raise TypeError(f"unsupported dtype {dtype}")
    p = SaParams(L_, B, H, T, D, int(window), len(offsets), offs, int(sinks),
                 float(rope_base), float(scale), dt)
    p._keep = offs
    return p


def workspace_size(shape, dtype, *, backward, **kw) -> int:
    p = make_params(shape, dtype, **kw)
    return int(lib().sparse_attn_workspace_size(ctypes.byref(p), int(bool(backward))))


def last_launch_count() -> int:
    """Kernels enqueued by the latest fwd/bwd call on this thread."""
    return int(lib().sparse_attn_last_launch_count())


def force_general(on: bool = True) -> None:
    """Route every call through the general kernels (diagnostics / testing)."""
    lib().sparse_attn_force_general(int(bool(on)))


def select_forward(which: int = 0) -> None:
    """Diagnostics: bf16 / d=64 forward kernel choice (0 auto, 1 CUDA-core
    staged, 2 tensor-core mma.sync, 3 tensor-core tcgen05); see
    sparse_attn_select_forward."""
    lib().sparse_attn_select_forward(int(which))


def device_error(clear: bool = True) -> int:
    """Device error word of the staged kernels (ERR_WAIT: a bounded staging
    wait gave up; ERR_BOUNDS: a bounds violation seen by the bounds-checking
    build; ERR_RANGE: an input beyond the staged operands' fp16 range);
    synchronises with the device; cleared after reading by default."""
    return int(lib().sparse_attn_device_error(int(bool(clear))))


def fma_probe(out, blocks, threads, iters, packed, stream=None) -> int:
    """Diagnostics: launch the fp32 FMA throughput probe (see
    sparse_attn_diag_fma_probe); out: a float32 CUDA tensor of blocks *
    threads elements.  Returns the probe's FLOPs per launch."""
    if out.dtype != torch.float32 or not out.is_cuda or out.numel() < blocks * threads:
        raise ValueError("out must be a float32 CUDA tensor of blocks * threads elements")
    _check("sparse_attn_diag_fma_probe",
           lib().sparse_attn_diag_fma_probe(int(blocks), int(threads), int(iters), int(packed),
                                            _ptr(out), _stream_handle(stream)))
    return int(blocks) * int(threads) * int(iters) * 8 * 2 * (2 if packed else 1)


def set_wait_limit(clocks: int = 0) -> None:
    """Diagnostics: SM clocks a staging wait waits before giving up (0: default)."""
    lib().sparse_attn_set_wait_limit(int(clocks))


def plant_stall(on: bool = True) -> None:
    """Diagnostics (failure-path test): later staged launches expect 16 bytes
    in their first staging round that no copy delivers, so that wait gives up."""
    lib().sparse_attn_plant_stall(int(bool(on)))


def trace_enable(on: bool = True) -> None:
    """Bracket every library kernel with CUDA events (see sparse_attn_trace_read)."""
    lib().sparse_attn_trace_enable(int(bool(on)))


def trace_read(max_kernels: int = 32):
    """{kernel name: (total ms, launches)} since the last read; waits for the GPU."""
    n = max_kernels
    names = (ctypes.c_char_p * n)()
    ms = (ctypes.c_double * n)()
    ct = (ctypes.c_int32 * n)()
    k = lib().sparse_attn_trace_read(n, names, ms, ct)
    return {names[i].decode(): (ms[i], ct[i]) for i in range(min(k, n))}


def _stream_handle(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _check_tensors(shape, dtype, device, **named):
    for name, t in named.items():
        if t is None:
            continue
        if t.device != device or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous tensor on {device}")
        if name in ("alpha", "dalpha", "lse"):
            if t.dtype != torch.float32:
                raise TypeError(f"{name} must be float32")
        elif tuple(t.shape) != tuple(shape) or t.dtype != dtype:
            raise ValueError(f"{name} must be {dtype} of shape {tuple(shape)}")


def context_size(shape, dtype, **kw) -> int:
    """Bytes of the training context (sparse_attn_context_size); 0 when the
    configuration has no staged kernels."""
    p = make_params(tuple(shape), dtype, **kw)
    return int(lib().sparse_attn_context_size(ctypes.byref(p)))


def _check_prior(shape, dev, **named):
    for name, t in named.items():
        if (t.device != dev or not t.is_contiguous() or t.dtype != torch.float32
                or tuple(t.shape) != tuple(shape[:4])):
            raise ValueError(f"{name} must be a contiguous CUDA fp32 tensor of shape "
                             f"{tuple(shape[:4])}")


def fwd(q, k, v, alpha, *, window, offsets=FIB15, sinks=0, rope_base=10000.0, scale=0.0,
        out=None, lse=None, want_lse=True, stream=None, context=None, beta=None,
        workspace=None):
    """Sparse attention forward over all layers: returns (O, LSE or None).

    q, k, v: CUDA tensors [L, B, H, T, D] (bf16 or fp32, contiguous).
    alpha: CUDA fp32 [L].  Output buffers may be passed in via out= / lse=.
    context: a CUDA uint8 buffer of context_size() bytes: the forward then
    runs as sparse_attn_fwd_train and saves what bwd(..., context=) reuses.
    beta: CUDA fp32 [L, B, H, T], a log-prior added to every offset member's
    score of each query (sparse_attn_fwd_prior).
    workspace: an optional CUDA uint8 buffer of at least
    workspace_size(..., backward=False) bytes (else one is allocated per call).
    """
    if beta is not None:
        return _fwd_prior(q, k, v, alpha, beta, window=window, offsets=offsets, sinks=sinks,
                          rope_base=rope_base, scale=scale, out=out, lse=lse, want_lse=want_lse,
                          stream=stream, context=context)
    if context is not None:
        return _fwd_train(q, k, v, alpha, window=window, offsets=offsets, sinks=sinks,
                          rope_base=rope_base, scale=scale, out=out, lse=lse, want_lse=want_lse,
                          stream=stream, context=context)
    shape, dtype, dev = tuple(q.shape), q.dtype, q.device
    if lse is None and want_lse:
        lse = torch.empty(shape[:4], dtype=torch.float32, device=dev)
    out = torch.empty_like(q) if out is None else out
    _check_tensors(shape, dtype, dev, q=q, k=k, v=v, o=out, alpha=alpha, lse=lse)
    p = make_params(shape, dtype, window=window, offsets=offsets, sinks=sinks,
                    rope_base=rope_base, scale=scale)
    L = lib()
    ws_n = int(L.sparse_attn_workspace_size(ctypes.byref(p), 0))
    if workspace is not None:
        if workspace.device != dev or workspace.numel() * workspace.element_size() < ws_n:
            raise ValueError(f"workspace must be a CUDA buffer of at least {ws_n} bytes")
        ws, ws_n = workspace, workspace.numel() * workspace.element_size()
    else:
        ws = torch.empty(ws_n, dtype=torch.uint8, device=dev) if ws_n else None
    st = L.sparse_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(out),
                           _ptr(lse), _ptr(ws), ws_n, _stream_handle(stream))
    _check("sparse_attn_fwd", st)
    return out, lse


def _fwd_prior(q, k, v, alpha, beta, *, window, offsets, sinks, rope_base, scale, out, lse,
               want_lse, stream, context):
    shape, dtype, dev = tuple(q.shape), q.dtype, q.device
    if lse is None and want_lse:
        lse = torch.empty(shape[:4], dtype=torch.float32, device=dev)
    out = torch.empty_like(q) if out is None else out
    _check_tensors(shape, dtype, dev, q=q, k=k, v=v, o=out, alpha=alpha, lse=lse)
    _check_prior(shape, dev, beta=beta)
    p = make_params(shape, dtype, window=window, offsets=offsets, sinks=sinks,
                    rope_base=rope_base, scale=scale)
    L = lib()
    ws_n = int(L.sparse_attn_workspace_size(ctypes.byref(p), 0)) if context is None else 0
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev) if ws_n else None
    st = L.sparse_attn_fwd_prior(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                 _ptr(beta), _ptr(out), _ptr(lse), _ptr(ws), ws_n, _ptr(context),
                                 context.numel() if context is not None else 0,
                                 _stream_handle(stream))
    _check("sparse_attn_fwd_prior", st)
    return out, lse


def _fwd_train(q, k, v, alpha, *, window, offsets, sinks, rope_base, scale, out, lse, want_lse,
               stream, context):
    shape, dtype, dev = tuple(q.shape), q.dtype, q.device
    if lse is None and want_lse:
        lse = torch.empty(shape[:4], dtype=torch.float32, device=dev)
    out = torch.empty_like(q) if out is None else out
    _check_tensors(shape, dtype, dev, q=q, k=k, v=v, o=out, alpha=alpha, lse=lse)
    p = make_params(shape, dtype, window=window, offsets=offsets, sinks=sinks,
                    rope_base=rope_base, scale=scale)
    st = lib().sparse_attn_fwd_train(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                     _ptr(out), _ptr(lse), _ptr(context), context.numel(),
                                     _stream_handle(stream))
    _check("sparse_attn_fwd_train", st)
    return out, lse


def alpha_from_theta(theta, alpha=None, stream=None):
    """alpha = 0.5 + sigmoid(theta) per layer (the learned-alpha map); CUDA fp32 [L]."""
    alpha = torch.empty_like(theta) if alpha is None else alpha
    if theta.dtype != torch.float32 or alpha.dtype != torch.float32 or not theta.is_cuda:
        raise ValueError("theta and alpha must be CUDA fp32 tensors")
    st = lib().sparse_attn_alpha_from_theta(theta.numel(), _ptr(theta), _ptr(alpha),
                                            _stream_handle(stream))
    _check("sparse_attn_alpha_from_theta", st)
    return alpha


def dtheta(theta, dalpha, out=None, stream=None):
    """Gradient to theta from dalpha through alpha = 0.5 + sigmoid(theta)."""
    out = torch.empty_like(theta) if out is None else out
    for t in (theta, dalpha, out):
        if t.dtype != torch.float32 or not t.is_cuda:
            raise ValueError("theta, dalpha and dtheta must be CUDA fp32 tensors")
    st = lib().sparse_attn_dtheta(theta.numel(), _ptr(theta), _ptr(dalpha), _ptr(out),
                                  _stream_handle(stream))
    _check("sparse_attn_dtheta", st)
    return out


def decode(q, k_cache, v_cache, alpha, pos, *, window, offsets=FIB15, sinks=0,
           rope_base=10000.0, scale=0.0, out=None, lse=None, want_lse=True, stream=None,
           beta=None):
    """Single-token decode: q [L, B, H, D] at position pos against the caches
    k_cache, v_cache [L, B, H, T_cache, D] (rows 0..pos hold the sequence,
    row pos the new token).  beta: optional CUDA fp32 [L, B, H] log-prior on
    the new queries' offset members.  Returns (O [L, B, H, D], LSE [L, B, H]
    or None)."""
    shape = tuple(k_cache.shape)
    dtype, dev = k_cache.dtype, k_cache.device
    if tuple(q.shape) != shape[:3] + shape[4:]:
        raise ValueError("q must be [L, B, H, D] matching the caches")
    _check_tensors(shape, dtype, dev, k=k_cache, v=v_cache, alpha=alpha)
    if q.dtype != dtype or not q.is_contiguous() or q.device != dev:
        raise ValueError("q must be a contiguous tensor of the caches' dtype and device")
    out = torch.empty_like(q) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty(shape[:3], dtype=torch.float32, device=dev)
    p = make_params(shape, dtype, window=window, offsets=offsets, sinks=sinks,
                    rope_base=rope_base, scale=scale)
    if beta is not None and (beta.device != dev or not beta.is_contiguous()
                             or beta.dtype != torch.float32 or tuple(beta.shape) != shape[:3]):
        raise ValueError(f"beta must be a contiguous CUDA fp32 tensor of shape {shape[:3]}")
    st = lib().sparse_attn_decode_prior(ctypes.byref(p), int(pos), _ptr(q), _ptr(k_cache),
                                        _ptr(v_cache), _ptr(alpha), _ptr(beta), _ptr(out),
                                        _ptr(lse), _stream_handle(stream))
    _check("sparse_attn_decode_prior", st)
    return out, lse


def fwd_noalloc(q, k, v, alpha, *, window, offsets=FIB15, sinks=0, rope_base=10000.0,
                scale=0.0, out=None, lse=None, want_lse=True, stream=None):
    """Forward through sparse_attn_fwd_noalloc: the library allocates nothing.

    For callers that cannot let a library allocate device memory (a pooling
    allocator that must see every byte, or no allocation after start-up).  The
    RoPE table lives in a fixed 8 MiB device array (T * D/2 * 8 bytes must fit);
    calls that overlap on the GPU share that array and must be serialised.
    Output buffers may be passed in; otherwise they are allocated here by torch,
    on the caller's side of the boundary.
    """
    shape, dtype, dev = tuple(q.shape), q.dtype, q.device
    if lse is None and want_lse:
        lse = torch.empty(shape[:4], dtype=torch.float32, device=dev)
    out = torch.empty_like(q) if out is None else out
    _check_tensors(shape, dtype, dev, q=q, k=k, v=v, o=out, alpha=alpha, lse=lse)
    p = make_params(shape, dtype, window=window, offsets=offsets, sinks=sinks,
                    rope_base=rope_base, scale=scale)
    st = lib().sparse_attn_fwd_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                       _ptr(out), _ptr(lse), _stream_handle(stream))
    _check("sparse_attn_fwd_noalloc", st)
    return out, lse


def bwd(q, k, v, o, lse, dout, alpha, *, window, offsets=FIB15, sinks=0, rope_base=10000.0,
        scale=0.0, dq=None, dk=None, dv=None, dalpha=None, workspace=None, stream=None,
        context=None, beta=None, dbeta=None):
    """Sparse attention backward: returns (dQ, dK, dV, dalpha[L]).

    context: the buffer a fwd(..., context=) call filled for the same inputs;
    the backward then runs as sparse_attn_bwd_ctx (no score pass).
    beta: the forward's log-prior [L, B, H, T]; the call then runs as
    sparse_attn_bwd_prior and returns (dQ, dK, dV, dalpha, dbeta)."""
    shape, dtype, dev = tuple(q.shape), q.dtype, q.device
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    dalpha = torch.empty(shape[0], dtype=torch.float32, device=dev) if dalpha is None else dalpha
    _check_tensors(shape, dtype, dev, q=q, k=k, v=v, o=o, dout=dout, dq=dq, dk=dk, dv=dv,
                   alpha=alpha, dalpha=dalpha, lse=lse)
    p = make_params(shape, dtype, window=window, offsets=offsets, sinks=sinks,
                    rope_base=rope_base, scale=scale)
    L = lib()
    ws_n = int(L.sparse_attn_workspace_size(ctypes.byref(p), 1))
    if workspace is None or workspace.numel() < ws_n:
        workspace = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev)
    if beta is not None:
        dbeta = torch.empty(shape[:4], dtype=torch.float32, device=dev) if dbeta is None else dbeta
        _check_prior(shape, dev, beta=beta, dbeta=dbeta)
        st = L.sparse_attn_bwd_prior(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                     _ptr(lse), _ptr(dout), _ptr(alpha), _ptr(beta),
                                     _ptr(context), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dalpha),
                                     _ptr(dbeta), _ptr(workspace), workspace.numel(),
                                     _stream_handle(stream))
        _check("sparse_attn_bwd_prior", st)
        return dq, dk, dv, dalpha, dbeta
    if context is not None:
        st = L.sparse_attn_bwd_ctx(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                   _ptr(dout), _ptr(alpha), _ptr(context), _ptr(dq), _ptr(dk),
                                   _ptr(dv), _ptr(dalpha), _ptr(workspace), workspace.numel(),
                                   _stream_handle(stream))
        _check("sparse_attn_bwd_ctx", st)
        return dq, dk, dv, dalpha
    st = L.sparse_attn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                           _ptr(dout), _ptr(alpha), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dalpha),
                           _ptr(workspace), workspace.numel(), _stream_handle(stream))
    _check("sparse_attn_bwd", st)
    return dq, dk, dv, dalpha
