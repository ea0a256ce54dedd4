"""Seeded synthetic workloads for the sparse-attention path.

This module holds workload definitions and random-number generation only: no
step of the attention itself.  The CUDA path and the CPU oracle both consume
the tensors it returns, so they see identical inputs.

Workload shapes follow "Depth-Staggered Fibonacci Spacing for Sparse
Attention" (technical summary): 16 layers, hidden 512 (8 heads of 64), trained
at length 1024 and evaluated at 4096 ("Length extrapolation"), windows
W in {6, 8, 10, 12}, the four per-layer alpha schedules of "Experimental
variables" (fixed alpha = 1; learned, initialised at 1; linear stagger 0.5 -> 1.5
over layers 0..15; the same multiset reassigned by l -> 7l mod 16).  The long
window-plus-sinks case adds four always-attended sink keys at positions 0..3.
No dataset is involved: all values are N(0, 1) draws from seeded generators.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple

import torch

FIB15 = (1, 2, 3, 5, 8, 13, 21, 34, 55, 89, 144, 233, 377, 610, 987)
# The power-of-2 base at the 4x evaluation length: every power of two below
# 4096 (the control ladder, which reaches 1024 and 2048 there).
POW2_4096 = tuple(1 << k for k in range(12))


def alpha_linear_stagger(L: int = 16):
    """alpha_l = 0.5 + l/(L-1), l = 0..L-1, as fp32 values."""
    return torch.tensor([0.5 + l / (L - 1) for l in range(L)], dtype=torch.float32)


def alpha_coprime_stagger(L: int = 16, step: int = 7):
    """The linear-stagger multiset reassigned across layers by l -> step*l mod L."""
    lin = alpha_linear_stagger(L)
    return torch.stack([lin[(step * l) % L] for l in range(L)])


def alpha_learned_init(L: int = 16, seed: int = 4000, std: float = 0.05):
    """A learned-alpha state near its initialisation: clamp(1 + N(0, std), 0.5, 1.5)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.clamp(1.0 + std * torch.randn(L, generator=g, dtype=torch.float32), 0.5, 1.5)


@dataclass(frozen=True)
class Workload:
    name: str
    L: int
    B: int
    H: int
    T: int
    D: int
    window: int
    sinks: int
    dtype: torch.dtype
    alpha_kind: str            # "fixed", "linear", "coprime", "learned"
    seed: int                  # layer l uses seed + l (the tiny case: seed 0 for all)
    backward: bool = False
    decode: bool = False       # one new token at position T - 1 against a T-row KV cache
    prior: bool = False        # a per-query log-prior beta on the offset members
    offsets: Tuple[int, ...] = FIB15
    rope_base: float = 10000.0
    note: str = ""

    @property
    def token_heads(self) -> int:
        return self.L * self.B * self.H * self.T

    def alpha(self) -> torch.Tensor:
        if self.alpha_kind == "fixed":
            return torch.ones(self.L, dtype=torch.float32)
        if self.alpha_kind == "linear":
            return alpha_linear_stagger(self.L)
        if self.alpha_kind == "coprime":
            return alpha_coprime_stagger(self.L)
        if self.alpha_kind == "learned":
            return alpha_learned_init(self.L)
        raise ValueError(self.alpha_kind)

    def shrink(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 1, 2, 64, 16, 6, 0, torch.float32, "fixed", 0,
                          note="B=1 H=2 T=64 d=16 fp32, W=6, 15 Fibonacci offsets, alpha=1"),
    "paper_fwd": Workload("paper_fwd", 16, 8, 8, 1024, 64, 12, 0, torch.bfloat16, "linear", 2000,
                          note="16 layers B=8 H=8 T=1024 d=64 bf16, W=12, linear stagger"),
    "extrap_4x": Workload("extrap_4x", 16, 2, 8, 4096, 64, 12, 0, torch.bfloat16, "coprime", 3000,
                          note="16 layers B=2 H=8 T=4096 d=64 bf16, W=12, coprime stagger"),
    "learned_train": Workload("learned_train", 16, 8, 8, 1024, 64, 12, 0, torch.bfloat16,
                              "learned", 4100, backward=True,
                              note="16 layers B=8 H=8 T=1024 d=64 bf16, W=12, learned alpha, fwd+bwd"),
    "pow2_extrap": Workload("pow2_extrap", 16, 2, 8, 4096, 64, 12, 0, torch.bfloat16, "linear",
                            9000, offsets=POW2_4096,
                            note="the power-of-2 control base at the 4x evaluation length: "
                                 "offsets 1, 2, 4, ..., 2048 with the linear stagger (reach "
                                 "1.5 x 2048 = 3072 rows), 16 layers B=2 H=8 T=4096 d=64 bf16, "
                                 "W=12"),
    "long_sinks": Workload("long_sinks", 1, 1, 16, 32768, 64, 64, 4, torch.bfloat16, "fixed", 5000,
                           note="B=1 H=16 T=32768 d=64 bf16, W=64, 4 sinks, alpha=1"),
    # forward-kernel comparisons across window lengths (the CUDA-core, mma.sync
    # and tcgen05 forwards); not among the five benchmark configurations
    "window_32": Workload("window_32", 1, 1, 16, 32768, 64, 32, 4, torch.bfloat16, "fixed", 5100,
                          note="B=1 H=16 T=32768 d=64 bf16, W=32, 4 sinks, alpha=1"),
    "window_64_stagger": Workload("window_64_stagger", 4, 1, 4, 32768, 64, 64, 4, torch.bfloat16,
                                  "linear", 5200,
                                  note="4 layers B=1 H=4 T=32768 d=64 bf16, W=64, 4 sinks, "
                                       "linear stagger (interpolated offsets)"),
    "pi_skip": Workload("pi_skip", 16, 8, 8, 1024, 64, 5, 0, torch.bfloat16, "fixed", 7000,
                        offsets=(16,),
                        note="periodic skip in autoregressive form: local window of the "
                             "current and 4 previous keys plus one skip to i - 16 (k = 4, "
                             "pi = 16, the best setting of the pi-Attention page), 16 layers "
                             "B=8 H=8 T=1024 d=64 bf16"),
    "pi_gate_train": Workload("pi_gate_train", 16, 8, 8, 1024, 64, 5, 0, torch.bfloat16, "fixed",
                              8000, backward=True, prior=True, offsets=(16,),
                              note="the periodic-skip pattern with pi-Attention's fusion of "
                                   "local and skip logits in one softmax: a per-query "
                                   "log-prior beta ~ N(0, 1) on the skip member, forward and "
                                   "backward (dQ, dK, dV, dbeta), 16 layers B=8 H=8 T=1024 "
                                   "d=64 bf16, W=5, offset 16"),
    "decode_4k": Workload("decode_4k", 16, 8, 8, 4096, 64, 12, 0, torch.bfloat16, "linear", 6000,
                          decode=True,
                          note="single-token decode: 16 layers B=8 H=8 d=64 bf16, one new query "
                               "at position 4095 against a 4096-row KV cache, W=12, linear "
                               "stagger (the page measures inference latency of this gather)"),
}


def make_inputs(wl: Workload, device: Optional[str] = None, layers: Optional[range] = None,
                pin: bool = False):
    """Q, K, V (and dO when the workload has a backward) as [L, B, H, T, D].

    Layer l draws Q, K, V (then dO) in that order, each N(0, 1) in fp32 from a
    CPU generator seeded with ``seed + l`` (every layer of the tiny case uses
    seed 0), then casts to the workload dtype.  ``layers`` restricts the
    draw to a subset of layers (same values as in the full draw).
    """
    layers = range(wl.L) if layers is None else layers
    shape = (wl.B, wl.H, wl.T, wl.D)
    n_t = 4 if wl.backward else 3
    outs = [torch.empty((len(layers),) + shape, dtype=wl.dtype, pin_memory=pin)
            for _ in range(n_t)]
    for li, l in enumerate(layers):
        g = torch.Generator(device="cpu").manual_seed(wl.seed + (l if wl.seed else 0))
        for t in range(n_t):
            outs[t][li].copy_(torch.randn(shape, generator=g, dtype=torch.float32))
    if device is not None:
        outs = [o.to(device) for o in outs]
    return tuple(outs)


def make_dout(wl: Workload, seed: int = 77, device: Optional[str] = None):
    """An upstream gradient dO ~ N(0, 1) for workloads drawn without one."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn((wl.L, wl.B, wl.H, wl.T, wl.D), generator=g, dtype=torch.float32)
    x = x.to(wl.dtype)
    return x if device is None else x.to(device)


def make_decode_inputs(wl: Workload, device: Optional[str] = None, pin: bool = False):
    """q [L, B, H, D] (the new token's queries) and the K, V caches
    [L, B, H, T, D] of a decode workload.  Layer l draws q, then K, then V,
    each N(0, 1) in fp32 from a CPU generator seeded with ``seed + l``, then
    casts to the workload dtype."""
    L, B, H, T, D = wl.L, wl.B, wl.H, wl.T, wl.D
    q = torch.empty((L, B, H, D), dtype=wl.dtype, pin_memory=pin)
    k = torch.empty((L, B, H, T, D), dtype=wl.dtype, pin_memory=pin)
    v = torch.empty((L, B, H, T, D), dtype=wl.dtype, pin_memory=pin)
    for l in range(L):
        g = torch.Generator(device="cpu").manual_seed(wl.seed + l)
        q[l].copy_(torch.randn((B, H, D), generator=g, dtype=torch.float32))
        k[l].copy_(torch.randn((B, H, T, D), generator=g, dtype=torch.float32))
        v[l].copy_(torch.randn((B, H, T, D), generator=g, dtype=torch.float32))
    if device is not None:
        q, k, v = q.to(device), k.to(device), v.to(device)
    return q, k, v


def make_prior(wl: Workload, device: Optional[str] = None, layers: Optional[range] = None,
               pin: bool = False):
    """The log-prior beta [L, B, H, T] of a workload with ``prior``: layer l
    draws N(0, 1) values in fp32 from a CPU generator seeded with
    ``seed + 500000 + l`` (the gate logits a fusion network would produce,
    here synthetic)."""
    layers = range(wl.L) if layers is None else layers
    out = torch.empty((len(layers), wl.B, wl.H, wl.T), dtype=torch.float32, pin_memory=pin)
    for li, l in enumerate(layers):
        g = torch.Generator(device="cpu").manual_seed(wl.seed + 500000 + l)
        out[li].copy_(torch.randn((wl.B, wl.H, wl.T), generator=g, dtype=torch.float32))
    return out if device is None else out.to(device)
