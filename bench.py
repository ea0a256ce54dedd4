"""Benchmark of the structured sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...        # the CPU oracle as the reference arm

One step is one pass of the whole path -- forward (offset geometry, RoPE,
gather with interpolation, softmax, PV) and, for a training workload, the
backward (dQ, dK, dV and the per-layer d-alpha) -- over one synthetic batch.
The default workload is the learned-alpha training step: 16 layers, B=8, H=8,
T=1024, d=64, W=12, bf16, forward plus backward.  With N GPUs every rank runs
its own batch (independent (layer, batch, head) units: weak scaling, no
collective on the data path); the step time is the max over ranks.

Prints one JSON line (rank 0): the headline workload's throughput, its
rooflines (HBM bytes and fp32 FMA work, by kernel and by phase), the end-to-end
figure through host buffers, the CPU oracle baseline, and a "workloads" record
timing the other benchmark configurations (forward only) the same way.

Roofline bytes (per token-head, d = 64, bf16; the unique bytes the path must
move, the definition the problem statement gives for the forward):
  forward  : read Q, K, V, write O                       = 4 * 128       = 512 B
  backward : read Q, K, V, O, dO and LSE, write dQ, dK, dV = 8 * 128 + 4  = 1028 B
Per kernel, the backward's bytes are split as the kernels touch the tensors:
the query side reads Q, K, V, dO, LSE and writes dQ (644 B); the key side
writes dK and dV and carries O's read (384 B).  The RoPE pre-passes, the
training context and the key-indexed weight blocks are intermediates the
implementation chose, so they count 0.  The fp32 tiny case uses 4-byte
elements.
ALU work (per token-head): every distinct K/V row a query's members touch
(window, sinks, both rows of each interpolated offset; rows shared by the
window and an offset counted once) costs one D-long dot product and one
D-long axpy in the forward (4 D FLOPs per row), and four in the backward
with a saved context (dO.V, dq += g K, dK += g q, dV += p dO: 8 D FLOPs per
row; a backward without context also recomputes the dot products, 10 D).
The ALU peak is the fp32 FMA throughput measured in the same run by the
library's probe (packed fp32x2 FMAs, register-only); the nominal figure is
148 SMs x 128 lanes x 2 FLOPs per clock at the sampled SM clock.
"""
import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

METRIC = "sparse-attn fwd/bwd tokens·heads/s at T=1024/4096; HBM GB/s vs B200 peak"
UNIT = "tokens·heads/s"
FALLBACK_HBM_GBS = 6650.0
B200_SMS, FP32_LANES_PER_SM = 148, 128
# Configurations timed beside the headline in the "workloads" record: the
# other four problem-statement configurations and the power-of-2 control.
# --forward: which bf16 / head-dim-64 forward kernel the plain forwards run
# (sparse_attn_select_forward; the training forward is always the CUDA-core one)
FORWARD_KERNELS = {"auto": 0, "cuda_core": 1, "mma_sync": 2, "tcgen05": 3}
OTHER_WORKLOADS = ("tiny_fp32", "paper_fwd", "extrap_4x", "long_sinks", "pow2_extrap")


def alg_bytes_per_token_head(kernel, D, elt, prior=False):
    """The roofline bytes a kernel is credited with per token-head (see the
    module docstring): the forward kernels Q, K, V and O; the backward query
    side Q, K, V, dO, LSE and dQ; the key side dK, dV and O; pre-passes 0.
    With a log-prior the forward also reads beta and the query side reads
    beta and writes dbeta (4 B each)."""
    row = D * elt
    if kernel.startswith("fwd"):
        return 4 * row + (4 if prior else 0)
    if kernel.startswith("bwd_q"):
        return 5 * row + 4 + (8 if prior else 0)
    if kernel.startswith("bwd_kv"):
        return 3 * row
    return 0


def phase_bytes_per_token_head(phase, D, elt, prior=False):
    """forward: Q, K, V, O; backward: Q, K, V, O, dO, dQ, dK, dV and LSE
    (plus beta, and dbeta in the backward, with a log-prior)."""
    row = D * elt
    if phase == "forward":
        return 4 * row + (4 if prior else 0)
    return 8 * row + 4 + (8 if prior else 0)


def distinct_rows(alpha, offsets, window, sinks):
    """Distinct K/V rows a query far from the sequence start touches at this
    alpha: window lags 0..W-1, each offset's lags lo and (when w != 0) lo + 1,
    the sinks.  d = fp32 product alpha * f, lo = floor(d)."""
    import numpy as np
    lags = set(range(window))
    a32 = np.float32(alpha)
    for f in offsets:
        d = float(a32 * np.float32(f))
        lo = int(np.floor(d))
        lags.add(lo)
        if d != lo:
            lags.add(lo + 1)
    return len(lags) + sinks


def alg_flops(wl, phase, context=True):
    """fp32 FLOPs of one pass over the workload (see the module docstring)."""
    per_row = {"forward": 4, "backward": 8 if context else 10}[phase] * wl.D
    rows = sum(distinct_rows(a, wl.offsets, wl.window, wl.sinks) for a in wl.alpha().tolist())
    return per_row * rows * (wl.B * wl.H * wl.T)


def kernel_flops(wl, kernel, context=True):
    """fp32 FLOPs one launch of a kernel is credited with: the forward 4 D per
    distinct row, the query side 4 D (6 D when it recomputes the dot products
    without a context), the key side 4 D; pre-passes and reductions 0."""
    if kernel.startswith("fwd"):
        per = 4
    elif kernel.startswith("bwd_q"):
        per = 4 if context else 6
    elif kernel.startswith("bwd_kv"):
        per = 4
    else:
        return 0
    rows = sum(distinct_rows(a, wl.offsets, wl.window, wl.sinks) for a in wl.alpha().tolist())
    return per * wl.D * rows * (wl.B * wl.H * wl.T)


def fma_peak(sa, torch, dev, reps=5):
    """The ALU roofline's peak, measured now: the library's register-only fp32
    FMA probe (scalar and packed), 8 CTAs of 256 threads per SM, best of
    `reps` launches of each, timed with CUDA events on the current stream.
    The nominal figure is 148 SMs x 128 lanes x 2 FLOPs at the GPU's maximum
    SM clock."""
    blocks, threads, iters = B200_SMS * 8, 256, 4096
    out = torch.empty(blocks * threads, dtype=torch.float32, device=dev)
    best = {}
    for packed in (0, 1):
        for _ in range(2):
            sa.fma_probe(out, blocks, threads, iters, packed)
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            flops = sa.fma_probe(out, blocks, threads, iters, packed)
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        best["packed" if packed else "scalar"] = flops / (min(ts) / 1e3) / 1e12
    try:
        mhz = float(torch.cuda.get_device_properties(dev).clock_rate) / 1e3
    except Exception:
        mhz = None
    if not mhz:
        mhz = 1965.0
    nominal = B200_SMS * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12
    kind = max(best, key=best.get)
    return {"peak": best[kind], "source": f"measured in-run: fp32 FMA probe ({kind}), "
                                          f"{blocks} CTAs x {threads} threads",
            "probe_TFLOPs": best, "nominal": nominal, "nominal_clock_mhz": mhz}


def time_forward_workload(sa, torch, dev, name, steps, warmup, peak, alu_peak):
    """Device time of `steps` forward passes of a benchmark workload (its
    inputs resident in HBM), with its rooflines; inputs smaller than L2 are
    timed step by step with an L2 flush (a 256 MiB write) between steps."""
    from structured_sparse_attention_fibonacci_b200.inputs import WORKLOADS, make_inputs
    wl = WORKLOADS[name]
    q, k, v = make_inputs(wl, device=str(dev))[:3]
    alpha = wl.alpha().to(dev)
    kw = dict(window=wl.window, sinks=wl.sinks, offsets=wl.offsets, rope_base=wl.rope_base)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:4], dtype=torch.float32, device=dev)
    ws_n = sa.workspace_size(tuple(q.shape), q.dtype, backward=False, **kw)
    ws = torch.empty(max(1, ws_n), dtype=torch.uint8, device=dev)
    elt = q.element_size()
    in_bytes = 3 * q.numel() * elt
    small = in_bytes < 126 * 2 ** 20
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev) if small else None

    def step():
        sa.fwd(q, k, v, alpha, out=o, lse=lse, workspace=ws, **kw)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    launches = 0
    if small:
        total = 0.0
        for _ in range(steps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            step()
            b.record()
            torch.cuda.synchronize()
            launches += sa.last_launch_count()
            total += a.elapsed_time(b)
        ms = total / steps
    else:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            step()
            launches += sa.last_launch_count()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / steps
    sa.trace_enable(True)
    for _ in range(steps):
        step()
    tr = sa.trace_read()
    sa.trace_enable(False)
    kern = {n: t / c for n, (t, c) in tr.items()}
    bpt = phase_bytes_per_token_head("forward", wl.D, elt, wl.prior)
    fl = alg_flops(wl, "forward")
    fwd_k = max(kern, key=kern.get)
    gbs = bpt * wl.token_heads / (ms / 1e3) / 1e9
    k_gbs = bpt * wl.token_heads / (kern[fwd_k] / 1e3) / 1e9
    rec = {"config": wl.note, "ms_per_step": ms, "value": wl.token_heads / (ms / 1e3),
           "unit": UNIT, "gpu_launches": launches, "l2": "flushed between steps (256 MiB write)"
           if small else "inputs larger than L2",
           "kernels_ms": kern, "alg_bytes_per_token_head": bpt,
           "hbm": {"achieved_GBps": gbs, "frac": gbs / peak, "kernel": fwd_k,
                   "kernel_frac": k_gbs / peak, **workload_traffic(wl.name, fwd_k)},
           "alu": {"alg_flops": fl, "achieved_TFLOPs": fl / (ms / 1e3) / 1e12,
                   "frac": fl / (ms / 1e3) / 1e12 / alu_peak if alu_peak else None}}
    del q, k, v, o, lse, ws, flush
    torch.cuda.empty_cache()
    return rec


def decode_bytes_per_token_head(wl, elt):
    """Decode: read the query and every K and V row of its attended set (W
    window rows, the sinks, two rows per offset); write O and LSE."""
    row = wl.D * elt
    rows = wl.window + wl.sinks + 2 * len(wl.offsets)
    return 2 * row + 4 + 2 * rows * row


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per token-head
# (per (layer, batch, head) for decode) of the dominant kernel, from one ncu
# capture per entry; keyed by workload, kernel and the hash of the kernel
# sources the capture ran (kernel_source_hash): a changed source reports null.
MEASURED_TRAFFIC = {
    "learned_train/bwd_q_fast@a3631b8328cf": 780.3,
    "pi_gate_train/bwd_q_fast@a3631b8328cf": 545.8,
    "paper_fwd/fwd_fast@a3631b8328cf": 494.4,
    "extrap_4x/fwd_fast@a3631b8328cf": 496.1,
    "pow2_extrap/fwd_fast@a3631b8328cf": 496.3,
    "pi_skip/fwd_fast@a3631b8328cf": 492.1,
    "long_sinks/fwd_tc@a3631b8328cf": 505.3,
    "decode_4k/decode@a3631b8328cf": 8121.5,
}


def workload_traffic(workload, kernel):
    """The kernel's DRAM bytes per token-head from MEASURED_TRAFFIC at the
    current kernel sources, with where the figure comes from."""
    h = kernel_source_hash()
    t = MEASURED_TRAFFIC.get(f"{workload}/{kernel}@{h}")
    return {"traffic_B_per_token_head": t,
            "traffic_source": f"ncu@{h}" if t is not None else f"none: no ncu capture of sources {h}"}


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(HERE, "structured_sparse_attention_fibonacci_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:12]


def measured_peaks():
    path = os.path.join(HERE, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---- clocks during the timed region -----------------------------------------
class ClockSampler:
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None):
        self.uuid = uuid
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            if self.uuid and parts[1] != self.uuid:
                continue
            try:
                sm.append(float(parts[2]))
                mx.append(float(parts[3]))
                power.append(float(parts[4]))
            except ValueError:
                continue
            for n, v in zip(names, parts[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "power_w_max": max(power) if power else None,
                "reasons": sorted(reasons)}


# ---- multi-rank helpers (host logic; tested with gloo on CPU) --------------
def max_over_ranks(value, device=None):
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank, world, steps, ms_max):
    """Whole-job units per second: all ranks' units over the slowest rank's time."""
    return units_per_rank * world * steps / (ms_max / 1e3)


# ---- CPU baseline: the oracle as it stands, on a bounded sample -------------
def cpu_model():
    """The host CPU's model name (Linux), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def on_one_thread(fn):
    """fn()'s result with the oracle's OpenMP limited to one thread (None if
    the OpenMP runtime cannot be reached)."""
    import ctypes
    try:
        gomp = ctypes.CDLL("libgomp.so.1")
    except OSError:
        return None
    before = gomp.omp_get_max_threads()
    gomp.omp_set_num_threads(1)
    try:
        return fn()
    finally:
        gomp.omp_set_num_threads(before)


def oracle_sample(wl, budget_s, single_thread=False):
    """Time the fp32 oracle (forward, plus backward for training workloads) on
    as many whole layers (all their (batch, head) units, OpenMP-parallel) as
    fit the time budget; at least one layer."""
    import oracle
    from structured_sparse_attention_fibonacci_b200.inputs import make_inputs
    kw = dict(window=wl.window, sinks=wl.sinks, offsets=wl.offsets, rope_base=wl.rope_base,
              precision="f32")
    alpha = wl.alpha().numpy()

    if wl.decode:
        from structured_sparse_attention_fibonacci_b200.inputs import make_decode_inputs
        q1, kc, vc = (t.float().numpy() for t in make_decode_inputs(wl))
        reps, t = 0, 0.0
        while reps == 0 or (t < budget_s and reps < 1000):
            t0 = time.perf_counter()
            oracle.decode(q1, kc, vc, alpha, wl.T - 1, **kw)
            t += time.perf_counter() - t0
            reps += 1
        cores = int(os.environ.get("OMP_NUM_THREADS", len(os.sched_getaffinity(0))))
        units = wl.L * wl.B * wl.H
        return {"value": reps * units / t, "unit": UNIT, "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
                "sample": f"{reps} decode steps of {units} (layer, batch, head) units at "
                          f"position {wl.T - 1}, fp32 oracle", "seconds": t}

    def one_layer(l):
        ts = make_inputs(wl, layers=range(l, l + 1))
        arr = [t.float().numpy() for t in ts]
        pkw = dict(kw)
        if wl.prior:
            from structured_sparse_attention_fibonacci_b200.inputs import make_prior
            pkw["beta"] = make_prior(wl, layers=range(l, l + 1)).numpy()
        t0 = time.perf_counter()
        oracle.fwd(arr[0], arr[1], arr[2], alpha[l:l + 1], **pkw)
        if wl.backward:
            oracle.bwd(arr[0], arr[1], arr[2], arr[3], alpha[l:l + 1], **pkw)
        return time.perf_counter() - t0

    t = one_layer(0)
    n = 1
    while n < wl.L and t * (n + 1) / n <= budget_s:
        t += one_layer(n)
        n += 1
    cores = int(os.environ.get("OMP_NUM_THREADS", len(os.sched_getaffinity(0))))
    extra = {}
    if single_thread:
        # the same oracle on one thread, layer 0 only
        extra["single_thread_layer0_s"] = on_one_thread(lambda: one_layer(0))
    units = n * wl.B * wl.H
    sample = (f"{n} of {wl.L} layers = {units} (layer, batch, head) units "
              f"({units * wl.T} token-heads), fp32 oracle "
              f"{'forward+backward' if wl.backward else 'forward'}")
    return {"value": units * wl.T / t, "unit": UNIT, "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
            "sample": sample, "seconds": t, **extra}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle, timed on the host cores."""
    from structured_sparse_attention_fibonacci_b200.inputs import WORKLOADS
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    per_step_budget = max(1.0, args.reference_budget_s / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(wl, per_step_budget)
    vals = [oracle_sample(wl, per_step_budget) for _ in range(args.steps)]
    secs = sum(v["seconds"] for v in vals)
    # time-weighted mean of the steps' rates (all units over all seconds)
    value = sum(v["value"] * v["seconds"] for v in vals) / max(secs, 1e-12)
    cb = dict(vals[-1])
    cb["value"] = value
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / len(vals), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(wl, world), "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl, world):
    if wl.decode:
        pass_ = f"decode (one token at position {wl.T - 1}, KV cache of {wl.T} rows)"
    else:
        pass_ = "forward+backward" if wl.backward else "forward"
    return {"workload": wl.name, "L": wl.L, "B": wl.B, "H": wl.H, "T": wl.T, "D": wl.D,
            "window": wl.window, "sinks": wl.sinks,
            "offsets": ("fib15 (1..987)" if tuple(wl.offsets) == (1, 2, 3, 5, 8, 13, 21, 34, 55, 89,
                                                                  144, 233, 377, 610, 987)
                        else list(wl.offsets)),
            "alpha": wl.alpha_kind, "pass": pass_,
            **({"prior": "log-prior beta ~ N(0, 1) per query on the offset members"}
               if wl.prior else {}),
            "global_batch": wl.B * world, "seq_len": wl.T, "parallelism": f"replicas{world}",
            "l2": ("inputs larger than L2 (no flush needed)" if not wl.decode else
                   "KV caches (1 GiB) larger than L2; each step gathers 42 rows per unit"),
            **({"launch": "the timed steps replay one CUDA graph of K decode calls"}
               if wl.decode else {})}


# ---- our arm -------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import torch
    import structured_sparse_attention_fibonacci_b200 as sa
    from structured_sparse_attention_fibonacci_b200.inputs import WORKLOADS, make_inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    sa.select_forward(FORWARD_KERNELS[args.forward])
    wl = WORKLOADS[args.workload]
    wl_rank = wl.shrink(seed=wl.seed + 100000 * rank) if world > 1 else wl
    host = make_inputs(wl_rank, pin=True)
    if wl.prior:
        from structured_sparse_attention_fibonacci_b200.inputs import make_prior
        host = host + (make_prior(wl_rank, pin=True),)
    q, k, v = (t.to(dev) for t in host[:3])
    do = host[3].to(dev) if wl.backward else None
    beta = host[-1].to(dev) if wl.prior else None
    dbeta = torch.empty_like(beta) if wl.prior and wl.backward else None
    alpha_h = wl.alpha().pin_memory()
    alpha = alpha_h.to(dev)
    kw = dict(window=wl.window, sinks=wl.sinks, offsets=wl.offsets, rope_base=wl.rope_base)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:4], dtype=torch.float32, device=dev)
    if wl.backward:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        dal = torch.empty(wl.L, dtype=torch.float32, device=dev)
        ws = torch.empty(max(1, sa.workspace_size(tuple(q.shape), q.dtype, backward=True, **kw)),
                         dtype=torch.uint8, device=dev)
        # training step: the forward saves what the backward reuses (rotated
        # keys, probabilities, row-score differences) in a context buffer
        n_ctx = sa.context_size(tuple(q.shape), q.dtype, **kw)
        ctx = torch.empty(n_ctx, dtype=torch.uint8, device=dev) if n_ctx else None
    launches = [0]

    def fwd_call():
        sa.fwd(q, k, v, alpha, out=o, lse=lse, context=ctx if wl.backward else None, beta=beta,
               **kw)
        launches[0] += sa.last_launch_count()

    def bwd_call():
        sa.bwd(q, k, v, o, lse, do, alpha, dq=dq, dk=dk, dv=dv, dalpha=dal, workspace=ws,
               context=ctx, beta=beta, dbeta=dbeta, **kw)
        launches[0] += sa.last_launch_count()

    def step():
        fwd_call()
        if wl.backward:
            bwd_call()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.4)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches[0] = 0
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    gpu_launches = launches[0]
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, dev)
    value = aggregate_throughput(wl.token_heads, world, args.steps, ms_max)

    # per-kernel times of the same steps, forward and backward traced apart
    # (library trace: CUDA events around each launch, on its stream)
    phases = [("forward", fwd_call)] + ([("backward", bwd_call)] if wl.backward else [])
    traced = {ph: {} for ph, _ in phases}
    sa.trace_enable(True)
    for _ in range(args.steps):
        for ph, call in phases:
            call()
            for n, (t, c) in sa.trace_read().items():
                tt, cc = traced[ph].get(n, (0.0, 0))
                traced[ph][n] = (tt + t, cc + c)
    sa.trace_enable(False)
    elt = 2 if wl.dtype == torch.bfloat16 else 4
    peak, peak_kind = measured_peaks()
    alu = fma_peak(sa, torch, dev)
    context = bool(wl.backward and ctx is not None)
    kernels = {}
    for ph, _ in phases:
        for n, (t, c) in traced[ph].items():
            key = n if n not in kernels else f"{n} ({ph})"
            ms_l = t / c
            b = alg_bytes_per_token_head(n, wl.D, elt, wl.prior) * wl.token_heads
            fl = kernel_flops(wl, n, context)
            kernels[key] = {"phase": ph, "ms_per_launch": ms_l, "launches": c,
                            "alg_GBps": b / (ms_l / 1e3) / 1e9 if b else None,
                            "alg_TFLOPs": fl / (ms_l / 1e3) / 1e12 if fl else None}
    dominant = max(kernels, key=lambda n: kernels[n]["ms_per_launch"] * kernels[n]["launches"])
    dom = kernels[dominant]
    bytes_launch = alg_bytes_per_token_head(dominant, wl.D, elt, wl.prior) * wl.token_heads
    achieved = bytes_launch / (dom["ms_per_launch"] / 1e3) / 1e9
    src_hash = kernel_source_hash()
    traffic = MEASURED_TRAFFIC.get(f"{wl.name}/{dominant}@{src_hash}")
    phase_ms = {ph: sum(kk["ms_per_launch"] * kk["launches"] for kk in kernels.values()
                        if kk["phase"] == ph) / args.steps for ph, _ in phases}
    phase_ms["step"] = sum(phase_ms.values())
    ph_rec = {}
    for ph, msp in phase_ms.items():
        if ph == "step":
            bpt = sum(phase_bytes_per_token_head(p, wl.D, elt, wl.prior) for p, _ in phases)
            fl = sum(alg_flops(wl, p, context) for p, _ in phases)
        else:
            bpt = phase_bytes_per_token_head(ph, wl.D, elt, wl.prior)
            fl = alg_flops(wl, ph, context)
        gbs = bpt * wl.token_heads / (msp / 1e3) / 1e9
        tfs = fl / (msp / 1e3) / 1e12
        ph_rec[ph] = {"ms": msp, "alg_bytes_per_token_head": bpt, "achieved_GBps": gbs,
                      "frac": gbs / peak, "alg_flops": fl, "achieved_TFLOPs": tfs,
                      "alu_frac": tfs / alu["peak"] if alu["peak"] else None}
    roofline = {"bound": "hbm", "kernel": dominant, "achieved": achieved, "peak": peak,
                "peak_source": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                "alg_bytes_per_launch": bytes_launch,
                "traffic": traffic * wl.token_heads if traffic is not None else None,
                "traffic_source": (f"ncu@{src_hash}" if traffic is not None else
                                   f"none: no ncu capture of sources {src_hash}"),
                "phases": {ph: {k_: r[k_] for k_ in ("ms", "alg_bytes_per_token_head",
                                                     "achieved_GBps", "frac")}
                           for ph, r in ph_rec.items()}}
    dom_fl = kernel_flops(wl, dominant, context)
    dom_tf = dom_fl / (dom["ms_per_launch"] / 1e3) / 1e12
    roofline_alu = {"bound": "alu", "kernel": dominant, "achieved": dom_tf, "peak": alu["peak"],
                    "peak_source": alu["source"], "peak_nominal": alu["nominal"],
                    "unit": "TFLOP/s", "frac": dom_tf / alu["peak"] if alu["peak"] else None,
                    "alg_flops_per_launch": dom_fl,
                    "phases": {ph: {"ms": r["ms"], "alg_flops": r["alg_flops"],
                                    "achieved_TFLOPs": r["achieved_TFLOPs"],
                                    "frac": r["alu_frac"]} for ph, r in ph_rec.items()}}

    # End to end through the public API: every step copies its inputs in from
    # pinned host memory and its results back out.  Two device buffer sets
    # and three streams (copy in, compute, copy out) let step n's results
    # travel to the host while step n+1's inputs arrive and step n+1 runs;
    # a set is refilled only after its previous results have left.
    h_in = [t for t in host[:3]] + ([host[3]] if wl.backward else []) + \
        ([host[-1]] if wl.prior else [])
    h2d = sum(t.numel() * t.element_size() for t in h_in) + alpha_h.numel() * 4
    sets = []
    for b in range(2):
        d_in = [torch.empty_like(t, device=dev) for t in h_in]
        d_alpha = torch.empty_like(alpha)
        d_out = [torch.empty_like(q), torch.empty(q.shape[:4], dtype=torch.float32, device=dev)]
        if wl.backward:
            d_out += [torch.empty_like(q), torch.empty_like(q), torch.empty_like(q),
                      torch.empty(wl.L, dtype=torch.float32, device=dev)]
            if wl.prior:
                d_out += [torch.empty_like(beta)]
        h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in d_out]
        sets.append((d_in, d_alpha, d_out, h_out))
    d2h = sum(t.numel() * t.element_size() for t in sets[0][2])
    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    started = [False, False]

    def e2e_step(n):
        b = n % 2
        d_in, d_alpha, d_out, h_out = sets[b]
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(ev_out[b])        # this set's last results have left
            for hs, ds in zip(h_in, d_in):
                ds.copy_(hs, non_blocking=True)
            d_alpha.copy_(alpha_h, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_in[b])
            qq, kk_, vv = d_in[:3]
            dd = d_in[3] if wl.backward else None
            bb = d_in[-1] if wl.prior else None
            sa.fwd(qq, kk_, vv, d_alpha, out=d_out[0], lse=d_out[1], stream=s_run,
                   context=ctx if wl.backward else None, beta=bb, **kw)
            if wl.backward:
                sa.bwd(qq, kk_, vv, d_out[0], d_out[1], dd, d_alpha, dq=d_out[2], dk=d_out[3],
                       dv=d_out[4], dalpha=d_out[5], workspace=ws, stream=s_run, context=ctx,
                       beta=bb, dbeta=d_out[6] if wl.prior else None, **kw)
            ev_run[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[b])
            for ho, dv_ in zip(h_out, d_out):
                ho.copy_(dv_, non_blocking=True)
            ev_out[b].record(s_out)
        started[b] = True

    for n in range(2):
        e2e_step(n)
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s_in)
    for n in range(args.steps):
        e2e_step(n)
    s_in.wait_stream(s_out)
    s_in.wait_stream(s_run)
    f1.record(s_in)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), dev)
    e2e = {"value": aggregate_throughput(wl.token_heads, world, args.steps, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": e2e_ms / args.steps}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(wl, args.cpu_budget_s, single_thread=True)

    # the other benchmark configurations, forward only, timed the same way
    # (every rank runs them, so that all ranks take the same steps)
    workloads = None
    if not args.no_workloads:
        del q, k, v, o, lse, host, sets
        if wl.backward:
            del dq, dk, dv, ws, ctx, do
        torch.cuda.empty_cache()
        workloads = {}
        for name in OTHER_WORKLOADS:
            if name != wl.name:
                workloads[name] = time_forward_workload(sa, torch, dev, name, args.steps,
                                                        args.warmup, peak, alu["peak"])

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32", "data": "synthetic",
                "config": workload_config(wl, world), "roofline": roofline,
                "roofline_alu": roofline_alu, "alu_peak": alu,
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": gpu_launches, "clocks": clocks,
                "kernels": kernels, "kernel_source": kernel_source_hash()}
        if workloads is not None:
            line["workloads"] = workloads
        print(json.dumps(line), flush=True)
    return 0


def run_ours_decode(args, rank, world, local_rank):
    """Decode workloads: one new token per (layer, batch, head) at position
    T - 1 against resident KV caches.  A step is one decode call over all
    units; end to end, each step copies the new token's q, k and v rows in
    (written into the caches at T - 1) and O and LSE out."""
    import torch
    import structured_sparse_attention_fibonacci_b200 as sa
    from structured_sparse_attention_fibonacci_b200.inputs import WORKLOADS, make_decode_inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[args.workload]
    wl_rank = wl.shrink(seed=wl.seed + 100000 * rank) if world > 1 else wl
    q1_h, kc_h, vc_h = make_decode_inputs(wl_rank, pin=True)
    q1, kc, vc = q1_h.to(dev), kc_h.to(dev), vc_h.to(dev)
    alpha_h = wl.alpha().pin_memory()
    alpha = alpha_h.to(dev)
    pos = wl.T - 1
    kw = dict(window=wl.window, sinks=wl.sinks, offsets=wl.offsets, rope_base=wl.rope_base)
    o = torch.empty_like(q1)
    lse = torch.empty(q1.shape[:3], dtype=torch.float32, device=dev)
    units = wl.L * wl.B * wl.H
    launches = [0]

    def step():
        sa.decode(q1, kc, vc, alpha, pos, out=o, lse=lse, **kw)
        launches[0] += sa.last_launch_count()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # The timed steps replay one CUDA graph of the K decode calls: a
    # single-token step (~17 us of GPU time) is shorter than a host-side call
    # through the binding, so launching the steps one by one from Python
    # would time the host, not the GPU.  The end-to-end figure below still
    # makes one public call per step.
    launches[0] = 0
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(args.steps):
            step()
    gpu_launches = launches[0]
    graph.replay()
    torch.cuda.synchronize()
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.4)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    ms_max = max_over_ranks(e0.elapsed_time(e1), dev)
    value = aggregate_throughput(units, world, args.steps, ms_max)
    del graph

    sa.trace_enable(True)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    trace = sa.trace_read()
    sa.trace_enable(False)
    kernels = {n: {"ms_per_launch": t / c, "launches": c} for n, (t, c) in trace.items()}
    elt = 2 if wl.dtype == torch.bfloat16 else 4
    peak, peak_kind = measured_peaks()
    bytes_launch = decode_bytes_per_token_head(wl, elt) * units
    # a step is exactly one decode launch: its device time is the graph's
    # time per step (the traced launches above also hold the host's gaps)
    achieved = bytes_launch / (ms_max / args.steps / 1e3) / 1e9
    src_hash = kernel_source_hash()
    traffic = MEASURED_TRAFFIC.get(f"{wl.name}/decode@{src_hash}")
    roofline = {"bound": "hbm", "kernel": "decode", "achieved": achieved, "peak": peak,
                "peak_source": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                "alg_bytes_per_launch": bytes_launch,
                "traffic": traffic * units if traffic is not None else None,
                "traffic_source": (f"ncu@{src_hash}" if traffic is not None else
                                   f"none: no ncu capture of sources {src_hash}")}

    # end to end: the new token's q, k, v rows in, O and LSE out, every step
    kr_h = kc_h[:, :, :, pos].contiguous().pin_memory()
    vr_h = vc_h[:, :, :, pos].contiguous().pin_memory()
    o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    lse_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    kr, vr = torch.empty_like(kr_h, device=dev), torch.empty_like(vr_h, device=dev)
    h2d = (q1_h.numel() + kr_h.numel() + vr_h.numel()) * q1_h.element_size() + alpha_h.numel() * 4
    d2h = o.numel() * o.element_size() + lse.numel() * 4

    def e2e_step():
        q1.copy_(q1_h, non_blocking=True)
        kr.copy_(kr_h, non_blocking=True)
        vr.copy_(vr_h, non_blocking=True)
        alpha.copy_(alpha_h, non_blocking=True)
        kc[:, :, :, pos].copy_(kr)
        vc[:, :, :, pos].copy_(vr)
        step()
        o_h.copy_(o, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    f1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), dev)
    e2e = {"value": aggregate_throughput(units, world, args.steps, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": e2e_ms / args.steps}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(wl, args.cpu_budget_s, single_thread=True)
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32", "data": "synthetic",
                "config": workload_config(wl, world), "roofline": roofline,
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": gpu_launches, "clocks": clocks,
                "kernels": kernels, "kernel_source": kernel_source_hash()}
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="learned_train")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the forward timings of the other configurations")
    ap.add_argument("--forward", choices=tuple(FORWARD_KERNELS), default="auto",
                    help="forward kernel of the plain (non-training) forwards")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--reference-budget-s", type=float, default=120.0)
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        from structured_sparse_attention_fibonacci_b200.inputs import WORKLOADS
        if WORKLOADS[args.workload].decode:
            return run_ours_decode(args, rank, world, local_rank)
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
