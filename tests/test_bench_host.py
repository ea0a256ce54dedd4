"""Host-side pieces of bench.py (no GPU): the byte accounting behind the
roofline, the workload description in the JSON line, and the measured-traffic
table's keys."""
import re

import bench
from structured_sparse_attention_fibonacci_b200.inputs import WORKLOADS


def test_algorithmic_bytes_per_token_head():
    """The roofline bytes follow the problem's definition: the forward's unique
    Q, K, V and O (512 B per token-head at d = 64, bf16) and the backward's
    Q, K, V, O, dO, dQ, dK, dV and LSE (1028 B), split between the two
    backward kernels as they touch the tensors; intermediates count 0."""
    assert bench.alg_bytes_per_token_head("fwd_fast", 64, 2) == 4 * 128 == 512
    assert bench.alg_bytes_per_token_head("fwd_tc", 64, 2) == 512
    assert bench.alg_bytes_per_token_head("fwd_fast", 64, 2, prior=True) == 516
    # query side: Q, K, V, dO, LSE read, dQ written; key side: dK, dV written, O
    assert bench.alg_bytes_per_token_head("bwd_q_fast", 64, 2) == 5 * 128 + 4 == 644
    assert bench.alg_bytes_per_token_head("bwd_kv_fast", 64, 2) == 3 * 128 == 384
    assert (bench.alg_bytes_per_token_head("bwd_q_fast", 64, 2)
            + bench.alg_bytes_per_token_head("bwd_kv_fast", 64, 2)
            == bench.phase_bytes_per_token_head("backward", 64, 2) == 1028)
    assert bench.phase_bytes_per_token_head("forward", 64, 2) == 512
    assert bench.phase_bytes_per_token_head("forward", 16, 4) == 256      # the fp32 d = 16 case
    # pre-passes, the training context and reductions are intermediates
    assert bench.alg_bytes_per_token_head("rope_keys", 64, 2) == 0
    assert bench.alg_bytes_per_token_head("reduce_dalpha", 64, 2) == 0


def test_distinct_rows_and_flops():
    """At alpha = 1 the Fibonacci ladder's lags 1, 2, 3, 5, 8 fall in the
    window of 12 and 13 .. 987 add 10 rows (integer distances read one row);
    a non-integer alpha reads both rows of every far offset."""
    assert bench.distinct_rows(1.0, WORKLOADS["paper_fwd"].offsets, 12, 0) == 22
    assert bench.distinct_rows(1.0, WORKLOADS["long_sinks"].offsets, 64, 4) == 64 + 6 + 4
    # alpha = 1.1234: lags 1, 2, 3, 5, 8, 14 lie in or next to the window
    n = bench.distinct_rows(1.1234, WORKLOADS["paper_fwd"].offsets, 12, 0)
    assert 12 + 2 * 8 <= n <= 12 + 2 * 10
    wl = WORKLOADS["tiny_fp32"]
    assert bench.alg_flops(wl, "forward") == 4 * 16 * bench.distinct_rows(1.0, wl.offsets, 6, 0) * 128
    lt = WORKLOADS["learned_train"]
    assert bench.alg_flops(lt, "backward") == 2 * bench.alg_flops(lt, "forward")
    assert (bench.kernel_flops(lt, "bwd_q_fast") + bench.kernel_flops(lt, "bwd_kv_fast")
            == bench.alg_flops(lt, "backward"))


def test_decode_bytes_count_every_member_row():
    wl = WORKLOADS["decode_4k"]
    rows = wl.window + wl.sinks + 2 * len(wl.offsets)          # 12 + 0 + 30
    assert bench.decode_bytes_per_token_head(wl, 2) == 2 * 128 + 4 + 2 * rows * 128 == 11012


def test_workload_config_names_the_workload():
    for name, wl in WORKLOADS.items():
        cfg = bench.workload_config(wl, 1)
        assert cfg["workload"] == name
        assert (cfg["L"], cfg["B"], cfg["H"], cfg["T"], cfg["D"]) == (wl.L, wl.B, wl.H, wl.T, wl.D)
        assert cfg["parallelism"] == "replicas1" and cfg["global_batch"] == wl.B
        assert ("prior" in cfg) == wl.prior
        assert ("launch" in cfg) == wl.decode
    assert bench.workload_config(WORKLOADS["learned_train"], 4)["global_batch"] == 32


def test_measured_traffic_keys_name_workload_kernel_and_source_hash():
    for key, per_unit in bench.MEASURED_TRAFFIC.items():
        m = re.fullmatch(r"([a-z0-9_]+)/([a-z_]+)@([0-9a-f]{12})", key)
        assert m, key
        assert m.group(1) in WORKLOADS, key
        assert per_unit > 0
    # one capture campaign: every entry was taken on the same sources (a
    # source change makes the bench report null until they are re-measured)
    hashes = {k.split("@")[1] for k in bench.MEASURED_TRAFFIC}
    assert len(hashes) <= 1
    assert re.fullmatch(r"[0-9a-f]{12}", bench.kernel_source_hash())


def test_aggregate_throughput_is_whole_job_units_per_second():
    # 1048576 token-heads per rank, 4 ranks, 20 steps in 40 ms
    assert bench.aggregate_throughput(1048576, 4, 20, 40.0) == 1048576 * 4 * 20 / 0.040


def test_reference_arm_prints_one_json_line():
    """`bench.py --impl reference` (the CPU oracle) on the tiny workload: one
    JSON line with the contract's keys."""
    import json
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(here, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_fp32", "--steps", "2", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, cwd=here)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
