"""CPU checks of bench.py's bookkeeping (no GPU, no kernels): every named workload
builds, its algorithmic counts are the closed forms the roofline uses, the roofline
object carries the contract's fields, and the reference arm's JSON line has the keys
the contract asks for."""
import json
import math
import os
import subprocess
import sys

import pytest
import torch

import bench
from gated_linear_attention_local_b200.workloads import WORKLOADS, make_workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_every_workload_has_counts_config_and_roofline(name):
    w = make_workload(name)
    c = bench.algorithmic_counts(w)
    assert c["bytes"] > 0 and c["flops"] > 0
    cfg = bench._config_of(w)
    assert isinstance(cfg, dict) and cfg
    kernel = next(iter(c.get("kernel", {"chunk_output_tc": None})))
    r = bench.roofline(dict(w, dtype_name="bf16"), c, 0.1, bench.load_peaks(), None, kernel)
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(r)
    assert r["bound"] in ("hbm", "tensor", "alu")
    # achieved is rounded for the JSON line; frac comes from the unrounded value
    assert math.isclose(r["frac"], r["achieved"] / r["peak"], rel_tol=1e-2, abs_tol=1e-4)


def test_dense_prefill_counts_are_the_closed_form():
    w = make_workload("dense_prefill")
    B, T, H, K, V, C = w["B"], w["T"], w["H"], w["K"], w["V"], w["chunk_size"]
    c = bench.algorithmic_counts(w)
    tokens = B * T
    assert c["tokens"] == tokens
    assert c["flops"] == H * (4 * tokens * K * V + tokens * (C + 1) * (K + V))
    io = tokens * H * (2 * K + 2 * V) * 2 + tokens * H * 4 + B * H * K * V * 4  # q,k,v,o bf16; g; final state
    assert c["bytes"] == io


def test_decode_counts_are_state_bytes_plus_io():
    w = make_workload("decode")
    N, H, K, V = w["N"], w["H"], w["K"], w["V"]
    c = bench.algorithmic_counts(w)
    assert c["bytes"] == 2 * N * H * K * V * 4 + N * H * (2 * K + 2 * V) * 2 + N * H * 4


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_fp32", "--steps", "1", "--warmup", "1"], capture_output=True, text=True, timeout=600,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling", "dtype",
                "config", "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    # per-step time: the whole tiny step (B*T tokens) at the sampled rate
    w = make_workload("tiny_fp32")
    assert math.isclose(line["ms_per_step"], w["B"] * w["T"] / line["value"] * 1e3, rel_tol=1e-9)


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    import socket
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    out = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                          "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
                          "--impl", "reference", "--gpus", "2", "--workload", "tiny_fp32", "--steps", "1",
                          "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0


def test_step_time_is_the_median_with_p10_p90():
    xs = [5.0, 1.0, 3.0, 2.0, 4.0]
    assert bench.percentile(xs, 50) == 3.0
    assert bench.percentile(xs, 0) == 1.0 and bench.percentile(xs, 100) == 5.0
    assert math.isclose(bench.percentile(xs, 10), 1.4) and math.isclose(bench.percentile(xs, 90), 4.6)


def test_secondary_workloads_end_with_the_hot_path_ones():
    order = bench.secondary_order("long_gamma")
    assert "long_gamma" not in order and set(order) == set(WORKLOADS) - {"long_gamma"}
    assert order[-4:] == ["tiny_fp32", "dense_prefill", "varlen_prefill", "decode"]
    r = dict(value=1.2345678e7, unit="tokens/s", ms_per_step=0.5, ms_p10=0.4, ms_p90=0.6,
             roofline=dict(bound="hbm", frac=0.5), call_roofline_frac=0.4,
             dominant_kernel=dict(name="chunk_output_tc", avg_ms=0.3), gpu_launches=10,
             clocks=dict(reasons=[], sm_mhz=1965.0))
    c = bench.compact(r)
    assert c["frac"] == 0.5 and c["kernel"] == "chunk_output_tc" and len(json.dumps(c)) < 300
