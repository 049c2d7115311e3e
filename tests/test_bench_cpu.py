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
