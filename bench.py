#!/usr/bin/env python
"""Benchmark of the Simple GLA forward (and decode step) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

One JSON line on rank 0.  A "step" is one pass of the whole forward hot path --
plan, chunk cumsum, segment states, carry, fused output walk -- over one batch of
the named workload (default: long_gamma, B=1 T=65536 H=32 K=V=128 bf16 with a
per-head decay -- the largest single-GPU workload), with inputs resident in HBM.
Each step is timed with CUDA events on the launching stream; L2 is flushed
(256 MiB write) between steps, outside the events; the step time reported is the
median over the timed steps (p10 and p90 beside it).  The other workloads are
measured the same way and reported, in compact form, under "secondary" (last key
of the line; the dense, packed and decode workloads are its last entries).

Multi-GPU (torchrun, one process per GPU): every (sequence, head) is independent,
so each rank runs its own batch of the workload with no collective on the data
path (weak scaling); the timed region is bracketed by a barrier and a device
synchronize, and the step time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only reference this method has:
the pages ship no implementation) on this machine's host cores, on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import functools
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Simple GLA fwd tokens/s & % roofline; decode-step state GB/s"
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------- counts

def algorithmic_counts(w):
    """Compulsory bytes and causal FLOPs of one forward (or one decode step).

    FLOPs per head = 4*T*K*V + T*(C+1)*(K+V): the state update and q.h_prev
    (2*T*K*V each) plus the causal half of the intra-chunk q k^T and P v.
    Bytes: q, k, v, g (or g_gamma), o, initial and final state, each moved once."""
    if w["kind"] == "decode":
        N, H, K, V = w["N"], w["H"], w["K"], w["V"]
        e = 2  # bf16 operands
        state = 2 * N * H * K * V * 4
        io = N * H * (2 * K + 2 * V) * e + N * H * 4
        flops = N * H * 4 * K * V
        return dict(bytes=state + io, flops=flops, tokens=N)
    H, K, V, C = w["H"], w["K"], w["V"], w["chunk_size"]
    tokens = w["B"] * w["T"] if w["kind"] == "dense" else w["T"]
    e = w["q"].element_size()
    b = tokens * H * (2 * K + 2 * V) * e
    b += w["g"].numel() * 4 if w["g"] is not None else (H * 4 if w["g_gamma"] is not None else 0)
    states = w["N"] * H * K * V * 4
    if w["h0"] is not None:
        b += states
    if w["output_final_state"]:
        b += states
    flops = H * (4 * tokens * K * V + tokens * (C + 1) * (K + V))
    if w.get("entry") in ("recurrent", "gla", "gla_chunk"):  # state update and read-out per token
        flops = H * tokens * 4 * K * V
    if w.get("entry") == "gla_chunk":
        # prep (CUDA cores): the causal half of the intra-chunk q k^T with per-key decays,
        # 128-token chunks; walk (tensor cores): q~ h, A v and the state update
        Cg = 128
        prep = dict(bytes=b, flops=H * tokens * (Cg + 1) * K)
        walk = dict(bytes=b, flops=H * tokens * (4 * K * V + (Cg + 1) * V))
        return dict(bytes=b, flops=prep["flops"] + walk["flops"], tokens=tokens,
                    kernel={"gla_chunk_prep": prep, "gla_chunk_walk_tc": walk})
    if w.get("entry") in ("recurrent_bwd", "chunk_bwd"):
        fwd = dict(bytes=b, flops=flops)  # one forward call with these operands (K == V)
        # read do; write dq, dk, dv, dg; read dht, write dh0
        b += tokens * H * (V + 2 * K + V) * e + w["g"].numel() * 4 + 2 * states
        if w["entry"] == "chunk_bwd":
            # three chunked forward calls (dv, dk, dq); the output walk of each moves
            # that call's compulsory bytes
            return dict(bytes=b, flops=3 * flops, tokens=tokens, kernel={"chunk_output_tc": fwd})
        # token-serial FLOPs per token and head: forward sweep 4KV (state update, dq)
        # and reverse sweep 6KV (dS update, dk, dv), one launch
        kernel = {"recurrent_bwd_sweeps": dict(bytes=b, flops=H * tokens * 10 * K * V)}
        return dict(bytes=b, flops=H * tokens * 10 * K * V, tokens=tokens, kernel=kernel)
    return dict(bytes=b, flops=flops, tokens=tokens)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# The source files each timed kernel is built from (its own file plus the shared
# headers), so that a stored ncu capture stays valid while unrelated files change.
_CSRC_COMMON = ["common.cuh", "kernels.h"]
KERNEL_SOURCES = {
    "chunk_output_tc": ["chunk_tc.cu", "walk_k128.cu", "walk_k512.cu", "tc_ptx.cuh", "tc_tiles.cuh", "tc_path.h"],
    "segment_state_tc": ["chunk_tc.cu", "state_k128.cu", "tc_ptx.cuh", "tc_tiles.cuh", "tc_path.h"],
    "decode_step": ["decode.cu"],
    "fused_recurrent": ["recurrent.cu"],
    "gla_fused_recurrent": ["recurrent.cu"],
    "recurrent_bwd_sweeps": ["recurrent_bwd.cu"],
    "recurrent_bwd_rows": ["recurrent_bwd.cu"],
    "gla_chunk_prep": ["gla_chunk.cu", "tc_ptx.cuh"],
    "bwd_reverse_inputs": ["chunk_bwd.cu"],
    "gla_chunk_walk_tc": ["gla_chunk_tc.cu", "tc_ptx.cuh", "tc_path.h"],
}


def sources_hash(kernel=None):
    """sha256[:16] of the CUDA sources a kernel is built from (all of csrc/ when the
    kernel is not listed), to tell whether a stored ncu capture still describes the
    kernel that runs."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_linear_attention_local_b200", "csrc")
    if kernel in KERNEL_SOURCES:
        paths = [os.path.join(csrc, f) for f in sorted(set(KERNEL_SOURCES[kernel] + _CSRC_COMMON))]
    else:
        paths = sorted(glob.glob(os.path.join(csrc, "*")))
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def captured_traffic(workload, kernel):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu capture
    (profiles/traffic.json), or None when there is none or the kernel's sources
    changed since."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[workload][kernel]
    except (OSError, KeyError, ValueError):
        return None
    if rec.get("sources_sha256_16") != sources_hash(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


# FP32 CUDA-core peak: 148 SMs x 128 FP32 lanes x 2 flops (FMA) x 1965 MHz max SM clock
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def roofline(w, counts, kernel_ms, peaks, traffic=None, kernel=None):
    """Roofline object for the dominant kernel of this workload.  The fused output
    walk (or the decode kernel) moves all compulsory bytes of the call.  The
    token-serial recurrence runs on the FP32 CUDA cores (two FMAs and a multiply per
    state element and token), so its bound is the ALU peak."""
    kc = counts.get("kernel", {}).get(kernel, counts)  # per-launch counts of that kernel
    if w.get("entry") in ("recurrent", "gla", "gla_chunk", "recurrent_bwd"):
        ach = kc["flops"] / (kernel_ms * 1e-3) / 1e12
        return dict(bound="alu", achieved=round(ach, 3), peak=round(FP32_ALU_TFLOPS, 1), unit="TFLOP/s",
                    frac=round(ach / FP32_ALU_TFLOPS, 4), traffic=traffic,
                    peak_source="derived: 148 SMs x 128 FP32 lanes x 2 x 1965 MHz")
    t_bytes = kc["bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_flops = kc["flops"] / (peaks["bf16_tflops"] * 1e12)
    if w["kind"] != "decode" and w.get("dtype_name") == "fp32":
        t_flops = 0.0  # FFMA path: never tensor-bound; report HBM
    if t_flops > t_bytes:
        ach = kc["flops"] / (kernel_ms * 1e-3) / 1e12
        return dict(bound="tensor", achieved=round(ach, 3), peak=peaks["bf16_tflops"], unit="TFLOP/s",
                    frac=round(ach / peaks["bf16_tflops"], 4), traffic=traffic,
                    peak_source=peaks["source"])
    ach = kc["bytes"] / (kernel_ms * 1e-3) / 1e9
    return dict(bound="hbm", achieved=round(ach, 1), peak=peaks["hbm_gbs"], unit="GB/s",
                frac=round(ach / peaks["hbm_gbs"], 4), traffic=traffic, peak_source=peaks["source"])


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.lines = []
        sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            pass
        self.cmd = ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                    "-lms", "100"]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, pw, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
                pw.append(float(parts[3]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=[], samples=0)
        # samples under load: power above the midpoint of the observed range
        lo, hi = min(pw), max(pw)
        loaded = [s for s, p in zip(sm, pw) if p >= lo + 0.5 * (hi - lo)] or sm
        return dict(sm_mhz=statistics.median(loaded), sm_max_mhz=mx, reasons=sorted(reasons),
                    samples=len(sm), power_w_max=hi)


# ----------------------------------------------------------------------------- running

def dev_inputs(w, device):
    keys = ("q", "k", "v", "g", "g_gamma", "h0", "cu_seqlens", "state", "do", "dht")
    return {k: (w[k].to(device) if w.get(k) is not None else None) for k in keys}


def make_step(w, d, sg, ws):
    if w["kind"] == "decode":
        S = w["steps"]
        state0 = d["state"].clone()
        o = torch.empty(w["N"], w["H"], w["V"], dtype=d["q"].dtype, device=d["q"].device)

        def reset():
            d["state"].copy_(state0)

        def step():
            for t in range(S):
                sg.simple_gla_decode_step(d["q"][t], d["k"][t], d["v"][t], d["state"], g=d["g"][t],
                                          scale=w["scale"], out=o)
        return step, reset
    if w.get("entry") == "normalized":
        def step():
            sg.simple_gla_normalized(d["q"], d["k"], d["v"], g=d["g"], g_gamma=d["g_gamma"], initial_state=d["h0"],
                                     output_final_state=w["output_final_state"], chunk_size=w["chunk_size"],
                                     workspace=ws)
        return step, (lambda: None)
    if w.get("entry") == "gla_chunk":
        def step():
            sg.gla_chunk(d["q"], d["k"], d["v"], d["g"], scale=w["scale"], initial_state=d["h0"],
                         output_final_state=w["output_final_state"], workspace=ws)
        return step, (lambda: None)
    if w.get("entry") == "gla":
        def step():
            sg.gla_fused_recurrent(d["q"], d["k"], d["v"], d["g"], scale=w["scale"], initial_state=d["h0"],
                                   output_final_state=w["output_final_state"])
        return step, (lambda: None)
    if w.get("entry") in ("recurrent_bwd", "chunk_bwd"):
        fn = sg.simple_gla_fused_recurrent_bwd if w["entry"] == "recurrent_bwd" else \
            functools.partial(sg.simple_gla_chunk_bwd, chunk_size=w["chunk_size"])

        def step():
            fn(d["q"], d["k"], d["v"], d["do"], g=d["g"], g_gamma=d["g_gamma"], scale=w["scale"],
               initial_state=d["h0"], dht=d["dht"], workspace=ws)
        return step, (lambda: None)
    if w.get("entry") == "recurrent":
        def step():
            sg.simple_gla_fused_recurrent(d["q"], d["k"], d["v"], g=d["g"], g_gamma=d["g_gamma"], scale=w["scale"],
                                          initial_state=d["h0"], output_final_state=w["output_final_state"])
        return step, (lambda: None)
    if w["kind"] == "varlen":
        def step():
            sg.simple_gla_fwd_varlen(d["q"], d["k"], d["v"], d["cu_seqlens"], g=d["g"], g_gamma=d["g_gamma"],
                                     scale=w["scale"], initial_state=d["h0"],
                                     output_final_state=w["output_final_state"], chunk_size=w["chunk_size"],
                                     workspace=ws)
    else:
        def step():
            sg.simple_gla_fwd(d["q"], d["k"], d["v"], g=d["g"], g_gamma=d["g_gamma"], scale=w["scale"],
                              initial_state=d["h0"], output_final_state=w["output_final_state"],
                              chunk_size=w["chunk_size"], workspace=ws)
    return step, (lambda: None)


def workspace_for(w, sg, device):
    if w["kind"] == "decode" or w.get("entry") in ("recurrent", "gla"):
        return None
    dt = w["q"].dtype
    if w.get("entry") == "recurrent_bwd":
        n = sg.lib().simple_gla_fused_recurrent_bwd_workspace_size(None, w["B"], w["T"], w["H"], w["K"])
        return torch.empty(max(int(n), 256), dtype=torch.uint8, device=device)
    if w.get("entry") == "gla_chunk":
        n = sg.lib().gla_chunk_workspace_size(None, w["B"], w["T"], w["H"], w["K"], w["V"], sg._DTYPES[dt])
        return torch.empty(max(int(n), 256), dtype=torch.uint8, device=device)
    if w.get("entry") == "chunk_bwd":
        n = sg.lib().simple_gla_chunk_bwd_workspace_size(None, w["B"], w["T"], w["H"], w["K"], w["V"],
                                                         w["chunk_size"], sg._DTYPES[dt])
        return torch.empty(max(int(n), 256), dtype=torch.uint8, device=device)
    if w.get("entry") == "normalized":
        n = sg.lib().simple_gla_normalized_workspace_size(None, w["B"], w["T"], w["H"], w["K"], w["V"],
                                                          w["chunk_size"], sg._DTYPES[dt])
        return torch.empty(max(int(n), 256), dtype=torch.uint8, device=device)
    if w["kind"] == "varlen":
        n = sg.varlen_workspace_size(w["N"], w["T"], w["H"], w["K"], w["V"], w["chunk_size"], dt)
    else:
        n = sg.fwd_workspace_size(w["B"], w["T"], w["H"], w["K"], w["V"], w["chunk_size"], dt)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def time_steps(step, reset, steps, warmup, flush, dist_on, profile=True):
    """Time `steps` steps with CUDA events on the launching stream (L2 flushed before
    each, outside the events).  The timed steps run without the library's per-kernel
    event recording; when `profile` is set, a separate pass of min(steps, 5) steps
    afterwards records the per-kernel times."""
    from gated_linear_attention_local_b200 import _lib
    for _ in range(warmup):
        reset()
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    n0 = _lib.kernel_launch_count()
    for i in range(steps):
        reset()
        flush.zero_()
        evs[i][0].record()
        step()
        evs[i][1].record()
    torch.cuda.synchronize()
    launches = _lib.kernel_launch_count() - n0
    if dist_on:
        torch.distributed.barrier()
    per_step = [a.elapsed_time(b) for a, b in evs]
    prof = {}
    if profile:
        _lib.profile_begin()
        for _ in range(min(steps, 5)):
            reset()
            flush.zero_()
            step()
        torch.cuda.synchronize()
        prof = _lib.profile_end()
    return per_step, prof, launches


def percentile(xs, p):
    """p-th percentile of xs (linear interpolation between order statistics)."""
    ys = sorted(xs)
    if not ys:
        return float("nan")
    x = (len(ys) - 1) * p / 100.0
    lo = int(math.floor(x))
    hi = min(lo + 1, len(ys) - 1)
    return ys[lo] + (ys[hi] - ys[lo]) * (x - lo)


def dominant(prof):
    if not prof:
        return None, 0, 0.0
    name = max(prof, key=lambda k: prof[k][1])
    n, ms = prof[name]
    return name, n, ms


def e2e_measure(w, sg, device, steps, warmup):
    """Same metric through the public API with inputs in pinned HOST memory.  Every
    step uploads its inputs host->device, runs the call and reads its results back
    into pinned host memory.  Steps are pipelined over three streams (upload,
    compute, read-back) with two device input buffers, so the upload of step i+1 and
    the read-back of step i-1 overlap the compute of step i (each PCIe direction has
    its own copy engine).  The time is taken with events from before the first
    upload to after the last read-back.  Returns (ms per step, h2d bytes per step,
    d2h bytes per step)."""
    keys = [k for k in ("q", "k", "v", "g", "g_gamma", "h0", "cu_seqlens", "do", "dht") if w.get(k) is not None]
    if w["kind"] == "decode":
        keys = ["q", "k", "v", "g", "state"]
    hostin = {k: w[k].pin_memory() for k in keys}
    h2d = sum(t.numel() * t.element_size() for t in hostin.values())
    bufs = [{k: torch.empty(t.shape, dtype=t.dtype, device=device) for k, t in hostin.items()} for _ in range(2)]
    ws = workspace_for(w, sg, device)
    host_out = {}

    def call(d):
        """One public-API call on the current (compute) stream; returns the device
        tensors to read back, by name."""
        if w["kind"] == "decode":
            outs = {}
            for t in range(w["steps"]):
                outs[f"o{t}"] = sg.simple_gla_decode_step(d["q"][t], d["k"][t], d["v"][t], d["state"], g=d["g"][t],
                                                          scale=w["scale"])
            outs["state"] = d["state"]
            return outs
        if w.get("entry") in ("recurrent_bwd", "chunk_bwd"):
            fn = sg.simple_gla_fused_recurrent_bwd if w["entry"] == "recurrent_bwd" else \
                functools.partial(sg.simple_gla_chunk_bwd, chunk_size=w["chunk_size"])
            r = fn(d["q"], d["k"], d["v"], d["do"], g=d.get("g"), g_gamma=d.get("g_gamma"), scale=w["scale"],
                   initial_state=d.get("h0"), dht=d.get("dht"), workspace=ws)
            return {n: r[n] for n in ("dq", "dk", "dv", "dg", "dh0") if r.get(n) is not None}
        if w["kind"] == "varlen":
            o, ht = sg.simple_gla_fwd_varlen(d["q"][0], d["k"][0], d["v"][0], d["cu_seqlens"], g=d["g"][0],
                                             g_gamma=d.get("g_gamma"), scale=w["scale"], initial_state=d.get("h0"),
                                             output_final_state=w["output_final_state"],
                                             chunk_size=w["chunk_size"], workspace=ws)
        elif w.get("entry") == "normalized":
            o, ht = sg.simple_gla_normalized(d["q"], d["k"], d["v"], g=d.get("g"), g_gamma=d.get("g_gamma"),
                                             initial_state=d.get("h0"), output_final_state=w["output_final_state"],
                                             chunk_size=w["chunk_size"], workspace=ws)
        elif w.get("entry") == "gla_chunk":
            o, ht = sg.gla_chunk(d["q"], d["k"], d["v"], d["g"], scale=w["scale"], initial_state=d.get("h0"),
                                 output_final_state=w["output_final_state"], workspace=ws)
        elif w.get("entry") == "gla":
            o, ht = sg.gla_fused_recurrent(d["q"], d["k"], d["v"], d["g"], scale=w["scale"],
                                           initial_state=d.get("h0"), output_final_state=w["output_final_state"])
        elif w.get("entry") == "recurrent":
            o, ht = sg.simple_gla_fused_recurrent(d["q"], d["k"], d["v"], g=d.get("g"), g_gamma=d.get("g_gamma"),
                                                  scale=w["scale"], initial_state=d.get("h0"),
                                                  output_final_state=w["output_final_state"])
        else:
            o, ht = sg.simple_gla_fwd(d["q"], d["k"], d["v"], g=d.get("g"), g_gamma=d.get("g_gamma"),
                                      scale=w["scale"], initial_state=d.get("h0"),
                                      output_final_state=w["output_final_state"], chunk_size=w["chunk_size"],
                                      workspace=ws)
        outs = {"o": o}
        if ht is not None:
            outs["final_state"] = ht
        return outs

    comp = torch.cuda.current_stream(device)
    s_up, s_down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer b uploaded
    ev_used = [torch.cuda.Event() for _ in range(2)]  # the call reading buffer b has been enqueued after
    used = [False, False]

    def one(i):
        b = i % 2
        d = bufs[b]
        with torch.cuda.stream(s_up):
            if used[b]:
                s_up.wait_event(ev_used[b])
            for k, t in hostin.items():
                d[k].copy_(t, non_blocking=True)
            ev_in[b].record(s_up)
        comp.wait_event(ev_in[b])
        outs = call(d)
        ev_used[b].record(comp)
        used[b] = True
        s_down.wait_event(ev_used[b])
        with torch.cuda.stream(s_down):
            for n, t in outs.items():
                if n not in host_out:
                    host_out[n] = torch.empty(t.shape, dtype=t.dtype).pin_memory()
                host_out[n].copy_(t, non_blocking=True)
                t.record_stream(s_down)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize(device)
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    s_up.wait_event(a)
    s_down.wait_event(a)
    for i in range(steps):
        one(i)
    done = torch.cuda.Event()
    done.record(s_down)
    comp.wait_event(done)
    b.record(comp)
    torch.cuda.synchronize(device)
    return a.elapsed_time(b) / steps, h2d, d2h


# ----------------------------------------------------------------------------- CPU oracle leg

def oracle_sample(w, budget_s=4.0, repeats=3):
    """Time the fp64 oracle on a bounded sample of the workload: all heads and
    sequences, a prefix of the tokens (decode: a subset of the sequences), sized
    from a short calibration run to take about budget_s seconds per run; the rate
    is the median of `repeats` runs of that sample.  Both bench arms (the native
    arm's cpu_baseline leg and --impl reference) time the oracle through this one
    function, so their figures differ only by run-to-run noise of the host."""
    import oracle
    threads = oracle.default_threads()
    if w["kind"] == "decode":
        def run(nseq):
            st = w["state"][:nseq].double().numpy().copy()
            t0 = time.perf_counter()
            for t in range(w["steps"]):
                oracle.simple_gla_decode_step(w["q"][t, :nseq], w["k"][t, :nseq], w["v"][t, :nseq], st,
                                              g=w["g"][t, :nseq], scale=w["scale"], threads=threads)
            return time.perf_counter() - t0
        cal = run(4)
        nseq = int(max(4, min(w["N"], 4 * budget_s / max(cal, 1e-6))))
        dt = statistics.median(run(nseq) for _ in range(repeats))
        # unit: GB/s over the sampled sequences, all steps, counting the bytes of a
        # step as the native arm does (state read + write and the step's q, k, v, g, o)
        gb = w["steps"] * algorithmic_counts(w)["bytes"] * nseq / w["N"] / 1e9
        return dict(value=gb / dt, unit="GB/s", cores=threads, kind="oracle",
                    sample=f"{nseq} of {w['N']} sequences x {w['steps']} steps, all heads "
                           f"(median of {repeats} runs of {dt:.1f} s)")

    def sub(tn):
        d = {}
        if w["kind"] == "varlen":
            cu = w["cu_seqlens"]
            lens = torch.clamp(cu[1:] - cu[:-1], max=tn)
            idx = torch.cat([torch.arange(int(cu[n]), int(cu[n]) + int(lens[n])) for n in range(w["N"])])
            for k in ("q", "k", "v", "g"):
                d[k] = None if w[k] is None else w[k][:, idx]
            d["cu"] = torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(lens, 0)])
            return d, int(lens.sum())
        for k in ("q", "k", "v", "g"):
            d[k] = None if w[k] is None else w[k][:, :tn]
        d["cu"] = None
        return d, w["B"] * min(tn, w["T"])

    def run(tn):
        d, ntok = sub(tn)
        t0 = time.perf_counter()
        if w.get("entry") in ("recurrent_bwd", "chunk_bwd"):
            oracle.simple_gla_bwd(d["q"], d["k"], d["v"], w["do"][:, :tn], g=d["g"], g_gamma=w["g_gamma"],
                                  scale=w["scale"], initial_state=w["h0"], dht=w["dht"])
        elif w.get("entry") in ("gla", "gla_chunk"):
            oracle.gla_fwd(d["q"], d["k"], d["v"], d["g"], scale=w["scale"], initial_state=w["h0"],
                           output_final_state=w["output_final_state"], threads=threads)
        elif w.get("entry") == "normalized":
            oracle.simple_gla_normalized(d["q"], d["k"], d["v"], g=d["g"], g_gamma=w["g_gamma"],
                                         initial_state=w["h0"], output_final_state=w["output_final_state"],
                                         cu_seqlens=d["cu"], threads=threads)
        else:
            oracle.simple_gla_fwd(d["q"], d["k"], d["v"], g=d["g"], g_gamma=w["g_gamma"], scale=w["scale"],
                                  initial_state=w["h0"], output_final_state=w["output_final_state"],
                                  cu_seqlens=d["cu"], threads=threads)
        return time.perf_counter() - t0, ntok
    cal_t, cal_tok = run(32)
    per_tok = cal_t / max(cal_tok, 1)
    max_t = w["T"] if w["kind"] == "dense" else int((w["cu_seqlens"][1:] - w["cu_seqlens"][:-1]).max())
    full_tokens = w["B"] * w["T"] if w["kind"] == "dense" else w["T"]
    tn = int(min(max_t, max(32, 32 * budget_s / max(cal_t, 1e-6))))
    runs = [run(tn) for _ in range(repeats)]
    dt, ntok = statistics.median(r[0] for r in runs), runs[0][1]
    bwd = w.get("entry") in ("recurrent_bwd", "chunk_bwd")
    what = "fp64 reverse-mode of the naive recurrence" if bwd else "fp64 naive recurrence"
    return dict(value=ntok / dt, unit="tokens/s", cores=1 if bwd else threads,
                kind="oracle", sample=f"first {tn} tokens of every sequence ({ntok} of {full_tokens} tokens), "
                                      f"all heads, {what} (median of {repeats} runs of {dt:.1f} s)")


# ----------------------------------------------------------------------------- main

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_gamma")
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-secondary", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seed", type=int, default=0)
    return ap.parse_args(argv)


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def reference_arm(args, world, rank):
    from gated_linear_attention_local_b200.workloads import make_workload
    if rank != 0:
        return None
    w = make_workload(args.workload, seed=args.seed)
    budget = max(2.0, min(4.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, budget_s=budget / 4, repeats=1)
    vals = [oracle_sample(w, budget_s=budget, repeats=1) for _ in range(args.steps)]
    v = statistics.median(x["value"] for x in vals)
    unit = vals[0]["unit"]
    # the time one whole step of the workload takes at the sampled rate
    counts = algorithmic_counts(w)
    if unit == "GB/s":
        ms = w["steps"] * counts["bytes"] / (v * 1e9) * 1e3
    else:
        ms = counts["tokens"] / v * 1e3
    line = dict(metric=METRIC, value=v, unit=unit, n_gpus=world, steps=args.steps, warmup=args.warmup,
                ms_per_step=ms, ms_per_step_basis="a whole step at the sampled rate", higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64",
                data="synthetic (seeded)", impl="reference",
                config=dict(workload=args.workload, **_config_of(w)),
                cpu_baseline=dict(value=v, unit=unit, cores=vals[0]["cores"], kind="oracle",
                                  sample=vals[0]["sample"]),
                e2e=dict(value=v, unit=unit, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    return line


def _config_of(w):
    if w["kind"] == "decode":
        return dict(N=w["N"], steps_per_call=w["steps"], H=w["H"], K=w["K"], V=w["V"], state="fp32")
    if w.get("entry") == "normalized":
        return dict(entry="simple_gla_normalized", B=w["B"], T=w["T"], H=w["H"], K=w["K"], V=w["V"],
                    gate="g" if w["g"] is not None else "none", feature_map="|x|+0.1", scale=1.0)
    if w.get("entry") == "gla_chunk":
        tc = w["q"].dtype == torch.bfloat16 and w["K"] == 128 and w["V"] % 64 == 0
        return dict(entry="gla_chunk", B=w["B"], T=w["T"], H=w["H"], K=w["K"], V=w["V"], chunk=128 if tc else 32,
                    sub_chunk=16, walk="tcgen05" if tc else "CUDA cores",
                    gate="gk [B,T,H,K] = logsigmoid(N(0,1))/16", initial_state=True)
    if w.get("entry") == "gla":
        return dict(entry="gla_fused_recurrent", B=w["B"], T=w["T"], H=w["H"], K=w["K"], V=w["V"],
                    gate="gk [B,T,H,K] = logsigmoid(N(0,1))/16", initial_state=True)
    if w.get("entry") == "chunk_bwd":
        return dict(entry="simple_gla_chunk_bwd", B=w["B"], T=w["T"], H=w["H"], K=w["K"], V=w["V"],
                    chunk_size=w["chunk_size"], gate="g", initial_state=True, dht=True)
    if w.get("entry") == "recurrent_bwd":
        return dict(entry="simple_gla_fused_recurrent_bwd", B=w["B"], T=w["T"], H=w["H"], K=w["K"], V=w["V"],
                    gate="g" if w["g"] is not None else "none", initial_state=True, dht=True)
    if w.get("entry") == "recurrent":
        return dict(entry="simple_gla_fused_recurrent", B=w["B"], T=w["T"], H=w["H"], K=w["K"], V=w["V"],
                    gate="g" if w["g"] is not None else "none", initial_state=w["h0"] is not None)
    c = dict(H=w["H"], K=w["K"], V=w["V"], chunk_size=w["chunk_size"],
             gate="g" if w["g"] is not None else ("g_gamma" if w["g_gamma"] is not None else "none"))
    if w["kind"] == "varlen":
        c.update(N=w["N"], T_total=w["T"], seqlens=[int(x) for x in (w["cu_seqlens"][1:] - w["cu_seqlens"][:-1])])
    else:
        c.update(B=w["B"], T=w["T"])
    return c


def measure_workload(name, args, device, world, rank, peaks, steps, warmup, flush, want_e2e, want_cpu):
    import gated_linear_attention_local_b200 as sg
    from gated_linear_attention_local_b200.workloads import make_workload
    w = make_workload(name, seed=args.seed + 1000 * rank)
    w["dtype_name"] = "fp32" if w["q"].dtype == torch.float32 else "bf16"
    d = dev_inputs(w, device)
    ws = workspace_for(w, sg, device)
    step, reset = make_step(w, d, sg, ws)
    timing = "eager launches"
    with ClockSampler(device) as clk:
        per_step, prof, launches = time_steps(step, reset, steps, warmup, flush, world > 1)
        if w["kind"] == "decode":
            # the 64 consecutive decode steps of a call are timed as one CUDA graph; the
            # eager pass above supplies the per-kernel times
            from gated_linear_attention_local_b200 import _lib
            graph = torch.cuda.CUDAGraph()
            reset()
            torch.cuda.synchronize()
            n0 = _lib.kernel_launch_count()
            with torch.cuda.graph(graph):
                step()
            per_graph = _lib.kernel_launch_count() - n0
            per_step, _, _ = time_steps(graph.replay, reset, steps, warmup, flush, world > 1, profile=False)
            launches = per_graph * steps
            timing = f"one CUDA graph of {per_graph} decode-step launches per call"
            del graph
    # median step (p10, p90 beside it); multi-GPU: the max over ranks of each
    ms = max_over_ranks(percentile(per_step, 50), world, device)
    ms_p10 = max_over_ranks(percentile(per_step, 10), world, device)
    ms_p90 = max_over_ranks(percentile(per_step, 90), world, device)
    counts = algorithmic_counts(w)
    kname, kn, kms = dominant(prof)
    if w["kind"] == "decode":
        value = world * counts["bytes"] * w["steps"] / (ms * 1e-3) / 1e9
        unit = "GB/s"
    else:
        value = world * counts["tokens"] / (ms * 1e-3)
        unit = "tokens/s"
    kernel_ms = kms / max(kn, 1)
    res = dict(value=value, unit=unit, ms_per_step=ms, ms_p10=ms_p10, ms_p90=ms_p90,
               ms_mean=max_over_ranks(sum(per_step) / len(per_step), world, device),
               tflops=counts["flops"] * (w["steps"] if w["kind"] == "decode" else 1) / (ms * 1e-3) / 1e12,
               gbs=counts["bytes"] * (w["steps"] if w["kind"] == "decode" else 1) / (ms * 1e-3) / 1e9,
               roofline=roofline(w, counts, kernel_ms, peaks, captured_traffic(name, kname), kname) if kname else None,
               dominant_kernel=dict(name=kname, launches=kn, avg_ms=kernel_ms,
                                    share=(kms / sum(v[1] for v in prof.values())) if prof else None),
               kernels={k: dict(launches=v[0], total_ms=round(v[1], 4)) for k, v in prof.items()},
               gpu_launches=launches, clocks=clk.summary(), config=dict(workload=name, timing=timing, **_config_of(w)),
               dtype=w["dtype_name"])
    # whole-call roofline fraction (all kernels, launches included)
    t_roof = max(counts["bytes"] / (peaks["hbm_gbs"] * 1e9), counts["flops"] / (peaks["bf16_tflops"] * 1e12))
    res["call_roofline_frac"] = t_roof * (w["steps"] if w["kind"] == "decode" else 1) / (ms * 1e-3)
    if want_e2e:
        e_ms, h2d, d2h = e2e_measure(w, sg, device, max(3, steps // 5), 2)
        e_ms = max_over_ranks(e_ms, world, device)
        ev = world * (counts["tokens"] / (e_ms * 1e-3) if w["kind"] != "decode"
                      else counts["bytes"] * w["steps"] / (e_ms * 1e-3) / 1e9)
        res["e2e"] = dict(value=ev, unit=unit, h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h, ms_per_step=e_ms)
    if want_cpu and rank == 0 and world == 1:
        res["cpu_baseline"] = oracle_sample(w)
    del d, ws
    return res


# Secondary workloads in the order they are printed: the rows built on the hot path
# first, the hot-path workloads last (a reader of the end of the line sees them).
_SECONDARY_LAST = ("tiny_fp32", "dense_prefill", "varlen_prefill", "long_gamma", "decode")


def secondary_order(headline):
    from gated_linear_attention_local_b200.workloads import WORKLOADS
    first = [n for n in WORKLOADS if n not in _SECONDARY_LAST]
    return [n for n in first + list(_SECONDARY_LAST) if n != headline]


def compact(r):
    """The figures of a secondary workload, without its per-kernel breakdown."""
    rf = r.get("roofline") or {}
    dk = r.get("dominant_kernel") or {}
    rnd = lambda x, n=4: None if x is None else round(x, n)
    return dict(value=float(f"{r['value']:.5g}"), unit=r["unit"], ms=rnd(r["ms_per_step"]),
                p10=rnd(r["ms_p10"]), p90=rnd(r["ms_p90"]), bound=rf.get("bound"), frac=rf.get("frac"),
                call_frac=rnd(r["call_roofline_frac"]), kernel=dk.get("name"), kernel_ms=rnd(dk.get("avg_ms")),
                launches=r["gpu_launches"], reasons=(r.get("clocks") or {}).get("reasons"),
                sm_mhz=(r.get("clocks") or {}).get("sm_mhz"))


def main(argv=None):
    args = parse_args(argv)
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        line = reference_arm(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return 0
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU path)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    peaks = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    main_res = measure_workload(args.workload, args, device, world, rank, peaks, args.steps, args.warmup, flush,
                                want_e2e=True, want_cpu=not args.no_cpu_baseline)
    secondary = {}
    if not args.no_secondary:
        for name in secondary_order(args.workload):
            r = measure_workload(name, args, device, world, rank, peaks, max(5, min(args.steps, 20)),
                                 max(3, args.warmup), flush, want_e2e=False, want_cpu=False)
            secondary[name] = compact(r)
            torch.cuda.empty_cache()
    if rank == 0:
        line = dict(metric=METRIC, value=main_res["value"], unit=main_res["unit"], n_gpus=world,
                    steps=args.steps, warmup=args.warmup, ms_per_step=main_res["ms_per_step"],
                    ms_per_step_stat="median over the timed steps", ms_p10=main_res["ms_p10"],
                    ms_p90=main_res["ms_p90"], ms_mean=main_res["ms_mean"],
                    higher_is_better=True, scaling="weak", vs_baseline=None, dtype=main_res["dtype"],
                    data="synthetic: seeded N(0,1) / logsigmoid(N(0,1)) inputs shaped like the pages' workloads",
                    config=dict(main_res["config"], parallelism=f"dp{world} (independent batches, no collective)",
                                l2="flushed between steps (256 MiB write outside the per-step events)"),
                    roofline=main_res["roofline"], call_roofline_frac=main_res["call_roofline_frac"],
                    cpu_baseline=main_res.get("cpu_baseline"), e2e=main_res["e2e"],
                    gpu_launches=main_res["gpu_launches"], clocks=main_res["clocks"],
                    kernels=main_res["kernels"], dominant_kernel=main_res["dominant_kernel"],
                    tflops=main_res["tflops"], gbs=main_res["gbs"], secondary=secondary)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
