"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, element by element.

Small cases span several chunks and segments plus ragged tails and the edge cases
of the method (empty and one-token sequences, gate 0 and gate 1, chunk sizes
16..128, scales and gate normalisers of the article's test matrix, section 5).
Full-size workloads run in the same launch configuration the bench times and are
checked on sampled heads / sequences the oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import gated_linear_attention_local_b200 as sg
from gated_linear_attention_local_b200.workloads import make_workload, random_inputs
from parity_utils import TOL, assert_close, host, oracle_fwd, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def run_dense(inp, scale=None, final=True, chunk=64):
    o, ht = sg.simple_gla_fwd(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), g=to_dev(inp["g"]),
                              g_gamma=to_dev(inp["g_gamma"]), scale=scale, initial_state=to_dev(inp["h0"]),
                              output_final_state=final, chunk_size=chunk)
    torch.cuda.synchronize()
    return host(o), host(ht)


def run_varlen(inp, cu, scale=None, final=True, chunk=64):
    o, ht = sg.simple_gla_fwd_varlen(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), to_dev(cu),
                                     g=to_dev(inp["g"]), g_gamma=to_dev(inp["g_gamma"]), scale=scale,
                                     initial_state=to_dev(inp["h0"]), output_final_state=final,
                                     chunk_size=chunk)
    torch.cuda.synchronize()
    return host(o), host(ht)


def check(inp, gpu, ref, dtype, what):
    tol = TOL[dtype]
    assert_close(gpu[0], ref[0], tol, what + " o")
    if ref[1] is not None:
        assert_close(gpu[1], ref[1], tol, what + " final_state")


# ----------------------------------------------------------------------------- small dense

DENSE_CASES = [
    # (B, T, H, K, V, dtype, gate, normalizer, h0, chunk, scale)
    (1, 256, 2, 64, 64, torch.float32, "g", 1.0, False, 64, 0.125),
    (2, 300, 3, 64, 64, torch.float32, "g", 1.0, True, 64, None),
    (1, 1, 2, 64, 32, torch.float32, "g", 1.0, True, 64, None),
    (1, 17, 1, 32, 64, torch.float32, "gamma", 1.0, True, 16, 1.0),
    (2, 100, 2, 128, 128, torch.bfloat16, "g", 1.0, True, 64, None),
    (1, 513, 2, 128, 128, torch.bfloat16, "g", 0.1, True, 64, 0.1),
    (1, 200, 2, 128, 128, torch.bfloat16, "g", 10.0, False, 64, 1.0),
    (1, 333, 4, 64, 128, torch.bfloat16, "gamma", 1.0, True, 64, None),
    (1, 130, 2, 128, 64, torch.bfloat16, "none", 1.0, True, 64, None),
    (1, 90, 2, 64, 64, torch.bfloat16, "zero", 1.0, False, 32, None),
    (1, 77, 2, 64, 64, torch.float32, "neg_inf", 1.0, True, 64, 1.0),
    (1, 250, 2, 40, 24, torch.float32, "g", 1.0, True, 128, None),
    (2, 129, 2, 256, 256, torch.bfloat16, "g", 1.0, True, 64, None),
    (1, 200, 1, 512, 512, torch.bfloat16, "g", 1.0, True, 64, None),
]


@pytest.mark.parametrize("case", DENSE_CASES, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}K{c[3]}V{c[4]}-"
                         f"{str(c[5])[6:]}-{c[6]}{c[7]}-h0{int(c[8])}-C{c[9]}-s{c[10]}")
def test_dense_small(case):
    B, T, H, K, V, dt, gate, norm, h0, chunk, scale = case
    inp = random_inputs(B, T, H, K, V, dt, gate=gate, normalizer=norm, h0=h0, seed=11)
    check(inp, run_dense(inp, scale, True, chunk), oracle_fwd(inp, scale), dt, "dense")


@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_chunk_size_only_changes_rounding(chunk, dt):
    inp = random_inputs(1, 301, 2, 64, 64, dt, gate="g", h0=True, seed=5)
    check(inp, run_dense(inp, None, True, chunk), oracle_fwd(inp), dt, f"chunk {chunk}")


def test_empty_sequence_dense_returns_initial_state():
    inp = random_inputs(2, 0, 2, 64, 64, torch.bfloat16, gate="g", h0=True, seed=3)
    o, ht = run_dense(inp)
    assert o.shape == (2, 0, 2, 64)
    np.testing.assert_array_equal(ht, inp["h0"].numpy())


# ----------------------------------------------------------------------------- varlen

VARLEN_CASES = [
    ([0, 15, 100, 300, 1200, 2000], torch.bfloat16, "g", True, 64),
    ([0, 15, 100, 300, 1200, 2000], torch.float32, "g", True, 32),
    ([0, 0, 5, 5, 70, 200, 201], torch.bfloat16, "g", True, 64),
    ([0, 64, 128, 129], torch.bfloat16, "gamma", True, 64),
    ([0, 1000], torch.float32, "none", False, 16),
]


@pytest.mark.parametrize("case", VARLEN_CASES, ids=lambda c: f"n{len(c[0]) - 1}-{str(c[1])[6:]}-{c[2]}-C{c[4]}")
def test_varlen(case):
    cu_list, dt, gate, h0, chunk = case
    cu = torch.tensor(cu_list, dtype=torch.int64)
    inp = random_inputs(1, cu_list[-1], 3, 64, 128, dt, gate=gate, h0=h0, seed=7, cu_seqlens=cu)
    check(inp, run_varlen(inp, cu, None, True, chunk), oracle_fwd(inp, cu=cu), dt, "varlen")


def test_varlen_equals_separate_calls():
    cu = torch.tensor([0, 40, 300, 301, 700], dtype=torch.int64)
    inp = random_inputs(1, 700, 2, 64, 64, torch.bfloat16, gate="g", h0=True, seed=9, cu_seqlens=cu)
    o, ht = run_varlen(inp, cu)
    for n in range(4):
        a, b = int(cu[n]), int(cu[n + 1])
        part = dict(q=inp["q"][:, a:b], k=inp["k"][:, a:b], v=inp["v"][:, a:b], g=inp["g"][:, a:b],
                    g_gamma=None, h0=inp["h0"][n:n + 1].contiguous())
        on, hn = run_dense({k_: (v_.contiguous() if v_ is not None else None) for k_, v_ in part.items()})
        assert_close(o[:, a:b], on, 1e-5, f"seq {n} o")
        assert_close(ht[n:n + 1], hn, 1e-5, f"seq {n} state")


def test_bad_cu_seqlens_is_reported_on_the_device():
    cu = torch.tensor([0, 50, 40, 100], dtype=torch.int64)  # decreasing
    inp = random_inputs(1, 100, 2, 64, 64, torch.bfloat16, gate="g", seed=1)
    q, k, v, g = (to_dev(inp[x]) for x in ("q", "k", "v", "g"))
    nbytes = sg.varlen_workspace_size(3, 100, 2, 64, 64)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    o, _ = sg.simple_gla_fwd_varlen(q, k, v, cu.cuda(), g=g, workspace=ws)
    assert sg.workspace_status(ws) == 1
    # a good call on the same workspace clears the status
    good = torch.tensor([0, 50, 60, 100], dtype=torch.int64, device="cuda")
    sg.simple_gla_fwd_varlen(q, k, v, good, g=g, workspace=ws)
    assert sg.workspace_status(ws) == 0


def test_initial_state_count_must_match():
    cu = torch.tensor([0, 10, 20], dtype=torch.int64, device="cuda")
    x = torch.zeros(1, 20, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        sg.simple_gla_fwd_varlen(x, x, x, cu, initial_state=torch.zeros(3, 2, 64, 64, device="cuda"))
    with pytest.raises(ValueError):
        sg.simple_gla_fwd_varlen(torch.zeros(2, 10, 2, 64, dtype=torch.bfloat16, device="cuda"),
                                 x[:, :10].expand(2, -1, -1, -1).contiguous(),
                                 x[:, :10].expand(2, -1, -1, -1).contiguous(), cu)


def test_split_and_carry_matches_one_call():
    inp = random_inputs(1, 400, 2, 128, 128, torch.bfloat16, gate="g", h0=True, seed=13)
    o, ht = run_dense(inp)
    t1 = 150
    first = {k_: (v_[:, :t1].contiguous() if k_ in ("q", "k", "v", "g") else v_) for k_, v_ in inp.items()}
    o1, h1 = run_dense(first)
    second = {k_: (v_[:, t1:].contiguous() if k_ in ("q", "k", "v", "g") else v_) for k_, v_ in inp.items()}
    second["h0"] = torch.from_numpy(h1)
    o2, h2 = run_dense(second)
    assert_close(np.concatenate([o1, o2], axis=1), o, 2e-2, "split o")
    assert_close(h2, ht, 2e-2, "split state")


# ----------------------------------------------------------------------------- decode

@pytest.mark.parametrize("dt,gate", [(torch.bfloat16, "g"), (torch.float32, "g"), (torch.bfloat16, "gamma"),
                                     (torch.float32, "none")])
def test_decode_steps_match_oracle(dt, gate):
    import oracle
    N, H, K, V, steps = 5, 3, 64, 128, 20
    inp = random_inputs(N, steps, H, K, V, dt, gate=gate, h0=True, seed=21)
    state = to_dev(inp["h0"]).clone()
    ref_state = inp["h0"].double().numpy().copy()
    for t in range(steps):
        q, k, v = (to_dev(inp[x][:, t].contiguous()) for x in ("q", "k", "v"))
        g = to_dev(inp["g"][:, t].contiguous()) if inp["g"] is not None else None
        o = sg.simple_gla_decode_step(q, k, v, state, g=g, g_gamma=to_dev(inp["g_gamma"]))
        ro = oracle.simple_gla_decode_step(inp["q"][:, t], inp["k"][:, t], inp["v"][:, t], ref_state,
                                           g=None if inp["g"] is None else inp["g"][:, t],
                                           g_gamma=inp["g_gamma"])
        assert_close(host(o), ro, TOL[dt], f"step {t} o")
    assert_close(host(state), ref_state, TOL[dt], "state")


def test_decode_equals_forward_on_gpu():
    inp = random_inputs(3, 64, 2, 128, 128, torch.bfloat16, gate="g", h0=True, seed=4)
    o_fwd, ht = run_dense(inp)
    state = to_dev(inp["h0"]).clone()
    for t in range(64):
        o = sg.simple_gla_decode_step(*(to_dev(inp[x][:, t].contiguous()) for x in ("q", "k", "v")), state,
                                      g=to_dev(inp["g"][:, t].contiguous()))
        assert_close(host(o), o_fwd[:, t], 2e-2, f"step {t}")
    assert_close(host(state), ht, 2e-2, "state")


# ----------------------------------------------------------------------------- full-size workloads

def _heads(inp, hs):
    out = {}
    for key in ("q", "k", "v", "g"):
        out[key] = None if inp[key] is None else inp[key][:, :, hs].contiguous()
    out["g_gamma"] = None if inp["g_gamma"] is None else inp["g_gamma"][hs].contiguous()
    out["h0"] = None if inp["h0"] is None else inp["h0"][:, hs].contiguous()
    return out


def _full_size(name, heads, batches=None):
    w = make_workload(name)
    if w["kind"] == "varlen":
        o, ht = run_varlen(w, w["cu_seqlens"], w["scale"], w["output_final_state"], w["chunk_size"])
    else:
        o, ht = run_dense(w, w["scale"], w["output_final_state"], w["chunk_size"])
    sub = _heads(w, heads)
    if batches is not None:
        sub = {k_: (None if v_ is None else (v_[batches].contiguous() if k_ != "g_gamma" else v_))
               for k_, v_ in sub.items()}
        o, ht = o[batches], (None if ht is None else ht[batches])
    ro, rht = oracle_fwd(sub, w["scale"], w["output_final_state"], w["cu_seqlens"])
    assert_close(o[:, :, heads], ro, 2e-2, f"{name} o")
    if w["output_final_state"]:
        assert_close(ht[:, heads], rht, 2e-2, f"{name} final_state")


def test_workload_tiny_fp32_full():
    w = make_workload("tiny_fp32")
    o, ht = run_dense(w, w["scale"], True, 64)
    ro, rht = oracle_fwd(w, w["scale"])
    assert_close(o, ro, 1e-4, "o")
    assert_close(ht, rht, 1e-4, "final_state")


def test_workload_dense_prefill_sampled():
    _full_size("dense_prefill", heads=[0, 3], batches=[0, 3])


def test_workload_varlen_prefill_sampled():
    _full_size("varlen_prefill", heads=[0, 15])


def test_workload_long_gamma_sampled():
    _full_size("long_gamma", heads=[0, 31])


def test_workload_decode_sampled():
    import oracle
    w = make_workload("decode")
    state = w["state"].cuda()
    sel_n, sel_h = [0, 77, 255], [0, 31]
    ref_state = w["state"][sel_n][:, sel_h].double().numpy().copy()
    for t in range(w["steps"]):
        o = sg.simple_gla_decode_step(w["q"][t].cuda(), w["k"][t].cuda(), w["v"][t].cuda(), state,
                                      g=w["g"][t].cuda())
        sub = lambda x: x[t][sel_n][:, sel_h]
        ro = oracle.simple_gla_decode_step(sub(w["q"]), sub(w["k"]), sub(w["v"]), ref_state, g=sub(w["g"]))
        assert_close(host(o)[sel_n][:, sel_h], ro, 2e-2, f"step {t}")
    assert_close(host(state)[sel_n][:, sel_h], ref_state, 2e-2, "state")


# ----------------------------------------------------------------------------- tensor-core path

TC_CASES = [
    # (B, T, H, V, gate, h0, chunk)   K = 128, bf16
    (1, 1, 1, 64, "g", True, 64),
    (1, 127, 2, 128, "g", True, 64),
    (1, 128, 2, 128, "gamma", False, 128),
    (2, 129, 2, 192, "g", True, 64),
    (1, 300, 3, 512, "g", True, 64),
    (1, 5000, 1, 64, "g", True, 64),        # many segments: state pass + carry
    (1, 5000, 1, 128, "gamma", True, 128),
    (2, 1000, 2, 128, "none", True, 64),
    (1, 700, 2, 64, "zero", False, 64),
    (1, 1030, 2, 128, "neg_inf", True, 64),
    (1, 900, 2, 128, "mixed", True, 64),    # positive log gates: exact-decay fallback
    (1, 256, 2, 128, "mixed", False, 128),  # positive log gates over a span short enough that
                                            # the intra-chunk terms dominate the error measure
]


def _ran(kernel_prefix, fn):
    from gated_linear_attention_local_b200 import _lib
    _lib.profile_begin()
    out = fn()
    torch.cuda.synchronize()
    prof = _lib.profile_end()
    assert any(k.startswith(kernel_prefix) for k in prof), f"{kernel_prefix} did not run: {sorted(prof)}"
    return out


@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}V{c[3]}-{c[4]}-h0{int(c[5])}-C{c[6]}")
def test_tensor_core_dense(case):
    B, T, H, V, gate, h0, chunk = case
    inp = random_inputs(B, T, H, 128, V, torch.bfloat16, gate=gate, h0=h0, seed=31)
    gpu = _ran("chunk_output_tc", lambda: run_dense(inp, None, True, chunk))
    check(inp, gpu, oracle_fwd(inp), torch.bfloat16, "tc dense")


@pytest.mark.parametrize("cu_list", [[0, 15, 100, 300, 1200, 2000], [0, 0, 129, 129, 2500, 2501, 6000]])
def test_tensor_core_varlen(cu_list):
    cu = torch.tensor(cu_list, dtype=torch.int64)
    inp = random_inputs(1, cu_list[-1], 4, 128, 128, torch.bfloat16, gate="g", h0=True, seed=41, cu_seqlens=cu)
    gpu = _ran("chunk_output_tc", lambda: run_varlen(inp, cu))
    check(inp, gpu, oracle_fwd(inp, cu=cu), torch.bfloat16, "tc varlen")


def test_tensor_core_workspace_status_clean():
    inp = random_inputs(1, 3000, 2, 128, 128, torch.bfloat16, gate="g", h0=True, seed=2)
    d = {k_: (v_.cuda() if v_ is not None else None) for k_, v_ in inp.items()}
    ws = torch.empty(sg.fwd_workspace_size(1, 3000, 2, 128, 128), dtype=torch.uint8, device="cuda")
    sg.simple_gla_fwd(d["q"], d["k"], d["v"], g=d["g"], initial_state=d["h0"], output_final_state=True,
                      workspace=ws)
    assert sg.workspace_status(ws) == 0


WIDE_K_CASES = [
    # (B, T, H, K, V, gate, h0)   bf16, tensor-core path with K > 128 (V tile 64)
    (2, 129, 2, 256, 256, "g", True),
    (1, 300, 1, 512, 512, "g", True),
    (1, 3000, 1, 512, 64, "g", True),     # many segments: k-block state pass + carry
    (1, 2500, 2, 256, 128, "gamma", True),
    (2, 700, 1, 512, 128, "mixed", False),
    (1, 256, 2, 256, 64, "mixed", False),
    (1, 200, 1, 512, 64, "mixed", False),
]


@pytest.mark.parametrize("case", WIDE_K_CASES, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}K{c[3]}V{c[4]}-{c[5]}-h0{int(c[6])}")
def test_tensor_core_wide_k(case):
    B, T, H, K, V, gate, h0 = case
    inp = random_inputs(B, T, H, K, V, torch.bfloat16, gate=gate, h0=h0, seed=51)
    gpu = _ran("chunk_output_tc", lambda: run_dense(inp))
    check(inp, gpu, oracle_fwd(inp), torch.bfloat16, "tc wide-k")


def test_tensor_core_wide_k_varlen():
    cu = torch.tensor([0, 100, 1600, 1601, 2900], dtype=torch.int64)
    inp = random_inputs(1, 2900, 2, 512, 128, torch.bfloat16, gate="g", h0=True, seed=52, cu_seqlens=cu)
    gpu = _ran("chunk_output_tc", lambda: run_varlen(inp, cu))
    check(inp, gpu, oracle_fwd(inp, cu=cu), torch.bfloat16, "tc wide-k varlen")


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs a second CUDA device")
def test_call_runs_on_the_device_of_its_tensors():
    inp = random_inputs(2, 300, 2, 128, 128, torch.bfloat16, gate="g", h0=True, seed=53)
    dev = torch.device("cuda", 1)
    d = {k_: (v_.to(dev) if v_ is not None else None) for k_, v_ in inp.items()}
    with torch.cuda.device(0):
        o, ht = sg.chunk_simple_gla(d["q"], d["k"], d["v"], g=d["g"], initial_state=d["h0"],
                                    output_final_state=True)
        assert o.device == dev and ht.device == dev
        torch.cuda.synchronize(dev)
    check(inp, (host(o), host(ht)), oracle_fwd(inp), torch.bfloat16, "second device")


@pytest.mark.parametrize("vf", [False, True])
def test_tensor_core_varlen_empty_sequences_both_state_layouts(vf):
    """Packed batch with empty sequences (their final state is their initial state) and
    long ones split into segments, through the chunked entry point in either state
    layout: the plan pass writes the empty sequences' final states in the [K,V] layout,
    the carry pass in the [V,K] one."""
    cu_list = [0, 0, 3000, 3000, 3001, 7200, 7200]
    cu = torch.tensor(cu_list, dtype=torch.int64)
    inp = random_inputs(1, cu_list[-1], 2, 128, 128, torch.bfloat16, gate="g", h0=True, seed=43, cu_seqlens=cu)
    h0 = inp["h0"].transpose(-1, -2).contiguous() if vf else inp["h0"]
    o, ht = sg.chunk_simple_gla(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), g=to_dev(inp["g"]),
                                initial_state=to_dev(h0), output_final_state=True, cu_seqlens=to_dev(cu),
                                state_v_first=vf)
    torch.cuda.synchronize()
    ht = host(ht)
    if vf:
        ht = np.swapaxes(ht, -1, -2)
    ro, rh = oracle_fwd(inp, cu=cu)
    check(inp, (host(o), ht), (ro, rh), torch.bfloat16, f"varlen empty sequences vf={vf}")
    for n in range(len(cu_list) - 1):
        if cu_list[n + 1] == cu_list[n]:
            np.testing.assert_array_equal(ht[n], inp["h0"][n].numpy())


# On packed batches the output walk starts while the segment-state pass that precedes
# it still runs: the CTAs of first segments begin at once, the others wait for that pass
# before they fold the earlier segments' states.  Sizes give long sequences many
# segments and short ones a single segment each.
OVERLAP_CASES = [
    ("varlen", 128, 128, "g"),
    ("varlen", 128, 128, "gamma"),
    ("varlen", 512, 128, "g"),
    ("dense", 128, 128, "gamma"),  # launched the ordinary way
]


@pytest.mark.parametrize("case", OVERLAP_CASES)
def test_walk_started_under_the_state_pass_is_repeatable(case):
    kind, K, V, gate = case
    if kind == "varlen":
        T = 12000 if K == 128 else 4000
        cu = torch.tensor([0, 3 * T // 4, 3 * T // 4 + 100, 3 * T // 4 + 101, T], dtype=torch.int64)
        inp = random_inputs(1, T, 2, K, V, torch.bfloat16, gate=gate, h0=True, seed=61, cu_seqlens=cu)
        call = lambda d: sg.simple_gla_fwd_varlen(d["q"], d["k"], d["v"], d["cu"], g=d["g"], g_gamma=d["g_gamma"],
                                                  initial_state=d["h0"], output_final_state=True)
        ref = oracle_fwd(inp, cu=cu)
    else:
        cu = None
        T = 12000 if K == 128 else 3000
        inp = random_inputs(1, T, 2 if K == 128 else 1, K, V, torch.bfloat16, gate=gate, h0=True, seed=62)
        call = lambda d: sg.simple_gla_fwd(d["q"], d["k"], d["v"], g=d["g"], g_gamma=d["g_gamma"],
                                           initial_state=d["h0"], output_final_state=True)
        ref = oracle_fwd(inp)
    d = {k_: to_dev(inp[k_]) for k_ in ("q", "k", "v", "g", "g_gamma", "h0")}
    d["cu"] = to_dev(cu)
    runs = []
    for _ in range(4):
        o, ht = call(d)
        runs.append((o.clone(), ht.clone()))
    torch.cuda.synchronize()
    for o, ht in runs[1:]:
        assert torch.equal(o, runs[0][0]) and torch.equal(ht, runs[0][1]), "calls differ"
    check(inp, (host(runs[0][0]), host(runs[0][1])), ref, torch.bfloat16, "walk under the state pass")
