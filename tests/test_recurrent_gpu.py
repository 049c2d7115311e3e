"""GPU parity of the token-serial recurrence (simple_gla_fused_recurrent) and of the
[V,K] state layout (state_v_first), through the C ABI, against the fp64 oracle.

The fused recurrence computes the same operator as the chunked forward (the
article's section 2 lists both entry points; section 5 checks one against the
other), so its oracle is the same naive recurrence; state_v_first stores the state
as [V,K] (section 2), which the oracle wrapper maps by transposition.
"""
import numpy as np
import pytest
import torch

import gated_linear_attention_local_b200 as sg
import oracle
from gated_linear_attention_local_b200.workloads import random_inputs
from parity_utils import TOL, assert_close, host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _vk(x):
    """[N,H,K,V] -> [N,H,V,K] (CPU tensor), the state_v_first layout."""
    return None if x is None else x.transpose(-1, -2).contiguous()


DENSE = [
    # (N, T, H, K, V, dtype, gate, normalizer, h0, state_v_first, scale)
    (2, 64, 3, 128, 128, torch.bfloat16, "g", 1.0, True, False, None),
    (2, 64, 3, 128, 128, torch.bfloat16, "g", 1.0, True, True, None),
    (3, 1, 2, 64, 96, torch.float32, "gamma", 1.0, True, True, 0.1),
    (1, 100, 2, 256, 64, torch.float32, "g", 1.0, False, False, None),
    (2, 17, 4, 512, 40, torch.bfloat16, "none", 1.0, True, True, None),
    (2, 33, 2, 20, 8, torch.float32, "g", 10.0, True, False, 1.0),
    (1, 64, 2, 64, 64, torch.float32, "g", 0.1, True, True, None),
    (2, 0, 2, 64, 64, torch.float32, "g", 1.0, True, True, None),
    # gate 0 and log gates of both signs: the blocks whose cumulative decay leaves the
    # range where it can be factored out take the exact per-token update
    (2, 40, 2, 64, 64, torch.float32, "neg_inf", 1.0, True, False, None),
    (2, 40, 2, 64, 64, torch.float32, "mixed", 1.0, True, False, None),
    (2, 40, 2, 64, 64, torch.float32, "g", 0.05, True, False, None),
]


@pytest.mark.parametrize("case", DENSE, ids=[f"N{c[0]}T{c[1]}H{c[2]}K{c[3]}V{c[4]}-{str(c[5])[6:]}-{c[6]}"
                                              f"-h0{int(c[8])}-vf{int(c[9])}" for c in DENSE])
def test_fused_recurrent_dense(case):
    N, T, H, K, V, dt, gate, norm, h0, vf, scale = case
    inp = random_inputs(N, T, H, K, V, dtype=dt, gate=gate, normalizer=norm, h0=h0, seed=17)
    s0 = _vk(inp["h0"]) if vf else inp["h0"]
    o, ht = sg.simple_gla_fused_recurrent(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), g=to_dev(inp["g"]),
                                          g_gamma=to_dev(inp["g_gamma"]), scale=scale, initial_state=to_dev(s0),
                                          output_final_state=True, state_v_first=vf)
    torch.cuda.synchronize()
    ro, rh = oracle.simple_gla_fwd(inp["q"], inp["k"], inp["v"], g=inp["g"], g_gamma=inp["g_gamma"], scale=scale,
                                   initial_state=s0, output_final_state=True, state_v_first=vf)
    assert tuple(ht.shape) == ((N, H, V, K) if vf else (N, H, K, V))
    assert_close(host(o), ro, TOL[dt], "o")
    assert_close(host(ht), rh, TOL[dt], "final_state")


@pytest.mark.parametrize("vf", [False, True])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_fused_recurrent_varlen(vf, dt):
    # the non-aligned packed lengths of the article's section 5 test matrix, plus an
    # empty sequence
    cu = torch.tensor([0, 15, 15, 100, 300, 1200, 2000], dtype=torch.int64)
    T, H, K, V = 2000, 2, 64, 64
    inp = random_inputs(1, T, H, K, V, dtype=dt, gate="g", h0=True, seed=5, cu_seqlens=cu)
    s0 = _vk(inp["h0"]) if vf else inp["h0"]
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    o, ht = sg.simple_gla_fused_recurrent(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), g=to_dev(inp["g"]),
                                          initial_state=to_dev(s0), output_final_state=True, cu_seqlens=to_dev(cu),
                                          state_v_first=vf, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ro, rh = oracle.simple_gla_fwd(inp["q"], inp["k"], inp["v"], g=inp["g"], initial_state=s0,
                                   output_final_state=True, cu_seqlens=cu, state_v_first=vf)
    assert_close(host(o), ro, TOL[dt], "o")
    assert_close(host(ht), rh, TOL[dt], "final_state")


def test_fused_recurrent_matches_chunked_forward():
    """Both entry points compute one operator (section 5 checks chunk against
    fused_recurrent): on the same inputs they agree within the bf16 bound."""
    inp = random_inputs(2, 64, 4, 128, 128, dtype=torch.bfloat16, gate="g", h0=True, seed=9)
    d = {k: to_dev(v) for k, v in inp.items()}
    o1, h1 = sg.simple_gla_fused_recurrent(d["q"], d["k"], d["v"], g=d["g"], initial_state=d["h0"],
                                           output_final_state=True)
    o2, h2 = sg.simple_gla_fwd(d["q"], d["k"], d["v"], g=d["g"], initial_state=d["h0"], output_final_state=True)
    torch.cuda.synchronize()
    assert_close(host(o1), host(o2), TOL[torch.bfloat16], "o")
    assert_close(host(h1), host(h2), TOL[torch.bfloat16], "final_state")


def test_bad_cu_seqlens_skips_only_the_bad_sequence():
    cu = torch.tensor([0, 50, 30, 80], dtype=torch.int64)  # sequence 1 runs backwards
    T, H, K, V = 80, 2, 64, 64
    inp = random_inputs(1, T, H, K, V, dtype=torch.float32, gate="g", seed=3)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sentinel = 12345.0
    ht = torch.full((3, H, K, V), sentinel, dtype=torch.float32, device="cuda")
    o = torch.full((T, H, V), sentinel, dtype=torch.float32, device="cuda")
    from gated_linear_attention_local_b200 import _lib
    import ctypes
    dq, dk, dv, dg, dcu = (to_dev(x) for x in (inp["q"][0], inp["k"][0], inp["v"][0], inp["g"][0], cu))
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = _lib.lib().simple_gla_fused_recurrent(
        P(dq), P(dk), P(dv), P(dg), None, ctypes.c_float(float("nan")), None, P(o), P(ht), P(dcu),
        3, T, H, K, V, 0, _lib.SGLA_FP32, P(status), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert st == _lib.SGLA_OK
    assert int(status.item()) == 1  # SGLA_DEVICE_BAD_CU_SEQLENS
    assert torch.all(ht[1] == sentinel)  # the skipped sequence wrote nothing
    for n, (a, b) in enumerate([(0, 50), (30, 80)]):
        sub = {k: inp[k][:, a:b] for k in ("q", "k", "v", "g")}
        ro, rh = oracle.simple_gla_fwd(sub["q"], sub["k"], sub["v"], g=sub["g"], output_final_state=True)
        assert_close(host(ht[2 * n]), rh[0], TOL[torch.float32], f"final_state {n}")
    # rows 30..49 belong to both valid sequences; rows 0..29 only to sequence 0
    ro, _ = oracle.simple_gla_fwd(inp["q"][:, :50], inp["k"][:, :50], inp["v"][:, :50], g=inp["g"][:, :50])
    assert_close(host(o[:30]), ro[0, :30], TOL[torch.float32], "o of sequence 0")


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_decode_step_state_v_first(dt):
    """A decode step on a [V,K] state (a one-token fused recurrence, in place) against
    the oracle's decode step on the transposed state, over several steps."""
    N, H, K, V, steps = 8, 4, 128, 64, 3
    gen = torch.Generator().manual_seed(21)
    state = torch.randn(N, H, K, V, generator=gen) * 0.1
    ref_state = state.double().numpy().copy()
    dev_state = _vk(state).cuda()
    for s in range(steps):
        q = torch.randn(N, H, K, generator=gen).to(dt)
        k = torch.randn(N, H, K, generator=gen).to(dt)
        v = torch.randn(N, H, V, generator=gen).to(dt)
        g = torch.nn.functional.logsigmoid(torch.randn(N, H, generator=gen))
        o = sg.simple_gla_decode_step(q.cuda(), k.cuda(), v.cuda(), dev_state, g=g.cuda(), state_v_first=True)
        ro = oracle.simple_gla_decode_step(q, k, v, ref_state, g=g)
        torch.cuda.synchronize()
        assert_close(host(o), ro, TOL[dt], f"o step {s}")
    assert_close(host(dev_state).transpose(0, 1, 3, 2), ref_state, TOL[dt], "state")


def test_fused_recurrent_inference_shape():
    """The routing case of section 4 (inference, at most 64 tokens) at the decode
    workload's size: 256 sequences x 64 tokens, H=32, K=V=128, bf16; sampled heads."""
    N, T, H, K, V = 256, 64, 32, 128, 128
    inp = random_inputs(N, T, H, K, V, dtype=torch.bfloat16, gate="g", h0=True, seed=2)
    o, ht = sg.simple_gla_fused_recurrent(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), g=to_dev(inp["g"]),
                                          initial_state=to_dev(inp["h0"]), output_final_state=True)
    torch.cuda.synchronize()
    o, ht = host(o), host(ht)
    for n in (0, 97, 255):
        sub = {k: (inp[k][n:n + 1] if inp[k] is not None else None) for k in ("q", "k", "v", "g", "h0")}
        ro, rh = oracle.simple_gla_fwd(sub["q"], sub["k"], sub["v"], g=sub["g"], initial_state=sub["h0"],
                                       output_final_state=True)
        assert_close(o[n:n + 1], ro, TOL[torch.bfloat16], f"o seq {n}")
        assert_close(ht[n:n + 1], rh, TOL[torch.bfloat16], f"final_state seq {n}")


CHUNK_VF = [
    # (B, T, H, K, V, dtype, gate, h0, chunk) -- tensor-core and SIMT paths, empty
    (2, 300, 2, 128, 128, torch.bfloat16, "g", True, 64),
    (1, 520, 2, 256, 64, torch.bfloat16, "gamma", True, 64),
    (2, 150, 3, 64, 32, torch.float32, "g", True, 32),
    (2, 0, 2, 64, 64, torch.float32, "g", True, 64),
]


@pytest.mark.parametrize("case", CHUNK_VF, ids=[f"B{c[0]}T{c[1]}K{c[3]}V{c[4]}-{str(c[5])[6:]}-C{c[8]}"
                                                 for c in CHUNK_VF])
def test_chunk_state_v_first_dense(case):
    B, T, H, K, V, dt, gate, h0, chunk = case
    inp = random_inputs(B, T, H, K, V, dtype=dt, gate=gate, h0=h0, seed=41)
    s0 = _vk(inp["h0"])
    o, ht = sg.chunk_simple_gla(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), g=to_dev(inp["g"]),
                                g_gamma=to_dev(inp["g_gamma"]), initial_state=to_dev(s0), output_final_state=True,
                                chunk_size=chunk, state_v_first=True)
    torch.cuda.synchronize()
    ro, rh = oracle.simple_gla_fwd(inp["q"], inp["k"], inp["v"], g=inp["g"], g_gamma=inp["g_gamma"],
                                   initial_state=s0, output_final_state=True, state_v_first=True)
    assert tuple(ht.shape) == (B, H, V, K)
    assert_close(host(o), ro, TOL[dt], "o")
    assert_close(host(ht), rh, TOL[dt], "final_state")


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_chunk_state_v_first_varlen(dt):
    cu = torch.tensor([0, 15, 15, 100, 300, 1200, 2000], dtype=torch.int64)
    T, H, K, V = 2000, 2, 128, 128
    inp = random_inputs(1, T, H, K, V, dtype=dt, gate="g", h0=True, seed=43, cu_seqlens=cu)
    s0 = _vk(inp["h0"])
    o, ht = sg.chunk_simple_gla(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), g=to_dev(inp["g"]),
                                initial_state=to_dev(s0), output_final_state=True, cu_seqlens=to_dev(cu),
                                state_v_first=True)
    torch.cuda.synchronize()
    ro, rh = oracle.simple_gla_fwd(inp["q"], inp["k"], inp["v"], g=inp["g"], initial_state=s0,
                                   output_final_state=True, cu_seqlens=cu, state_v_first=True)
    assert_close(host(o), ro, TOL[dt], "o")
    assert_close(host(ht), rh, TOL[dt], "final_state")


def test_bounded_wait_gives_up_and_the_context_survives():
    """Failure detection without a GPU fault: a CTA waits on an mbarrier phase that
    nothing completes; the bounded wait gives up after its 2 s limit, raises the CTA's
    abort flag (the second waiter gives up through it) and reports the time-out in a
    status word the host reads.  The context then runs a forward normally."""
    import ctypes
    import time
    from gated_linear_attention_local_b200 import _lib
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    st = _lib.lib().sgla_selftest_wait_timeout(ctypes.c_void_p(status.data_ptr()),
                                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert st == _lib.SGLA_OK
    assert int(status.item()) == 2  # SGLA_DEVICE_TIMEOUT
    assert 1.5 < dt < 30.0, dt
    inp = random_inputs(1, 256, 2, 128, 128, dtype=torch.bfloat16, gate="g", seed=1)
    o, _ = sg.simple_gla_fwd(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), g=to_dev(inp["g"]))
    torch.cuda.synchronize()
    ro, _ = oracle.simple_gla_fwd(inp["q"], inp["k"], inp["v"], g=inp["g"])
    assert_close(host(o), ro, TOL[torch.bfloat16], "o after the time-out")
