"""GPU parity of GLA with a gate vector over the key dimension (gla_fused_recurrent,
the token-serial form) against the fp64 oracle of the same recurrence; the scalar
head-wise gate of Simple GLA is its special case ("relinear", fla-org kernel
integration, gate-shape item)."""
import pytest
import torch
import torch.nn.functional as F

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


def _gk(shape, seed, normalizer=16.0):
    """GLA-style log gates: logsigmoid(N(0,1)) / 16 per key (the gate logit normaliser
    of the article's layer, section 4)."""
    gen = torch.Generator().manual_seed(seed)
    return F.logsigmoid(torch.randn(*shape, generator=gen)) / normalizer


CASES = [
    # (B, T, H, K, V, dtype, h0, vf, normalizer)
    (2, 64, 3, 128, 128, torch.bfloat16, True, False, 16.0),
    (2, 100, 2, 64, 64, torch.float32, True, True, 1.0),
    (1, 33, 2, 256, 40, torch.bfloat16, False, False, 16.0),
    (3, 1, 2, 64, 96, torch.float32, True, False, 0.1),
]


@pytest.mark.parametrize("case", CASES, ids=[f"K{c[3]}V{c[4]}-{str(c[5])[6:]}-h0{int(c[6])}-vf{int(c[7])}" for c in CASES])
def test_gla_fused_recurrent_dense(case):
    B, T, H, K, V, dt, h0, vf, norm = case
    inp = random_inputs(B, T, H, K, V, dtype=dt, gate="none", h0=h0, seed=81)
    gk = _gk((B, T, H, K), 82, norm)
    s0 = inp["h0"]
    s0_dev = None if s0 is None else (s0.transpose(-1, -2).contiguous() if vf else s0)
    o, ht = sg.gla_fused_recurrent(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), gk.cuda(),
                                   initial_state=to_dev(s0_dev), output_final_state=True, state_v_first=vf)
    torch.cuda.synchronize()
    ro, rh = oracle.gla_fwd(inp["q"], inp["k"], inp["v"], gk, initial_state=s0, output_final_state=True)
    gh = host(ht)
    if vf:
        gh = gh.transpose(0, 1, 3, 2)
    assert_close(host(o), ro, TOL[dt], "o")
    assert_close(gh, rh, TOL[dt], "final_state")


def test_gla_fused_recurrent_varlen():
    cu = torch.tensor([0, 15, 15, 100, 300, 1200], dtype=torch.int64)
    T, H, K, V = 1200, 2, 64, 64
    inp = random_inputs(1, T, H, K, V, dtype=torch.bfloat16, gate="none", h0=True, seed=83, cu_seqlens=cu)
    gk = _gk((1, T, H, K), 84)
    o, ht = sg.gla_fused_recurrent(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), gk.cuda(),
                                   initial_state=to_dev(inp["h0"]), output_final_state=True, cu_seqlens=to_dev(cu))
    torch.cuda.synchronize()
    ro, rh = oracle.gla_fwd(inp["q"], inp["k"], inp["v"], gk, initial_state=inp["h0"], output_final_state=True,
                            cu_seqlens=cu)
    assert_close(host(o), ro, TOL[torch.bfloat16], "o")
    assert_close(host(ht), rh, TOL[torch.bfloat16], "final_state")


def test_gla_with_equal_gates_is_simple_gla():
    """All K entries of the gate vector equal: GLA reduces to Simple GLA (both GPU
    entry points, same inputs)."""
    inp = random_inputs(2, 64, 4, 128, 128, dtype=torch.bfloat16, gate="g", h0=True, seed=85)
    gk = inp["g"][..., None].expand(2, 64, 4, 128).contiguous()
    d = {k: to_dev(v) for k, v in inp.items()}
    o1, h1 = sg.gla_fused_recurrent(d["q"], d["k"], d["v"], gk.cuda(), initial_state=d["h0"], output_final_state=True)
    o2, h2 = sg.simple_gla_fused_recurrent(d["q"], d["k"], d["v"], g=d["g"], initial_state=d["h0"],
                                           output_final_state=True)
    torch.cuda.synchronize()
    assert_close(host(o1), host(o2), 1e-5, "o")
    assert_close(host(h1), host(h2), 1e-5, "final_state")
