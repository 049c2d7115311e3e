"""GPU parity of the normalised variant (o = q.S / q.z, scale 1, through the
augmented value of "relinear -- convert pretrained transformers to linear/hybrid-
attention models") against the fp64 oracle, prefill and decode.  q and k are
feature-mapped to be positive, as the method requires q.z > 0."""
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


def _positive(inp, h0_cols=None, seed=0):
    out = dict(inp)
    for n in ("q", "k"):
        out[n] = (inp[n].float().abs() + 0.1).to(inp[n].dtype)
    if h0_cols is not None:
        gen = torch.Generator().manual_seed(seed)
        shp = inp["h0"].shape
        out["h0"] = torch.rand(shp[0], shp[1], shp[2], h0_cols, generator=gen) * 0.1
    return out


CASES = [
    # (B, T, H, K, V, dtype, gate, h0)  V+1 = 128 (no padding), 129 (padded to 192), SIMT
    (2, 300, 2, 128, 127, torch.bfloat16, "g", True),
    (1, 200, 2, 128, 128, torch.bfloat16, "g", False),
    (2, 150, 3, 64, 63, torch.float32, "gamma", True),
    (1, 100, 2, 64, 40, torch.float32, "g", True),
]


@pytest.mark.parametrize("case", CASES, ids=[f"K{c[3]}V{c[4]}-{str(c[5])[6:]}-{c[6]}-h0{int(c[7])}" for c in CASES])
def test_normalized_prefill_dense(case):
    B, T, H, K, V, dt, gate, h0 = case
    inp = random_inputs(B, T, H, K, V, dtype=dt, gate=gate, h0=h0, seed=61)
    inp = _positive(inp, h0_cols=V + 1 if h0 else None, seed=62)
    o, ht = sg.simple_gla_normalized(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), g=to_dev(inp["g"]),
                                     g_gamma=to_dev(inp["g_gamma"]), initial_state=to_dev(inp["h0"]),
                                     output_final_state=True)
    torch.cuda.synchronize()
    ro, rh = oracle.simple_gla_normalized(inp["q"], inp["k"], inp["v"], g=inp["g"], g_gamma=inp["g_gamma"],
                                          initial_state=inp["h0"], output_final_state=True)
    assert tuple(ht.shape) == (B, H, K, V + 1)
    assert_close(host(o), ro, TOL[dt], "o")
    assert_close(host(ht), rh, TOL[dt], "augmented final_state")


def test_normalized_prefill_varlen():
    cu = torch.tensor([0, 15, 100, 300, 1200], dtype=torch.int64)
    T, H, K, V = 1200, 2, 128, 64
    inp = random_inputs(1, T, H, K, V, dtype=torch.bfloat16, gate="g", h0=True, seed=63, cu_seqlens=cu)
    inp = _positive(inp, h0_cols=V + 1, seed=64)
    o, ht = sg.simple_gla_normalized(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), g=to_dev(inp["g"]),
                                     initial_state=to_dev(inp["h0"]), output_final_state=True, cu_seqlens=to_dev(cu))
    torch.cuda.synchronize()
    ro, rh = oracle.simple_gla_normalized(inp["q"], inp["k"], inp["v"], g=inp["g"], initial_state=inp["h0"],
                                          output_final_state=True, cu_seqlens=cu)
    assert_close(host(o), ro, TOL[torch.bfloat16], "o")
    assert_close(host(ht), rh, TOL[torch.bfloat16], "augmented final_state")


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_normalized_decode(dt):
    N, H, K, V, steps = 8, 4, 128, 63, 4
    W = sg.normalized_decode_state_width(V)
    gen = torch.Generator().manual_seed(71)
    state = torch.zeros(N, H, K, W)
    state[..., :V + 1] = torch.rand(N, H, K, V + 1, generator=gen) * 0.1
    ref = state.double().numpy().copy()
    dev_state = state.cuda()
    for s in range(steps):
        q = (torch.randn(N, H, K, generator=gen).abs() + 0.1).to(dt)
        k = (torch.randn(N, H, K, generator=gen).abs() + 0.1).to(dt)
        v = torch.randn(N, H, V, generator=gen).to(dt)
        g = torch.nn.functional.logsigmoid(torch.randn(N, H, generator=gen))
        o = sg.simple_gla_normalized_decode_step(q.cuda(), k.cuda(), v.cuda(), dev_state, g=g.cuda())
        v_aug = np.zeros((N, H, W))
        v_aug[..., :V] = v.double().numpy()
        v_aug[..., V] = 1.0
        ro_aug = oracle.simple_gla_decode_step(q, k, v_aug, ref, g=g, scale=1.0)
        torch.cuda.synchronize()
        assert_close(host(o), ro_aug[..., :V] / ro_aug[..., V:V + 1], TOL[dt], f"o step {s}")
    assert_close(host(dev_state), ref, TOL[dt], "augmented state")
