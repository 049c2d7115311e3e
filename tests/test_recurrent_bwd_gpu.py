"""GPU parity of the backward of the token-serial recurrence
(simple_gla_fused_recurrent_bwd), through the C ABI, against the fp64 oracle's
reverse-mode gradients (which are pinned by finite differences on the CPU).

The article's section 5 checks the recurrent path for o, the final state and the
gradients dq, dk, dv, dg and dh0 over scales, gate normalisers, dtypes and packed
non-aligned lengths; the cases below follow those axes, plus the edges of the kernels
(a head dimension that is not a multiple of 32, a V that leaves a ragged 64-column
tile, empty sequences, gates of 0 and above 1).
"""
import numpy as np
import pytest
import torch

import gated_linear_attention_local_b200 as sg
import oracle
from gated_linear_attention_local_b200.workloads import random_cotangents, random_inputs
from parity_utils import TOL, assert_close, compare_grads, host, oracle_bwd, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _run(inp, do, dht, scale=None, cu=None):
    dev = {k: to_dev(v) for k, v in inp.items()}
    gpu = sg.simple_gla_fused_recurrent_bwd(dev["q"], dev["k"], dev["v"], to_dev(do), g=dev["g"],
                                            g_gamma=dev["g_gamma"], scale=scale, initial_state=dev["h0"],
                                            dht=to_dev(dht), cu_seqlens=to_dev(cu))
    torch.cuda.synchronize()
    ref = oracle_bwd(inp, do, dht, scale=scale, cu=cu)
    return gpu, ref


DENSE = [
    # (N, T, H, K, V, dtype, gate, normalizer, h0, dht, scale)
    (2, 64, 3, 128, 128, torch.bfloat16, "g", 1.0, True, True, None),
    (2, 64, 3, 128, 128, torch.float32, "gamma", 1.0, True, True, None),
    (1, 100, 2, 256, 64, torch.float32, "g", 1.0, False, False, None),
    (2, 17, 4, 512, 40, torch.bfloat16, "none", 1.0, True, True, None),
    (2, 33, 2, 20, 8, torch.float32, "g", 10.0, True, False, 1.0),
    (1, 64, 2, 64, 64, torch.float32, "g", 0.1, True, True, 0.1),
    (2, 0, 2, 64, 64, torch.float32, "g", 1.0, True, True, None),
    (2, 40, 2, 64, 64, torch.float32, "neg_inf", 1.0, True, True, None),
    (2, 40, 2, 64, 72, torch.float32, "mixed", 1.0, True, True, None),
    (1, 300, 1, 32, 200, torch.bfloat16, "gamma", 1.0, False, True, None),
]


@pytest.mark.parametrize("case", DENSE, ids=[f"N{c[0]}T{c[1]}H{c[2]}K{c[3]}V{c[4]}-{str(c[5])[6:]}-{c[6]}"
                                              f"-h0{int(c[8])}-dht{int(c[9])}" for c in DENSE])
def test_fused_recurrent_bwd_dense(case):
    N, T, H, K, V, dt, gate, norm, h0, dht, scale = case
    inp = random_inputs(N, T, H, K, V, dtype=dt, gate=gate, normalizer=norm, h0=h0, seed=23)
    do, dh = random_cotangents(inp["v"].shape, N, H, K, V, dtype=dt, dht=dht, seed=24)
    gpu, ref = _run(inp, do, dh, scale=scale)
    compare_grads(gpu, ref, TOL[dt], inp)


@pytest.mark.parametrize("gate", ["g", "gamma"])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_fused_recurrent_bwd_varlen(dt, gate):
    # the non-aligned packed lengths of the article's section 5 test matrix, plus an
    # empty sequence
    cu = torch.tensor([0, 15, 15, 100, 300, 1200, 2000], dtype=torch.int64)
    T, H, K, V = 2000, 2, 64, 64
    inp = random_inputs(1, T, H, K, V, dtype=dt, gate=gate, h0=True, seed=31, cu_seqlens=cu)
    do, dh = random_cotangents(inp["v"].shape, len(cu) - 1, H, K, V, dtype=dt, seed=32)
    gpu, ref = _run(inp, do, dh, cu=cu)
    compare_grads(gpu, ref, TOL[dt], inp)


def test_fused_recurrent_bwd_bad_cu_seqlens():
    """A sequence whose bounds fall outside the packed tokens is skipped; the valid one
    is exact."""
    T, H, K, V = 30, 2, 64, 64
    inp = random_inputs(1, T, H, K, V, dtype=torch.float32, gate="g", h0=True, seed=41,
                        cu_seqlens=torch.zeros(4))
    do, dh = random_cotangents(inp["v"].shape, 3, H, K, V, dtype=torch.float32, seed=42)
    bad = torch.tensor([0, 10, 40, 30], dtype=torch.int64)
    dev = {k: to_dev(v) for k, v in inp.items()}
    gpu = sg.simple_gla_fused_recurrent_bwd(dev["q"], dev["k"], dev["v"], to_dev(do), g=dev["g"],
                                            initial_state=dev["h0"], dht=to_dev(dh), cu_seqlens=to_dev(bad))
    torch.cuda.synchronize()
    sl = {k: (v[:, :10] if k in ("q", "k", "v", "g") else v) for k, v in inp.items() if v is not None}
    ref = oracle.simple_gla_bwd(sl["q"], sl["k"], sl["v"], do[:, :10], g=sl["g"], initial_state=inp["h0"][:1],
                                dht=dh[:1], cu_seqlens=torch.tensor([0, 10]))
    tol = TOL[torch.float32]
    for name in ("dq", "dk", "dv", "dg"):
        assert_close(host(gpu[name])[:, :10], ref[name], tol, name)
    assert_close(host(gpu["dh0"])[:1], ref["dh0"], tol, "dh0")


def test_fused_recurrent_bwd_matches_autograd_of_the_forward():
    """Cross-check of the two CUDA entry points: the gradient of sum(o * do) through
    the forward recurrence, taken by finite differences of the forward kernel along a
    random direction, equals <backward gradient, direction> (fp32)."""
    N, T, H, K, V = 1, 24, 2, 32, 32
    inp = random_inputs(N, T, H, K, V, dtype=torch.float32, gate="g", h0=True, seed=51)
    do, dh = random_cotangents(inp["v"].shape, N, H, K, V, dtype=torch.float32, seed=52)
    dev = {k: to_dev(v) for k, v in inp.items()}
    gpu = sg.simple_gla_fused_recurrent_bwd(dev["q"], dev["k"], dev["v"], to_dev(do), g=dev["g"],
                                            initial_state=dev["h0"], dht=to_dev(dh))
    gen = torch.Generator(device="cpu").manual_seed(53)
    dirs = {n: torch.randn(inp[n].shape, generator=gen) for n in ("q", "k", "v", "g", "h0")}

    def loss(eps):
        x = {n: to_dev(inp[n] + eps * dirs[n]) for n in dirs}
        o, ht = sg.simple_gla_fused_recurrent(x["q"], x["k"], x["v"], g=x["g"], initial_state=x["h0"],
                                              output_final_state=True)
        return float((o.double() * to_dev(do).double()).sum() + (ht.double() * to_dev(dh).double()).sum())

    eps = 1e-2
    fd = (loss(eps) - loss(-eps)) / (2 * eps)
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "h0": "dh0"}
    an = sum(float((gpu[names[n]].double().cpu() * dirs[n].double()).sum()) for n in dirs)
    assert abs(fd - an) <= 2e-3 * max(1.0, abs(an)), (fd, an)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_simple_gla_fused_recurrent_bwd_state_v_first(dt):
    """States and their gradients in the [V,K] layout (the article's section 2
    state_v_first; section 5 checks both layouts' gradients against each other): the
    oracle runs on the transposed [K,V] states and its dh0 is transposed back."""
    N, T, H, K, V = 2, 150, 2, 128, 64
    inp = random_inputs(N, T, H, K, V, dtype=dt, gate="g", h0=True, seed=71)
    do, dh = random_cotangents(inp["v"].shape, N, H, K, V, dtype=dt, seed=72)
    h0_vk, dh_vk = inp["h0"].transpose(-1, -2).contiguous(), dh.transpose(-1, -2).contiguous()
    dev = {k: to_dev(v) for k, v in inp.items()}
    gpu = sg.simple_gla_fused_recurrent_bwd(dev["q"], dev["k"], dev["v"], to_dev(do), g=dev["g"], initial_state=to_dev(h0_vk),
             dht=to_dev(dh_vk), state_v_first=True)
    torch.cuda.synchronize()
    assert tuple(gpu["dh0"].shape) == (N, H, V, K)
    gpu["dh0"] = gpu["dh0"].transpose(-1, -2)
    ref = oracle.simple_gla_bwd(inp["q"], inp["k"], inp["v"], do, g=inp["g"], initial_state=inp["h0"], dht=dh)
    compare_grads(gpu, ref, TOL[dt], inp)
