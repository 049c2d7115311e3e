"""GPU parity of the chunked backward (simple_gla_chunk_bwd), through the C ABI,
against the fp64 oracle's reverse mode (pinned by finite differences on the CPU).

The chunked backward runs the chunked forward three times on permuted and
time-reversed operands (the gradient recurrence is the forward recurrence backward in
time), so the cases cover what changes under those permutations: K != V in both
orders, lengths that leave a ragged last chunk after reversal, packed sequences of the
article's section 5 test matrix with an empty one, sequences long enough for the
segmented state pass, every chunk size, the SIMT (fp32) and tensor-core (bf16)
paths, and the full training-scale batch on sampled sequences.
"""
import pytest
import torch

import gated_linear_attention_local_b200 as sg
import oracle
from gated_linear_attention_local_b200.workloads import make_workload, random_cotangents, random_inputs
from parity_utils import TOL, compare_grads, host, oracle_bwd, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _gpu(inp, do, dht, scale=None, cu=None, chunk_size=64):
    dev = {k: to_dev(v) for k, v in inp.items()}
    out = sg.simple_gla_chunk_bwd(dev["q"], dev["k"], dev["v"], to_dev(do), g=dev["g"], g_gamma=dev["g_gamma"],
                                  scale=scale, initial_state=dev["h0"], dht=to_dev(dht), cu_seqlens=to_dev(cu),
                                  chunk_size=chunk_size)
    torch.cuda.synchronize()
    return out


def _oracle(inp, do, dht, scale=None, cu=None):
    return oracle_bwd(inp, do, dht, scale=scale, cu=cu)


DENSE = [
    # (N, T, H, K, V, dtype, gate, normalizer, h0, dht, scale)
    (2, 256, 3, 128, 128, torch.bfloat16, "g", 1.0, True, True, None),
    (2, 200, 2, 64, 128, torch.bfloat16, "gamma", 1.0, True, True, None),
    (2, 200, 2, 128, 64, torch.bfloat16, "g", 10.0, False, True, 0.1),
    (1, 300, 2, 128, 64, torch.float32, "g", 1.0, True, True, None),
    (2, 130, 2, 64, 64, torch.bfloat16, "none", 1.0, True, True, None),
    (2, 0, 2, 64, 64, torch.float32, "g", 1.0, True, True, None),
    (2, 90, 2, 64, 64, torch.float32, "neg_inf", 1.0, True, True, None),
    (2, 90, 2, 64, 72, torch.float32, "mixed", 1.0, True, True, None),
    (1, 4096, 2, 128, 128, torch.bfloat16, "g", 1.0, True, True, None),
    (1, 300, 1, 512, 512, torch.bfloat16, "g", 1.0, True, True, None),
    (1, 77, 2, 40, 24, torch.float32, "gamma", 1.0, True, False, 1.0),
]


@pytest.mark.parametrize("case", DENSE, ids=[f"N{c[0]}T{c[1]}H{c[2]}K{c[3]}V{c[4]}-{str(c[5])[6:]}-{c[6]}"
                                              f"-h0{int(c[8])}-dht{int(c[9])}" for c in DENSE])
def test_chunk_bwd_dense(case):
    N, T, H, K, V, dt, gate, norm, h0, dht, scale = case
    inp = random_inputs(N, T, H, K, V, dtype=dt, gate=gate, normalizer=norm, h0=h0, seed=61)
    do, dh = random_cotangents(inp["v"].shape, N, H, K, V, dtype=dt, dht=dht, seed=62)
    compare_grads(_gpu(inp, do, dh, scale=scale), _oracle(inp, do, dh, scale=scale), TOL[dt], inp)


@pytest.mark.parametrize("chunk_size", [16, 32, 64, 128])
def test_chunk_bwd_chunk_sizes(chunk_size):
    inp = random_inputs(2, 150, 2, 64, 64, dtype=torch.bfloat16, gate="g", h0=True, seed=63)
    do, dh = random_cotangents(inp["v"].shape, 2, 2, 64, 64, dtype=torch.bfloat16, seed=64)
    compare_grads(_gpu(inp, do, dh, chunk_size=chunk_size), _oracle(inp, do, dh), TOL[torch.bfloat16], inp)


@pytest.mark.parametrize("gate", ["g", "gamma"])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_chunk_bwd_varlen(dt, gate):
    cu = torch.tensor([0, 15, 15, 100, 300, 1200, 2000], dtype=torch.int64)
    T, H, K, V = 2000, 2, 64, 64
    inp = random_inputs(1, T, H, K, V, dtype=dt, gate=gate, h0=True, seed=65, cu_seqlens=cu)
    do, dh = random_cotangents(inp["v"].shape, len(cu) - 1, H, K, V, dtype=dt, seed=66)
    compare_grads(_gpu(inp, do, dh, cu=cu), _oracle(inp, do, dh, cu=cu), TOL[dt], inp)


def test_chunk_bwd_bad_cu_seqlens_is_reported():
    T, H, K, V = 64, 2, 64, 64
    inp = random_inputs(1, T, H, K, V, dtype=torch.bfloat16, gate="g", h0=True, seed=67, cu_seqlens=torch.zeros(3))
    do, dh = random_cotangents(inp["v"].shape, 2, H, K, V, dtype=torch.bfloat16, seed=68)
    bad = torch.tensor([0, 40, 30], dtype=torch.int64, device="cuda")
    dev = {k: to_dev(v) for k, v in inp.items()}
    n = sg.lib().simple_gla_chunk_bwd_workspace_size(sg._ptr(bad), 2, T, H, K, V, 64, sg.SGLA_BF16)
    ws = torch.empty(int(n), dtype=torch.uint8, device="cuda")
    sg.simple_gla_chunk_bwd(dev["q"][0], dev["k"][0], dev["v"][0], to_dev(do)[0], g=dev["g"][0],
                            initial_state=dev["h0"], dht=to_dev(dh), cu_seqlens=bad, workspace=ws)
    assert sg.workspace_status(ws) != 0


def test_chunk_bwd_training_batch_sampled():
    """The full training-scale batch (B=8, T=512, H=16, K=V=128, bf16) in the launch
    configuration the benchmark times; the oracle checks sequences 0 and 7 (every
    (sequence, head) is independent) and the token-serial backward cross-checks all."""
    w = make_workload("recurrent_bwd")
    inp = dict(q=w["q"], k=w["k"], v=w["v"], g=w["g"], g_gamma=w["g_gamma"], h0=w["h0"])
    gpu = _gpu(inp, w["do"], w["dht"])
    for n in (0, 7):
        sl = dict(q=w["q"][n:n + 1], k=w["k"][n:n + 1], v=w["v"][n:n + 1], g=w["g"][n:n + 1], g_gamma=None,
                  h0=w["h0"][n:n + 1])
        ref = _oracle(sl, w["do"][n:n + 1], w["dht"][n:n + 1])
        part = {k: (None if t is None else t[n:n + 1]) for k, t in gpu.items()}
        compare_grads(part, ref, TOL[torch.bfloat16], sl)
    dev = {k: to_dev(v) for k, v in inp.items()}
    rec = sg.simple_gla_fused_recurrent_bwd(dev["q"], dev["k"], dev["v"], to_dev(w["do"]), g=dev["g"],
                                            initial_state=dev["h0"], dht=to_dev(w["dht"]))
    torch.cuda.synchronize()
    for name in ("dq", "dk", "dv", "dh0"):
        a, b = host(gpu[name]), host(rec[name])
        assert abs(a - b).max() <= 2e-2 * abs(b).max(), name


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_simple_gla_chunk_bwd_state_v_first(dt):
    """States and their gradients in the [V,K] layout (the article's section 2
    state_v_first; section 5 checks both layouts' gradients against each other): the
    oracle runs on the transposed [K,V] states and its dh0 is transposed back."""
    N, T, H, K, V = 2, 150, 2, 128, 64
    inp = random_inputs(N, T, H, K, V, dtype=dt, gate="g", h0=True, seed=71)
    do, dh = random_cotangents(inp["v"].shape, N, H, K, V, dtype=dt, seed=72)
    h0_vk, dh_vk = inp["h0"].transpose(-1, -2).contiguous(), dh.transpose(-1, -2).contiguous()
    dev = {k: to_dev(v) for k, v in inp.items()}
    gpu = sg.simple_gla_chunk_bwd(dev["q"], dev["k"], dev["v"], to_dev(do), g=dev["g"], initial_state=to_dev(h0_vk),
             dht=to_dev(dh_vk), state_v_first=True)
    torch.cuda.synchronize()
    assert tuple(gpu["dh0"].shape) == (N, H, V, K)
    gpu["dh0"] = gpu["dh0"].transpose(-1, -2)
    ref = oracle.simple_gla_bwd(inp["q"], inp["k"], inp["v"], do, g=inp["g"], initial_state=inp["h0"], dht=dh)
    compare_grads(gpu, ref, TOL[dt], inp)


@pytest.mark.parametrize("packed", [False, True])
def test_chunk_simple_gla_is_differentiable(packed):
    """chunk_simple_gla with inputs that require gradients: loss.backward() fills
    q.grad .. initial_state.grad with the oracle's reverse-mode gradients."""
    dt = torch.bfloat16
    if packed:
        cu = torch.tensor([0, 100, 100, 300], dtype=torch.int64)
        T, H, K, V = 300, 2, 128, 128
        inp = random_inputs(1, T, H, K, V, dtype=dt, gate="g", h0=True, seed=81, cu_seqlens=cu)
        N = 3
    else:
        cu = None
        N, T, H, K, V = 2, 200, 2, 128, 64
        inp = random_inputs(N, T, H, K, V, dtype=dt, gate="g", h0=True, seed=81)
    do, dh = random_cotangents(inp["v"].shape, N, H, K, V, dtype=dt, seed=82)
    leaves = {n: to_dev(inp[n]).requires_grad_(True) for n in ("q", "k", "v", "g", "h0")}
    o, ht = sg.chunk_simple_gla(leaves["q"], leaves["k"], leaves["v"], g=leaves["g"], initial_state=leaves["h0"],
                                output_final_state=True, cu_seqlens=to_dev(cu))
    loss = (o.float() * to_dev(do).float()).sum() + (ht * to_dev(dh)).sum()
    loss.backward()
    torch.cuda.synchronize()
    ref = oracle.simple_gla_bwd(inp["q"], inp["k"], inp["v"], do, g=inp["g"], initial_state=inp["h0"], dht=dh,
                                cu_seqlens=cu)
    got = dict(dq=leaves["q"].grad, dk=leaves["k"].grad, dv=leaves["v"].grad, dg=leaves["g"].grad,
               dg_gamma=None, dh0=leaves["h0"].grad)
    compare_grads(got, ref, TOL[dt], inp)
