"""GPU parity of GLA with a gate vector over the key dimension in the chunked form
(gla_chunk: vector chunk-local cumsum, intra-chunk scores from 16-token sub-chunks,
inter-chunk state; "relinear", fla-org kernel integration, gate-shape item) against
the fp64 oracle of the recurrence, and against the token-serial form on the GPU.

Cases span several chunks with a ragged last chunk (and sub-chunk), both chunk sizes
(64 tokens for K <= 128, 32 for K <= 256), K that is not a multiple of the key pass,
V leaving a ragged 64-column tile, packed sequences with an empty one, gates from weak
(logsigmoid / 16) to strong (logsigmoid, and 0 = exp(-inf)), log gates of both
signs, and the full token-serial workload on sampled sequences.
"""
import pytest
import torch
import torch.nn.functional as F

import gated_linear_attention_local_b200 as sg
import oracle
from gated_linear_attention_local_b200.workloads import make_workload, random_inputs
from parity_utils import TOL, assert_close, host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _gk(shape, seed, kind="weak"):
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=gen)
    if kind == "weak":       # the layer's normaliser 16
        return F.logsigmoid(x) / 16.0
    if kind == "strong":     # normaliser 1
        return F.logsigmoid(x)
    if kind == "zero":       # gate 0 everywhere
        return torch.full(shape, float("-inf"))
    if kind == "mixed":      # log gates of both signs (a gate above 1 is outside the forget-gate range)
        return 0.05 * x
    raise ValueError(kind)


CASES = [
    # (B, T, H, K, V, dtype, h0, gate kind)
    (2, 200, 2, 128, 128, torch.bfloat16, True, "weak"),
    (2, 200, 2, 128, 128, torch.float32, True, "strong"),
    (1, 130, 3, 64, 72, torch.float32, True, "weak"),
    (2, 77, 2, 256, 64, torch.bfloat16, True, "weak"),
    (1, 100, 2, 200, 40, torch.float32, False, "strong"),
    (2, 64, 2, 40, 24, torch.float32, True, "mixed"),
    (2, 90, 2, 64, 64, torch.float32, True, "zero"),
    (2, 0, 2, 64, 64, torch.float32, True, "weak"),
    (3, 1, 2, 128, 64, torch.bfloat16, True, "weak"),
    # tensor-core walk (bf16, K = 128, V a multiple of 64): several 128-token chunks,
    # a ragged last one, three V tiles, strong and zero gates, no initial state
    (2, 300, 2, 128, 192, torch.bfloat16, True, "strong"),
    (1, 1000, 2, 128, 64, torch.bfloat16, False, "weak"),
    (2, 129, 1, 128, 128, torch.bfloat16, True, "zero"),
    (2, 0, 2, 128, 64, torch.bfloat16, True, "weak"),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}T{c[1]}K{c[3]}V{c[4]}-{str(c[5])[6:]}-h0{int(c[6])}-{c[7]}"
                                             for c in CASES])
def test_gla_chunk_dense(case):
    B, T, H, K, V, dt, h0, kind = case
    inp = random_inputs(B, T, H, K, V, dtype=dt, gate="none", h0=h0, seed=91)
    gk = _gk((B, T, H, K), 92, kind)
    o, ht = sg.gla_chunk(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), gk.cuda(),
                         initial_state=to_dev(inp["h0"]), output_final_state=True)
    torch.cuda.synchronize()
    ro, rh = oracle.gla_fwd(inp["q"], inp["k"], inp["v"], gk, initial_state=inp["h0"], output_final_state=True)
    assert_close(host(o), ro, TOL[dt], "o")
    assert_close(host(ht), rh, TOL[dt], "final_state")


@pytest.mark.parametrize("dt,K", [(torch.bfloat16, 64), (torch.float32, 64), (torch.bfloat16, 128)])
def test_gla_chunk_varlen(dt, K):
    cu = torch.tensor([0, 15, 15, 100, 300, 1200], dtype=torch.int64)
    T, H, V = 1200, 2, 64
    inp = random_inputs(1, T, H, K, V, dtype=dt, gate="none", h0=True, seed=93, cu_seqlens=cu)
    gk = _gk((1, T, H, K), 94, "strong")
    o, ht = sg.gla_chunk(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), gk.cuda(),
                         initial_state=to_dev(inp["h0"]), output_final_state=True, cu_seqlens=cu.cuda())
    torch.cuda.synchronize()
    ro, rh = oracle.gla_fwd(inp["q"], inp["k"], inp["v"], gk, initial_state=inp["h0"], output_final_state=True,
                            cu_seqlens=cu)
    assert_close(host(o), ro, TOL[dt], "o")
    assert_close(host(ht), rh, TOL[dt], "final_state")


def test_gla_chunk_bad_cu_seqlens_is_reported():
    T, H, K, V = 64, 2, 64, 64
    inp = random_inputs(1, T, H, K, V, dtype=torch.bfloat16, gate="none", seed=95)
    gk = _gk((1, T, H, K), 96)
    bad = torch.tensor([0, 40, 30], dtype=torch.int64, device="cuda")
    n = sg.lib().gla_chunk_workspace_size(sg._ptr(bad), 2, T, H, K, V, sg.SGLA_BF16)
    ws = torch.empty(int(n), dtype=torch.uint8, device="cuda")
    sg.gla_chunk(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), gk.cuda(), cu_seqlens=bad, workspace=ws)
    assert sg.workspace_status(ws) != 0


def test_gla_chunk_workload_sampled():
    """The token-serial GLA workload at full size (256 sequences x 64 tokens, H=32,
    K=V=128, bf16) through the chunked form: sequences 0 and 255 against the oracle,
    all of it against the token-serial kernel."""
    w = make_workload("gla_recurrent")
    d = {k: to_dev(w[k]) for k in ("q", "k", "v", "g", "h0")}
    o, ht = sg.gla_chunk(d["q"], d["k"], d["v"], d["g"], initial_state=d["h0"], output_final_state=True)
    o2, ht2 = sg.gla_fused_recurrent(d["q"], d["k"], d["v"], d["g"], initial_state=d["h0"], output_final_state=True)
    torch.cuda.synchronize()
    for n in (0, 255):
        ro, rh = oracle.gla_fwd(w["q"][n:n + 1], w["k"][n:n + 1], w["v"][n:n + 1], w["g"][n:n + 1],
                                initial_state=w["h0"][n:n + 1], output_final_state=True)
        assert_close(host(o[n:n + 1]), ro, TOL[torch.bfloat16], f"o[{n}]")
        assert_close(host(ht[n:n + 1]), rh, TOL[torch.bfloat16], f"final_state[{n}]")
    assert_close(host(o), host(o2), TOL[torch.bfloat16], "o vs token-serial")
    assert_close(host(ht), host(ht2), TOL[torch.bfloat16], "final_state vs token-serial")


def test_gla_chunk_takes_the_tensor_core_walk():
    """bf16 with K = 128 and V a multiple of 64 runs the tcgen05 walk; other shapes the
    CUDA-core one."""
    from gated_linear_attention_local_b200 import _lib
    for K, V, dt, want in ((128, 128, torch.bfloat16, "gla_chunk_walk_tc"), (64, 64, torch.bfloat16, "gla_chunk_walk"),
                           (128, 128, torch.float32, "gla_chunk_walk")):
        inp = random_inputs(1, 200, 2, K, V, dtype=dt, gate="none", seed=97)
        gk = _gk((1, 200, 2, K), 98)
        _lib.profile_begin()
        sg.gla_chunk(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]), gk.cuda())
        torch.cuda.synchronize()
        names = set(_lib.profile_end())
        assert want in names and ({"gla_chunk_walk", "gla_chunk_walk_tc"} - {want}).isdisjoint(names), names
