"""The state-only chunked pass (simple_gla_chunk_final_state: the state recurrence of
"Simple GLA in flash-linear-attention", section 3, without the output) against the
fp64 oracle's final state, and a check that it launches no output kernel."""
import numpy as np
import pytest
import torch

import gated_linear_attention_local_b200 as sg
from gated_linear_attention_local_b200.workloads import random_inputs
from parity_utils import TOL, assert_close, host, oracle_fwd

pytestmark = pytest.mark.gpu

CASES = [
    # (B, T, H, K, V, gate, h0, dtype)
    (2, 300, 2, 128, 128, "g", True, torch.bfloat16),
    (1, 5000, 2, 128, 128, "g", False, torch.bfloat16),     # many segments: state pass + carry
    (1, 4100, 2, 128, 64, "gamma", True, torch.bfloat16),   # V not a multiple of 128: k-block state kernel
    (1, 3000, 1, 512, 64, "g", True, torch.bfloat16),       # K = 512
    (2, 700, 2, 128, 128, "none", True, torch.bfloat16),
    (1, 256, 2, 128, 128, "mixed", False, torch.bfloat16),  # positive log gates
    (1, 0, 2, 128, 128, "g", True, torch.bfloat16),         # empty: final state = initial state
    (2, 200, 2, 64, 32, "g", True, torch.float32),          # fp32: CUDA-core state pass
]


def _run(inp, cu=None):
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    from gated_linear_attention_local_b200 import _lib
    _lib.profile_begin()
    ht = sg.simple_gla_chunk_final_state(d["k"], d["v"], g=d["g"], g_gamma=d["g_gamma"], initial_state=d["h0"],
                                         cu_seqlens=None if cu is None else cu.cuda())
    torch.cuda.synchronize()
    prof = _lib.profile_end()
    assert not any(k.startswith("chunk_output") for k in prof), f"an output kernel ran: {sorted(prof)}"
    return ht


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}K{c[3]}V{c[4]}-{c[5]}-h0{int(c[6])}-"
                                                      f"{str(c[7]).split('.')[-1]}")
def test_final_state_matches_oracle(case):
    B, T, H, K, V, gate, h0, dtype = case
    inp = random_inputs(B, T, H, K, V, dtype, gate=gate, h0=h0, seed=71)
    ht = _run(inp)
    _, rh = oracle_fwd(inp)
    assert_close(host(ht), rh, TOL[dtype], "final_state")


@pytest.mark.parametrize("cu_list", [[0, 15, 100, 300, 1200, 2000], [0, 0, 129, 129, 2500, 2501, 6000]])
def test_final_state_varlen(cu_list):
    cu = torch.tensor(cu_list, dtype=torch.int64)
    inp = random_inputs(1, cu_list[-1], 4, 128, 128, torch.bfloat16, gate="g", h0=True, seed=72, cu_seqlens=cu)
    ht = _run(inp, cu)
    _, rh = oracle_fwd(inp, cu=cu)
    assert_close(host(ht), rh, TOL[torch.bfloat16], "final_state varlen")
    # every sequence on its own scale: an empty sequence keeps its initial state exactly
    for n in range(len(cu_list) - 1):
        if cu_list[n + 1] == cu_list[n]:
            np.testing.assert_array_equal(host(ht)[n], inp["h0"][n].numpy())
