"""The workspace-free forward (simple_gla_fwd_noalloc) against the regular one.

simple_gla_fwd_noalloc exists for callers that are not allowed to allocate device
memory (e.g. a plugin inside a runtime that owns the GPU memory pool); it draws
its scratch from a fixed array inside the library.  Here it is called twice in a
row through the C ABI -- with different inputs, so stale scratch from the first
call could not hide a fault in the second -- and each result is compared with
simple_gla_fwd on the same inputs and with the fp64 oracle, within the parity
tolerance of the other GPU tests; the status word it leaves in the built-in
scratch must read clean.  The Python wrapper is checked too: without a gate and
without a final state, and refusing mis-shaped gates before anything is launched.
This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import gated_linear_attention_local_b200 as sg
from gated_linear_attention_local_b200 import _lib as L
from gated_linear_attention_local_b200.workloads import random_inputs
from parity_utils import TOL, assert_close, host, oracle_fwd

pytestmark = pytest.mark.gpu


def _call_noalloc(d, scale=None, chunk=64):
    q, k, v = d["q"], d["k"], d["v"]
    B, T, H, K = q.shape
    V = v.shape[3]
    o = torch.empty((B, T, H, V), dtype=q.dtype, device=q.device)
    ht = torch.empty((B, H, K, V), dtype=torch.float32, device=q.device)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    dt = L.SGLA_BF16 if q.dtype == torch.bfloat16 else L.SGLA_FP32
    st = L.lib().simple_gla_fwd_noalloc(p(q), p(k), p(v), p(d["g"]), p(d["g_gamma"]),
                                        ctypes.c_float(float("nan") if scale is None else scale), p(d["h0"]),
                                        p(o), p(ht), B, T, H, K, V, chunk, dt,
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == L.SGLA_OK, L.status_name(st)
    return o, ht


@pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cases = [(2, 300, 2, 128, 128, torch.bfloat16, "g", 11), (1, 257, 3, 64, 64, torch.float32, "gamma", 12)]
    for B, T, H, K, V, dt, gate, seed in cases:
        inp = random_inputs(B, T, H, K, V, dt, gate=gate, h0=True, seed=seed)
        d = {k_: (v_.cuda() if v_ is not None else None) for k_, v_ in inp.items()}
        o_na, ht_na = _call_noalloc(d)
        o_ws, ht_ws = sg.simple_gla_fwd(d["q"], d["k"], d["v"], g=d["g"], g_gamma=d["g_gamma"],
                                        initial_state=d["h0"], output_final_state=True)
        torch.cuda.synchronize()
        assert sg.noalloc_status() == 0
        assert_close(host(o_na), host(o_ws), TOL[dt], "o")
        assert_close(host(ht_na), host(ht_ws), TOL[dt], "final_state")
        ro, rht = oracle_fwd(inp)
        assert_close(host(o_na), ro, TOL[dt], "o vs oracle")
        assert_close(host(ht_na), rht, TOL[dt], "final_state vs oracle")


@pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")
def test_noalloc_python_wrapper_without_gate_or_final_state():
    inp = random_inputs(1, 200, 2, 128, 64, torch.bfloat16, gate="none", h0=False, seed=13)
    d = {k_: (v_.cuda() if v_ is not None else None) for k_, v_ in inp.items()}
    o, ht = sg.simple_gla_fwd_noalloc(d["q"], d["k"], d["v"], output_final_state=False)
    assert ht is None
    o_ws, _ = sg.simple_gla_fwd(d["q"], d["k"], d["v"])
    torch.cuda.synchronize()
    assert sg.noalloc_status() == 0
    assert_close(host(o), host(o_ws), TOL[torch.bfloat16], "o")
    ro, _ = oracle_fwd(inp, final=False)
    assert_close(host(o), ro, TOL[torch.bfloat16], "o vs oracle")


@pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")
def test_noalloc_python_wrapper_refuses_misshaped_gates():
    q = torch.zeros(1, 64, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        sg.simple_gla_fwd_noalloc(q, q, q, g=torch.zeros(1, 32, 2, device="cuda"))
    with pytest.raises(ValueError):
        sg.simple_gla_fwd_noalloc(q, q, q, g_gamma=torch.zeros(3, device="cuda"))


@pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")
def test_noalloc_refuses_problems_beyond_its_scratch():
    x = torch.zeros(1, 1, 1, 16, dtype=torch.bfloat16, device="cuda")
    # a size whose workspace is far above 16 MiB: refused before any pointer is used
    st = L.lib().simple_gla_fwd_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(x.data_ptr()),
                                        ctypes.c_void_p(x.data_ptr()), None, None, ctypes.c_float(1.0), None,
                                        ctypes.c_void_p(x.data_ptr()), None, 64, 65536, 32, 128, 128, 64,
                                        L.SGLA_BF16, None)
    assert st == L.SGLA_ERR_WORKSPACE
