"""One long sequence split along time across ranks (the exchange step of
gated_linear_attention_local_b200.seqsplit).

CPU: world-size-3 gloo ranks run the orchestration with the fp64 oracle as the
local forward (and the carry written out in the test), one rank holding an empty
slice; every rank's output and the sequence's final state must equal the oracle on
the whole sequence -- this checks the call order, the all-gather and the indexing
without a GPU.  GPU: the library's kernels (forward, decay total, carry) run for
every rank in turn in one process, the all-gather replaced by stacking (ranks that
wait on one another never run as separate launches on one GPU).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_linear_attention_local_b200.workloads import random_inputs

LENS = [50, 0, 80]
T, H, K, V = sum(LENS), 2, 16, 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_ops():
    import oracle
    from types import SimpleNamespace

    def forward(q, k, v, g, g_gamma, scale, initial_state, output_final_state, chunk_size):
        o, ht = oracle.simple_gla_fwd(q, k, v, g=g, g_gamma=g_gamma, scale=scale, initial_state=initial_state,
                                      output_final_state=True)
        return torch.from_numpy(np.asarray(o)), torch.from_numpy(np.asarray(ht))

    def final_state(k, v, g, g_gamma, chunk_size):
        q = torch.zeros_like(k)
        return forward(q, k, v, g, g_gamma, None, None, True, chunk_size)[1]

    def log_decay_total(g, g_gamma, T_r, H_):
        if g is not None:
            return g[0].double().sum(0)
        if g_gamma is not None:
            return T_r * g_gamma.double()
        return torch.zeros(H_, dtype=torch.float64)

    def state_carry(d_all, s_all, h0, rank):
        h = torch.zeros_like(s_all[0]) if h0 is None else h0.double().clone()
        for r in range(rank):
            h = torch.exp(d_all[r])[:, None, None] * h + s_all[r]
        return h

    return SimpleNamespace(forward=forward, final_state=final_state, log_decay_total=log_decay_total,
                           state_carry=state_carry)


def _slices(inp):
    bounds = np.cumsum([0] + LENS)
    return [{k_: (v_[:, bounds[r]:bounds[r + 1]] if k_ in ("q", "k", "v", "g") and v_ is not None else v_)
             for k_, v_ in inp.items()}
            for r in range(len(LENS))]


def _worker(rank, world, port, out, gate, h0):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from gated_linear_attention_local_b200.seqsplit import chunk_simple_gla_seq_split
    inp = random_inputs(1, T, H, K, V, dtype=torch.float32, gate=gate, h0=h0, seed=7)
    sl = _slices(inp)[rank]
    o, ht = chunk_simple_gla_seq_split(sl["q"], sl["k"], sl["v"], g=sl["g"], g_gamma=inp["g_gamma"],
                                       initial_state=inp["h0"], output_final_state=True, ops=_oracle_ops())
    out[rank] = (o.numpy(), ht.numpy())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("gate,h0", [("g", True), ("gamma", False)])
def test_seq_split_orchestration_on_cpu_ranks(gate, h0):
    import oracle
    world = len(LENS)
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out, gate, h0), nprocs=world, start_method="spawn")
    inp = random_inputs(1, T, H, K, V, dtype=torch.float32, gate=gate, h0=h0, seed=7)
    ro, rh = oracle.simple_gla_fwd(inp["q"], inp["k"], inp["v"], g=inp["g"], g_gamma=inp["g_gamma"],
                                   initial_state=inp["h0"], output_final_state=True)
    bounds = np.cumsum([0] + LENS)
    for r in range(world):
        o, ht = out[r]
        np.testing.assert_allclose(o, ro[:, bounds[r]:bounds[r + 1]], rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(ht, rh, rtol=1e-10, atol=1e-10)


@pytest.mark.gpu
@pytest.mark.parametrize("gate", ["g", "gamma"])
def test_seq_split_kernels_on_one_gpu(gate):
    import oracle
    import gated_linear_attention_local_b200 as sg
    from parity_utils import TOL, assert_close, host
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lens = [700, 0, 300, 1048]
    Tn, Hn, Kn, Vn = sum(lens), 4, 128, 128
    inp = random_inputs(1, Tn, Hn, Kn, Vn, dtype=torch.bfloat16, gate=gate, h0=True, seed=9)
    dev = {k_: (v_.cuda() if v_ is not None else None) for k_, v_ in inp.items()}
    bounds = np.cumsum([0] + lens)
    sl = [{k_: (v_[:, bounds[r]:bounds[r + 1]].contiguous() if k_ in ("q", "k", "v", "g") and v_ is not None else v_)
           for k_, v_ in dev.items()} for r in range(len(lens))]
    summaries = []
    for s in sl:  # phase A on every rank: the state pass alone
        s_r = sg.simple_gla_chunk_final_state(s["k"], s["v"], g=s["g"], g_gamma=s["g_gamma"])
        d_r = sg.simple_gla_log_decay_total(g=s["g"], g_gamma=s["g_gamma"], T=s["q"].shape[1], H=Hn)
        summaries.append((d_r, s_r[0]))
    d_all = torch.stack([d for d, _ in summaries])
    s_all = torch.stack([s_ for _, s_ in summaries])
    outs = []
    for r, s in enumerate(sl):  # phase C on every rank
        h_r = sg.simple_gla_state_carry(d_all, s_all, dev["h0"][0], r)
        o, _ = sg.chunk_simple_gla(s["q"], s["k"], s["v"], g=s["g"], g_gamma=s["g_gamma"], initial_state=h_r[None])
        outs.append(o)
    n0 = sg.lib().sgla_kernel_launch_count()
    final = sg.simple_gla_state_carry(d_all, s_all, dev["h0"][0], len(lens))
    assert sg.lib().sgla_kernel_launch_count() == n0 + 1  # the carry is one counted launch
    torch.cuda.synchronize()
    ro, rh = oracle.simple_gla_fwd(inp["q"], inp["k"], inp["v"], g=inp["g"], g_gamma=inp["g_gamma"],
                                   initial_state=inp["h0"], output_final_state=True)
    assert_close(host(torch.cat(outs, dim=1)), ro, TOL[torch.bfloat16], "o")
    assert_close(host(final), rh[0], TOL[torch.bfloat16], "final_state")
