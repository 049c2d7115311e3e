"""One long sequence split along time across the ranks of a process group.

Every (sequence, head) of a batch is independent, so the data-parallel path needs
no collective (``bench.py`` runs replicas).  A single sequence split along T does
have an exchange step: a rank's outputs depend on the state entering its slice.
Because the gate is one scalar per head, the carry between slices is associative
("Simple GLA in flash-linear-attention: maths and kernels", section 3: the
inter-chunk propagation is only a scalar multiplication of S), so one all-gather of
every rank's summary (total log decay, end state from a zero state) lets each rank
fold the ranks before it:

  phase A   end state of the local slice from a zero state -> S_r (the state pass
            alone, no output); its log decay D_r
  exchange  all_gather of (D_r, S_r) over the group (NCCL on GPUs)
  phase C   h_r = exp(D_{r-1}) h_{r-1} + S_{r-1} (h_0 = the initial state), then the
            forward of the local slice from h_r

The state pass, the forward, the decay total and the fold run in the library's
kernels; this module only orders the calls and moves the summaries
(torch.distributed).
"""
from __future__ import annotations

from types import SimpleNamespace

import torch
import torch.distributed as dist


def library_ops():
    """The CUDA implementations of the local steps."""
    from . import (chunk_simple_gla, simple_gla_chunk_final_state, simple_gla_log_decay_total,
                   simple_gla_state_carry)

    def forward(q, k, v, g, g_gamma, scale, initial_state, output_final_state, chunk_size):
        return chunk_simple_gla(q, k, v, g=g, g_gamma=g_gamma, scale=scale, initial_state=initial_state,
                                output_final_state=output_final_state, chunk_size=chunk_size)

    def final_state(k, v, g, g_gamma, chunk_size):
        return simple_gla_chunk_final_state(k, v, g=g, g_gamma=g_gamma, chunk_size=chunk_size)

    def log_decay_total(g, g_gamma, T, H):
        return simple_gla_log_decay_total(g=g, g_gamma=g_gamma, T=T, H=H)

    return SimpleNamespace(forward=forward, final_state=final_state, log_decay_total=log_decay_total,
                           state_carry=simple_gla_state_carry)


def chunk_simple_gla_seq_split(q, k, v, g=None, g_gamma=None, scale=None, initial_state=None,
                               output_final_state=False, chunk_size=64, group=None, ops=None):
    """q, k [1,T_r,H,K], v [1,T_r,H,V], g [1,T_r,H]: this rank's contiguous slice of one
    sequence (rank order is time order; slices may differ in length).  initial_state
    [1,H,K,V] fp32: the sequence's, the same on every rank, or None.  Returns
    (o [1,T_r,H,V], final_state [1,H,K,V] of the whole sequence on every rank, or
    None).  One all-gather per call; every rank makes the same collective calls."""
    ops = ops or library_ops()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T, H = q.shape[1], q.shape[2]
    # phase A: this slice's summary
    s_r = ops.final_state(k, v, g, g_gamma, chunk_size)
    d_r = ops.log_decay_total(g, g_gamma, T, H)
    # exchange
    d_all = [torch.empty_like(d_r) for _ in range(world)]
    s_all = [torch.empty_like(s_r[0]) for _ in range(world)]
    dist.all_gather(d_all, d_r.contiguous(), group=group)
    dist.all_gather(s_all, s_r[0].contiguous(), group=group)
    d_all, s_all = torch.stack(d_all), torch.stack(s_all)
    h0 = None if initial_state is None else initial_state[0]
    # phase C: the state entering this slice, then the slice from it
    h_r = ops.state_carry(d_all, s_all, h0, rank)
    o, _ = ops.forward(q, k, v, g, g_gamma, scale, h_r[None], False, chunk_size)
    final = ops.state_carry(d_all, s_all, h0, world)[None] if output_final_state else None
    return o, final
