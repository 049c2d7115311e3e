"""Seeded synthetic inputs for the Simple GLA workloads (no method arithmetic here).

Both the CUDA path and the fp64 oracle are fed from these generators; nothing in
this module computes any part of the operator.  Every tensor is drawn in fp32 on
the CPU from one ``torch.Generator`` seeded with ``seed``, in the fixed order
lengths -> q -> k -> v -> g -> initial state, and then rounded once to the
workload's operand dtype, so both sides see bit-identical operands.

Shapes and distributions follow the workloads the pages describe ("Simple GLA in
flash-linear-attention: maths and kernels", xxqk.cn article, section 2 example:
B=4, T=2048, H=4, K=V=512, q,k,v ~ N(0,1), g = logsigmoid(N(0,1)); section 5: the
test matrix with gate normalisers 0.1/1/10, scales 0.1/1 and the packed lengths
[0,15,100,300,1200,2000]):

  tiny_fp32     B=1 T=256 H=2 K=V=64, fp32 operands, g, scale 1/sqrt(K), final state
  dense_prefill B=4 T=2048 H=4 K=V=512, bf16, g, default scale, final state
  varlen_prefill 8 sequences, lengths uniform in [128, 4096], H=16 K=V=128, bf16, g,
                initial state 0.1*N(0,1), final state
  long_gamma    B=1 T=65536 H=32 K=V=128, bf16 q,k,v ~ N(0,1)/sqrt(K),
                g_gamma[h] = log(1 - 2^(-5 - 5h/31)) (RetNet-style per-head decays),
                no per-token gate, no states
  decode        256 sequences x 64 single-token steps, H=32 K=V=128, bf16, g per step,
                state 0.1*N(0,1) fp32 updated in place
  normalized_prefill  relinear's normalised variant at its measured scale (B=8, T=512,
                d=2048 as H=16 heads of K=V=128): bf16, g, feature-mapped q, k = |N(0,1)| + 0.1,
                scale 1 -- simple_gla_normalized
  gla_recurrent  GLA with a gate vector over the key dimension, token-serial, at the
                recurrent_prefill size: gk = logsigmoid(N(0,1)) / 16 per key -- gla_fused_recurrent
  recurrent_bwd  gradients of the token-serial recurrence at relinear's training scale
                (B=8, T=512, H=16, K=V=128, bf16, g, initial state, output gradient do ~
                N(0,1) and final-state gradient dht ~ 0.1 N(0,1)) --
                simple_gla_fused_recurrent_bwd
  chunk_bwd     the same gradients through the chunked tensor-core path at the same
                size -- simple_gla_chunk_bwd
  gla_chunk_prefill  GLA (gate vector over K) in the chunked form at relinear's training
                scale: B=8, T=512, H=16, K=V=128, bf16, gk = logsigmoid(N(0,1)) / 16 per key,
                initial and final state -- gla_chunk
  recurrent_prefill  the inference routing case of section 4 (at most 64 tokens go to
                the fused recurrence): 256 sequences x 64 tokens, H=32 K=V=128, bf16,
                g, initial state 0.1*N(0,1), final state -- simple_gla_fused_recurrent
"""
from __future__ import annotations

import math

import torch
import torch.nn.functional as F

WORKLOADS = {
    "tiny_fp32": dict(kind="dense", B=1, T=256, H=2, K=64, V=64, dtype=torch.float32, gate="g",
                      h0=False, final_state=True, scale=1.0 / 8.0, chunk_size=64),
    "dense_prefill": dict(kind="dense", B=4, T=2048, H=4, K=512, V=512, dtype=torch.bfloat16, gate="g",
                          h0=False, final_state=True, scale=None, chunk_size=64),
    "varlen_prefill": dict(kind="varlen", N=8, len_lo=128, len_hi=4096, H=16, K=128, V=128,
                           dtype=torch.bfloat16, gate="g", h0=True, final_state=True, scale=None,
                           chunk_size=64),
    "long_gamma": dict(kind="dense", B=1, T=65536, H=32, K=128, V=128, dtype=torch.bfloat16,
                       gate="gamma", qkv_std="rsqrt_k", h0=False, final_state=False, scale=None,
                       chunk_size=64),
    "decode": dict(kind="decode", N=256, steps=64, H=32, K=128, V=128, dtype=torch.bfloat16, gate="g",
                   scale=None),
    "normalized_prefill": dict(kind="dense", entry="normalized", B=8, T=512, H=16, K=128, V=128,
                               dtype=torch.bfloat16, gate="g", h0=False, final_state=True, scale=1.0,
                               chunk_size=64, feature_map="abs"),
    "gla_recurrent": dict(kind="dense", entry="gla", B=256, T=64, H=32, K=128, V=128, dtype=torch.bfloat16,
                          gate="gk", h0=True, final_state=True, scale=None, chunk_size=64),
    "recurrent_bwd": dict(kind="dense", entry="recurrent_bwd", B=8, T=512, H=16, K=128, V=128,
                          dtype=torch.bfloat16, gate="g", h0=True, final_state=False, scale=None, chunk_size=64),
    "chunk_bwd": dict(kind="dense", entry="chunk_bwd", B=8, T=512, H=16, K=128, V=128, dtype=torch.bfloat16,
                      gate="g", h0=True, final_state=False, scale=None, chunk_size=64),
    "gla_chunk_prefill": dict(kind="dense", entry="gla_chunk", B=8, T=512, H=16, K=128, V=128,
                              dtype=torch.bfloat16, gate="gk", h0=True, final_state=True, scale=None, chunk_size=32),
    "recurrent_prefill": dict(kind="dense", entry="recurrent", B=256, T=64, H=32, K=128, V=128,
                              dtype=torch.bfloat16, gate="g", h0=True, final_state=True, scale=None,
                              chunk_size=64),
}


def retnet_gammas(H: int) -> torch.Tensor:
    """log(1 - 2^(-5 - 5h/(H-1))) for h = 0..H-1 (for H == 1: log(1 - 2^-5))."""
    step = 5.0 / (H - 1) if H > 1 else 0.0
    return torch.tensor([math.log(1.0 - 2.0 ** (-5.0 - h * step)) for h in range(H)], dtype=torch.float32)


def random_inputs(B, T, H, K, V, dtype=torch.bfloat16, gate="g", normalizer=1.0, h0=False, seed=0,
                  cu_seqlens=None, qkv_std=1.0, h0_std=0.1):
    """Generic seeded inputs (tests use this for edge cases).

    gate: "g" -> g = logsigmoid(N(0,1)) / normalizer [B,T,H]; "gamma" -> retnet_gammas(H);
          "none" -> no gate; "zero" -> g = 0; "neg_inf" -> g = -inf (gate 0);
          "mixed" -> g = 0.3 N(0,1) (log gates of both signs: a gate above 1 is outside the
          method's forget-gate range, but the operator is still defined).
    With cu_seqlens, B must be 1 and initial states number len(cu_seqlens) - 1.
    Returns a dict of CPU tensors: q,k,v (dtype), g / g_gamma (fp32 or None), h0 (fp32 or None).
    """
    gen = torch.Generator(device="cpu").manual_seed(seed)
    q = (torch.randn(B, T, H, K, generator=gen) * qkv_std).to(dtype)
    k = (torch.randn(B, T, H, K, generator=gen) * qkv_std).to(dtype)
    v = (torch.randn(B, T, H, V, generator=gen) * qkv_std).to(dtype)
    g = g_gamma = None
    if gate == "g":
        g = F.logsigmoid(torch.randn(B, T, H, generator=gen)) / normalizer
    elif gate == "gamma":
        g_gamma = retnet_gammas(H)
    elif gate == "zero":
        g = torch.zeros(B, T, H)
    elif gate == "neg_inf":
        g = torch.full((B, T, H), float("-inf"))
    elif gate == "mixed":
        g = 0.3 * torch.randn(B, T, H, generator=gen)
    N = (len(cu_seqlens) - 1) if cu_seqlens is not None else B
    s0 = (torch.randn(N, H, K, V, generator=gen) * h0_std) if h0 else None
    return dict(q=q, k=k, v=v, g=g, g_gamma=g_gamma, h0=s0)


def random_cotangents(v_shape, N, H, K, V, dtype=torch.bfloat16, dht=True, seed=0, dht_std=0.1):
    """Seeded output gradients for the backward: do shaped like v (dtype) and dht
    [N,H,K,V] fp32 (or None).  CPU tensors."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    do = torch.randn(*v_shape, generator=gen).to(dtype)
    dh = (torch.randn(N, H, K, V, generator=gen) * dht_std) if dht else None
    return do, dh


def make_workload(name: str, seed: int = 0):
    """Inputs of a named workload as CPU tensors plus its call options."""
    w = WORKLOADS[name]
    gen = torch.Generator(device="cpu").manual_seed(seed)
    dt = w["dtype"]
    if w["kind"] == "decode":
        S, N, H, K, V = w["steps"], w["N"], w["H"], w["K"], w["V"]
        q = torch.randn(S, N, H, K, generator=gen).to(dt)
        k = torch.randn(S, N, H, K, generator=gen).to(dt)
        v = torch.randn(S, N, H, V, generator=gen).to(dt)
        g = F.logsigmoid(torch.randn(S, N, H, generator=gen))
        state = torch.randn(N, H, K, V, generator=gen) * 0.1
        return dict(name=name, kind="decode", q=q, k=k, v=v, g=g, g_gamma=None, state=state,
                    scale=w["scale"], N=N, H=H, K=K, V=V, steps=S)
    H, K, V = w["H"], w["K"], w["V"]
    cu = None
    if w["kind"] == "varlen":
        lens = torch.randint(w["len_lo"], w["len_hi"] + 1, (w["N"],), generator=gen)
        cu = torch.zeros(w["N"] + 1, dtype=torch.int64)
        cu[1:] = torch.cumsum(lens, 0)
        B, T = 1, int(cu[-1])
    else:
        B, T = w["B"], w["T"]
    std = 1.0 / math.sqrt(K) if w.get("qkv_std") == "rsqrt_k" else 1.0
    q = torch.randn(B, T, H, K, generator=gen) * std
    k = torch.randn(B, T, H, K, generator=gen) * std
    if w.get("feature_map") == "abs":  # positive feature maps: q.z > 0 for the normalised variant
        q, k = q.abs() + 0.1, k.abs() + 0.1
    q, k = q.to(dt), k.to(dt)
    v = (torch.randn(B, T, H, V, generator=gen) * std).to(dt)
    g = F.logsigmoid(torch.randn(B, T, H, generator=gen)) if w["gate"] == "g" else None
    if w["gate"] == "gk":  # GLA: one log gate per key, gate logit normaliser 16 (section 4)
        g = F.logsigmoid(torch.randn(B, T, H, K, generator=gen)) / 16.0
    g_gamma = retnet_gammas(H) if w["gate"] == "gamma" else None
    N = (len(cu) - 1) if cu is not None else B
    h0 = torch.randn(N, H, K, V, generator=gen) * 0.1 if w["h0"] else None
    do = dht = None
    if w.get("entry") in ("recurrent_bwd", "chunk_bwd"):
        do, dht = random_cotangents(v.shape, N, H, K, V, dtype=dt, seed=seed + 1)
    return dict(name=name, kind=w["kind"], entry=w.get("entry", "chunk"), q=q, k=k, v=v, g=g, g_gamma=g_gamma,
                h0=h0, cu_seqlens=cu, scale=w["scale"], output_final_state=w["final_state"],
                chunk_size=w["chunk_size"], B=B, T=T, N=N, H=H, K=K, V=V, do=do, dht=dht)
