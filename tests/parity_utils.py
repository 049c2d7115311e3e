"""Shared helpers for the GPU parity tests: run the CUDA path and the fp64 oracle
on the same seeded inputs and compare.

Tolerance (a reading of the stated "max-abs/rel error 2e-2 for bf16 operands and
1e-4 for fp32 operands"): per output tensor, max|gpu - oracle| <= tol * max|oracle|,
i.e. the max-abs error normalised by the oracle's largest magnitude, and every
value finite.  A plain absolute threshold would be vacuous for small outputs and
narrower than one bf16 rounding of o for large ones.
"""
import numpy as np
import torch

import oracle

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def norm_err(x, y):
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    assert x.shape == y.shape, (x.shape, y.shape)
    if y.size == 0:
        return 0.0
    assert np.all(np.isfinite(x)), "non-finite values in the GPU result"
    denom = max(float(np.max(np.abs(y))), 1e-30)
    return float(np.max(np.abs(x - y))) / denom


def assert_close(x, y, tol, what=""):
    e = norm_err(x, y)
    assert e <= tol, f"{what}: normalised max error {e:.3e} > {tol:.1e}"
    return e


def to_dev(t):
    return None if t is None else t.cuda()


def host(t):
    return None if t is None else t.detach().float().cpu().numpy()


def oracle_fwd(inp, scale=None, final=True, cu=None):
    return oracle.simple_gla_fwd(inp["q"], inp["k"], inp["v"], g=inp.get("g"), g_gamma=inp.get("g_gamma"),
                                 scale=scale, initial_state=inp.get("h0"), output_final_state=final,
                                 cu_seqlens=cu)


def dg_scale(inp, ref):
    """Magnitude of the terms the gate gradient is assembled from: dg_t sums
    q_i . dq_i - k_i . dk_i over the tokens from t on (a reverse cumulative sum), so
    its rounding error is relative to those terms, not to dg itself -- which is
    exactly 0 when every gate is 0."""
    q = np.asarray(inp["q"].double().numpy())
    k = np.asarray(inp["k"].double().numpy())
    terms = np.abs((q * ref["dq"]).sum(-1)) + np.abs((k * ref["dk"]).sum(-1))
    return float(terms.max()) if terms.size else 0.0


def oracle_bwd(inp, do, dht, scale=None, cu=None):
    """The oracle's reverse mode on `inp`.  With a per-head decay (g_gamma) it also
    returns, as "dg_tokens", the per-token gate gradients of the same loss: the
    oracle run again with that decay given as a per-token gate.  dg_gamma is their
    sum over the tokens of every sequence, so its rounding error is measured against
    the sum of their magnitudes."""
    ref = oracle.simple_gla_bwd(inp["q"], inp["k"], inp["v"], do, g=inp.get("g"), g_gamma=inp.get("g_gamma"),
                                scale=scale, initial_state=inp.get("h0"), dht=dht, cu_seqlens=cu)
    if inp.get("g_gamma") is not None:
        B, T, H = inp["q"].shape[:3]
        g_tok = inp["g_gamma"].view(1, 1, H).expand(B, T, H).contiguous()
        tok = oracle.simple_gla_bwd(inp["q"], inp["k"], inp["v"], do, g=g_tok, scale=scale,
                                    initial_state=inp.get("h0"), dht=dht, cu_seqlens=cu)
        ref["dg_tokens"] = tok["dg"]
    return ref


def compare_grads(gpu, ref, tol, inp):
    """Every gradient of the backward within tol: dq, dk, dv, dh0 normalised by their
    largest oracle magnitude; dg by the larger of that and dg_scale; dg_gamma[h] (a
    sum over tokens of per-token gate gradients) by the larger of |dg_gamma[h]| and
    the sum over tokens of |per-token gate gradient| + |q.dq| + |k.dk| for head h,
    taken from the oracle (``oracle_bwd`` supplies the per-token gradients)."""
    for name in ("dq", "dk", "dv", "dg", "dg_gamma", "dh0"):
        if ref[name] is None:
            assert gpu[name] is None, name
            continue
        x, y = host(gpu[name]), ref[name]
        if name == "dg" and y.size:
            assert np.all(np.isfinite(x)), name
            err = float(np.max(np.abs(x - y)))
            assert err <= tol * max(float(np.max(np.abs(y))), dg_scale(inp, ref)), f"{name}: max error {err:.3e}"
        elif name == "dg_gamma" and y.size:
            assert "dg_tokens" in ref, "dg_gamma needs the per-token gate gradients (parity_utils.oracle_bwd)"
            assert np.all(np.isfinite(x)), name
            q = np.asarray(inp["q"].double().numpy())
            k = np.asarray(inp["k"].double().numpy())
            terms = np.abs(ref["dg_tokens"]) + np.abs((q * ref["dq"]).sum(-1)) + np.abs((k * ref["dk"]).sum(-1))
            floor = terms.sum(axis=(0, 1))  # per head
            err = np.abs(x - y)
            bound = tol * np.maximum(np.abs(y), floor)
            assert np.all(err <= bound), f"{name}: errors {err} above {bound}"
        else:
            assert_close(x, y, tol, name)
