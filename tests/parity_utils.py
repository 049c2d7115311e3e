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


def compare_grads(gpu, ref, tol, inp):
    """Every gradient of the backward within tol: dq, dk, dv, dh0 normalised by their
    largest oracle magnitude; dg and dg_gamma by the larger of that and dg_scale
    (times the token count for dg_gamma, a sum over tokens)."""
    for name in ("dq", "dk", "dv", "dg", "dg_gamma", "dh0"):
        if ref[name] is None:
            assert gpu[name] is None, name
            continue
        x, y = host(gpu[name]), ref[name]
        if name in ("dg", "dg_gamma") and y.size:
            floor = dg_scale(inp, ref) * (inp["q"].shape[0] * inp["q"].shape[1] if name == "dg_gamma" else 1)
            assert np.all(np.isfinite(x)), name
            err = float(np.max(np.abs(x - y)))
            assert err <= tol * max(float(np.max(np.abs(y))), floor), f"{name}: max error {err:.3e}"
        else:
            assert_close(x, y, tol, name)
