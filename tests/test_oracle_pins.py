"""Pins for the fp64 oracle against things other than itself (CPU only).

The method ("Simple GLA in flash-linear-attention: maths and kernels",
xxqk.cn article) defines, per head and token, S_t = exp(g_t) S_{t-1} + k_t v_t^T
and o_t = scale q_t^T S_t (section 1), with the layout, g/g_gamma and varlen
conventions of section 2.  The pages print no numeric example, so the pins are:

* hand-derived worked examples (tests/golden/worked_examples.json), forward and
  gradients;
* brute force of the parallel form: the explicit decay-masked attention matrix
  D_ij = exp(sum_{l=j+1..i} g_l) (j <= i, diagonal included), built by explicit
  summation, O(T^3) -- the view behind parallel_simple_gla / test_parallel in
  section 2 and section 5 of the article;
* closed forms: g == 0 (plain causal linear attention via a library prefix sum),
  gate 0 (g = -inf), constant gate (integer powers gamma^(i-j)), T = 1;
* invariants: split-and-carry (final_state fed back as initial_state), varlen ==
  separate per-sequence calls, decode == forward, linearity, default scale;
* planted mistakes: plausible bugs are planted in a copy of the oracle source and
  each must fail at least one of the pins above.

The brute-force forms (Simple GLA and GLA) and the finite-difference check of the
backward also run over many small random shapes (hypothesis, derandomised),
T = 0 and one-element head dims included.
"""
import json
import math
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
RTOL = 1e-12


def _logsigmoid(x):
    return -np.logaddexp(0.0, -x)


def _inputs(rng, B, T, H, K, V, gate="g", normalizer=1.0, h0=True):
    q = rng.standard_normal((B, T, H, K))
    k = rng.standard_normal((B, T, H, K))
    v = rng.standard_normal((B, T, H, V))
    g = _logsigmoid(rng.standard_normal((B, T, H))) / normalizer if gate == "g" else None
    g_gamma = np.log(1 - 2.0 ** (-5 - np.arange(H) * 0.5)) if gate == "gamma" else None
    s0 = 0.5 * rng.standard_normal((B, H, K, V)) if h0 else None
    return q, k, v, g, g_gamma, s0


def _brute_force_head(q, k, v, a, scale, h0):
    """Parallel form for one (sequence, head): q,k [T,K], v [T,V], a [T] log-gates."""
    T = a.shape[0]
    D = np.zeros((T, T))
    for i in range(T):
        for j in range(i + 1):
            D[i, j] = math.exp(math.fsum(a[l] for l in range(j + 1, i + 1)))
    o = scale * ((q @ k.T) * D) @ v
    ST = np.zeros((q.shape[1], v.shape[1]))
    for j in range(T):
        ST += math.exp(math.fsum(a[j + 1:])) * np.outer(k[j], v[j])
    if h0 is not None:
        lead = np.array([math.exp(math.fsum(a[: i + 1])) for i in range(T)])
        o += scale * lead[:, None] * (q @ h0)
        ST += math.exp(math.fsum(a)) * h0
    return o, ST


def _brute_force(q, k, v, g=None, g_gamma=None, scale=None, h0=None, cu=None):
    B, T, H, K = q.shape
    V = v.shape[3]
    scale = 1.0 / math.sqrt(K) if scale is None else scale
    spans = ([(b, 0, T) for b in range(B)] if cu is None
             else [(0, int(cu[n]), int(cu[n + 1])) for n in range(len(cu) - 1)])
    o = np.zeros((B, T, H, V))
    hT = np.zeros((len(spans), H, K, V))
    for n, (b, t0, t1) in enumerate(spans):
        for h in range(H):
            if g is not None:
                a = g[b, t0:t1, h]
            elif g_gamma is not None:
                a = np.full(t1 - t0, g_gamma[h])
            else:
                a = np.zeros(t1 - t0)
            s0 = None if h0 is None else h0[n, h]
            oo, st = _brute_force_head(q[b, t0:t1, h], k[b, t0:t1, h], v[b, t0:t1, h], a, scale, s0)
            o[b, t0:t1, h] = oo
            hT[n, h] = st
    return o, hT


def _close(x, y, rtol=RTOL):
    scale = max(1.0, float(np.max(np.abs(y)))) if y.size else 1.0
    np.testing.assert_allclose(x, y, rtol=0, atol=rtol * scale)


# ----------------------------------------------------------------------------- pins


def _golden_bwd(c, lib_path):
    """A hand-derived gradient example: every gradient of the loss
    sum_t <o_t, do_t> + <S_T, dht> against the values worked out in its note."""
    T, K = np.array(c["q"]).shape
    V = np.array(c["v"]).shape[1]
    arr = lambda key, *shape: np.array(c[key], dtype=np.float64).reshape(*shape)  # noqa: E731
    g = np.log(arr("gate", 1, T, 1)) if "gate" in c else None
    g_gamma = np.log(np.array([c["gamma"]])) if "gamma" in c else None
    r = oracle.simple_gla_bwd(arr("q", 1, T, 1, K), arr("k", 1, T, 1, K), arr("v", 1, T, 1, V),
                              arr("do", 1, T, 1, V), g=g, g_gamma=g_gamma, scale=c["scale"],
                              initial_state=arr("h0", 1, 1, K, V), dht=arr("dht", 1, 1, K, V), lib_path=lib_path)
    _close(r["dq"].reshape(T, K), arr("dq", T, K), 1e-12)
    _close(r["dk"].reshape(T, K), arr("dk", T, K), 1e-12)
    _close(r["dv"].reshape(T, V), arr("dv", T, V), 1e-12)
    _close(r["dh0"].reshape(K, V), arr("dh0", K, V), 1e-12)
    if "dg" in c:
        _close(r["dg"].reshape(T), arr("dg", T), 1e-12)
    else:
        _close(r["dg_gamma"].reshape(1), np.array([c["dg_gamma"]]), 1e-12)

def pin_golden(lib_path=None):
    with open(os.path.join(HERE, "golden", "worked_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        if c.get("bwd"):
            _golden_bwd(c, lib_path)
            continue
        if c.get("gla"):
            T, K = np.array(c["q"]).shape
            V = np.array(c["v"]).shape[1]
            gk = np.log(np.array(c["gate_vec"])).reshape(1, T, 1, K)
            h0 = np.array(c["h0"]).reshape(1, 1, K, V)
            o, hT = oracle.gla_fwd(np.array(c["q"]).reshape(1, T, 1, K), np.array(c["k"]).reshape(1, T, 1, K),
                                   np.array(c["v"]).reshape(1, T, 1, V), gk, scale=c["scale"], initial_state=h0,
                                   output_final_state=True, lib_path=lib_path)
            _close(o.reshape(T, V), np.array(c["o"]), 1e-13)
            _close(hT.reshape(K, V), np.array(c["hT"]), 1e-13)
            continue
        T, K = np.array(c["q"]).shape
        V = np.array(c["v"]).shape[1]
        q = np.array(c["q"]).reshape(1, T, 1, K)
        k = np.array(c["k"]).reshape(1, T, 1, K)
        v = np.array(c["v"]).reshape(1, T, 1, V)
        g = np.log(np.array(c["gate"])).reshape(1, T, 1)
        if c.get("normalized"):
            o, hT = oracle.simple_gla_normalized(q, k, v, g=g, output_final_state=True, lib_path=lib_path)
            _close(o.reshape(T, V), np.array(c["o"]), 1e-13)
            _close(hT.reshape(K, V + 1), np.array(c["hT"]), 1e-13)
            continue
        vf = bool(c.get("state_v_first", False))
        sshape = (V, K) if vf else (K, V)
        h0 = None if c["h0"] is None else np.array(c["h0"]).reshape(1, 1, *sshape)
        o, hT = oracle.simple_gla_fwd(q, k, v, g=g, scale=c["scale"], initial_state=h0,
                                      output_final_state=True, state_v_first=vf, lib_path=lib_path)
        _close(o.reshape(T, V), np.array(c["o"]), 1e-13)
        _close(hT.reshape(*sshape), np.array(c["hT"]), 1e-13)


def pin_brute_force_dense(lib_path=None):
    rng = np.random.default_rng(1)
    for gate, norm, T, K, V, h0 in [("g", 1.0, 37, 3, 5, True), ("g", 0.1, 20, 4, 2, True),
                                    ("g", 10.0, 41, 2, 3, False), ("gamma", 1.0, 33, 5, 4, True),
                                    ("none", 1.0, 19, 3, 3, True)]:
        q, k, v, g, gg, s0 = _inputs(rng, 2, T, 2, K, V, gate, norm, h0)
        for scale in (None, 0.1, 1.0):
            o, hT = oracle.simple_gla_fwd(q, k, v, g=g, g_gamma=gg, scale=scale, initial_state=s0,
                                          output_final_state=True, lib_path=lib_path)
            ob, hb = _brute_force(q, k, v, g, gg, scale, s0)
            _close(o, ob)
            _close(hT, hb)


def pin_brute_force_varlen(lib_path=None):
    rng = np.random.default_rng(2)
    cu = np.array([0, 5, 5, 17, 30, 31], dtype=np.int64)  # includes an empty and a 1-token sequence
    for gate in ("g", "gamma"):
        q, k, v, g, gg, _ = _inputs(rng, 1, int(cu[-1]), 3, 4, 6, gate)
        s0 = 0.1 * rng.standard_normal((len(cu) - 1, 3, 4, 6))
        o, hT = oracle.simple_gla_fwd(q, k, v, g=g, g_gamma=gg, initial_state=s0,
                                      output_final_state=True, cu_seqlens=cu, lib_path=lib_path)
        ob, hb = _brute_force(q, k, v, g, gg, None, s0, cu)
        _close(o, ob)
        _close(hT, hb)
        _close(hT[1], s0[1])  # zero-length sequence keeps its initial state


def pin_closed_form_no_decay(lib_path=None):
    rng = np.random.default_rng(3)
    q, k, v, _, _, s0 = _inputs(rng, 2, 50, 2, 4, 3, gate="none")
    for g in (None, np.zeros((2, 50, 2))):
        o, hT = oracle.simple_gla_fwd(q, k, v, g=g, scale=0.5, initial_state=s0,
                                      output_final_state=True, lib_path=lib_path)
        kv = np.einsum("bthk,bthv->bthkv", k, v)
        S = np.cumsum(kv, axis=1) + s0[:, None]                 # library prefix sum
        _close(o, 0.5 * np.einsum("bthk,bthkv->bthv", q, S))
        _close(hT, s0 + np.einsum("bthk,bthv->bhkv", k, v))


def pin_special_cases(lib_path=None):
    rng = np.random.default_rng(4)
    # gate 0 everywhere (g = -inf): only the current token survives
    q, k, v, _, _, s0 = _inputs(rng, 1, 9, 2, 3, 4, gate="none")
    g = np.full((1, 9, 2), -np.inf)
    o, hT = oracle.simple_gla_fwd(q, k, v, g=g, scale=1.0, initial_state=s0,
                                  output_final_state=True, lib_path=lib_path)
    _close(o, np.einsum("bthk,bthk->bth", q, k)[..., None] * v)
    _close(hT[0], np.einsum("hk,hv->hkv", k[0, -1], v[0, -1]))
    # constant gate gamma: D_ij = gamma^(i-j) by integer powers (RetNet-style)
    T, gam = 23, 0.9
    q, k, v, _, _, _ = _inputs(rng, 1, T, 1, 3, 2, gate="none", h0=False)
    o, _ = oracle.simple_gla_fwd(q, k, v, g_gamma=np.array([math.log(gam)]), scale=1.0,
                                 lib_path=lib_path)
    idx = np.arange(T)
    D = np.where(idx[:, None] >= idx[None, :],
                 np.power(gam, np.maximum(idx[:, None] - idx[None, :], 0)), 0.0)
    _close(o[0, :, 0], ((q[0, :, 0] @ k[0, :, 0].T) * D) @ v[0, :, 0])
    # T == 1 with an initial state
    q, k, v, g, _, s0 = _inputs(rng, 1, 1, 1, 4, 3)
    o, _ = oracle.simple_gla_fwd(q, k, v, g=g, scale=0.3, initial_state=s0, lib_path=lib_path)
    S = math.exp(g[0, 0, 0]) * s0[0, 0] + np.outer(k[0, 0, 0], v[0, 0, 0])
    _close(o[0, 0, 0], 0.3 * S.T @ q[0, 0, 0])


def pin_split_invariant(lib_path=None):
    rng = np.random.default_rng(5)
    q, k, v, g, _, s0 = _inputs(rng, 2, 150, 2, 4, 5)
    o, hT = oracle.simple_gla_fwd(q, k, v, g=g, initial_state=s0, output_final_state=True,
                                  lib_path=lib_path)
    for t1 in (1, 17, 64, 100, 149):
        o1, h1 = oracle.simple_gla_fwd(q[:, :t1], k[:, :t1], v[:, :t1], g=g[:, :t1],
                                       initial_state=s0, output_final_state=True, lib_path=lib_path)
        o2, h2 = oracle.simple_gla_fwd(q[:, t1:], k[:, t1:], v[:, t1:], g=g[:, t1:],
                                       initial_state=h1, output_final_state=True, lib_path=lib_path)
        _close(np.concatenate([o1, o2], axis=1), o)
        _close(h2, hT)


def pin_varlen_equals_separate(lib_path=None):
    rng = np.random.default_rng(6)
    cu = np.array([0, 15, 100, 130, 131, 200], dtype=np.int64)
    q, k, v, g, _, _ = _inputs(rng, 1, 200, 2, 4, 3)
    s0 = 0.1 * rng.standard_normal((5, 2, 4, 3))
    o, hT = oracle.simple_gla_fwd(q, k, v, g=g, initial_state=s0, output_final_state=True,
                                  cu_seqlens=cu, lib_path=lib_path)
    for n in range(5):
        a, b = cu[n], cu[n + 1]
        on, hn = oracle.simple_gla_fwd(q[:, a:b], k[:, a:b], v[:, a:b], g=g[:, a:b],
                                       initial_state=s0[n:n + 1], output_final_state=True,
                                       lib_path=lib_path)
        _close(o[:, a:b], on)
        _close(hT[n:n + 1], hn)


def pin_decode_equals_forward(lib_path=None):
    rng = np.random.default_rng(7)
    N, T, H, K, V = 3, 20, 2, 4, 5
    q, k, v, g, _, s0 = _inputs(rng, N, T, H, K, V)
    o, hT = oracle.simple_gla_fwd(q, k, v, g=g, initial_state=s0, output_final_state=True,
                                  lib_path=lib_path)
    state = s0.copy()
    for t in range(T):
        ot = oracle.simple_gla_decode_step(q[:, t], k[:, t], v[:, t], state, g=g[:, t],
                                           lib_path=lib_path)
        _close(ot, o[:, t])
    _close(state, hT)
    # per-head decay in decode
    gg = np.log(np.array([0.5, 0.9]))
    o2, h2 = oracle.simple_gla_fwd(q, k, v, g_gamma=gg, initial_state=s0, output_final_state=True,
                                   lib_path=lib_path)
    state = s0.copy()
    for t in range(T):
        ot = oracle.simple_gla_decode_step(q[:, t], k[:, t], v[:, t], state, g_gamma=gg,
                                           lib_path=lib_path)
        _close(ot, o2[:, t])
    _close(state, h2)


def pin_normalized_brute_force(lib_path=None):
    """The normalised variant against its definition written out for positive
    (feature-mapped) q, k: o_i = sum_j D_ij (q_i.k_j) v_j / sum_j D_ij (q_i.k_j), with
    the initial state's S and z entering both sums through the decay from the start."""
    rng = np.random.default_rng(11)
    B, T, H, K, V = 2, 23, 2, 3, 4
    q = np.abs(rng.standard_normal((B, T, H, K))) + 0.1
    k = np.abs(rng.standard_normal((B, T, H, K))) + 0.1
    v = rng.standard_normal((B, T, H, V))
    g = _logsigmoid(rng.standard_normal((B, T, H)))
    s0 = np.abs(rng.standard_normal((B, H, K, V + 1)))
    o, hT = oracle.simple_gla_normalized(q, k, v, g=g, initial_state=s0, output_final_state=True,
                                         lib_path=lib_path)
    for b in range(B):
        for h in range(H):
            a = g[b, :, h]
            for i in range(T):
                num = np.zeros(V)
                den = 0.0
                for j in range(i + 1):
                    w = math.exp(math.fsum(a[j + 1:i + 1])) * float(q[b, i, h] @ k[b, j, h])
                    num += w * v[b, j, h]
                    den += w
                lead = math.exp(math.fsum(a[:i + 1]))
                num += lead * (q[b, i, h] @ s0[b, h, :, :V])
                den += lead * float(q[b, i, h] @ s0[b, h, :, V])
                _close(o[b, i, h], num / den)
            zT = sum(math.exp(math.fsum(a[j + 1:])) * k[b, j, h] for j in range(T)) + \
                math.exp(math.fsum(a)) * s0[b, h, :, V]
            _close(hT[b, h, :, V], zT)


def _gla_brute_force_head(q, k, v, gk, scale, h0):
    """Parallel form of the vector-gate recurrence for one (sequence, head):
    o_t = scale sum_{j<=t} sum_i q_t[i] k_j[i] exp(sum_{l=j+1..t} gk_l[i]) v_j
          + scale sum_i q_t[i] exp(sum_{l<=t} gk_l[i]) h0[i]."""
    T, K = q.shape
    V = v.shape[1]
    o = np.zeros((T, V))
    for t in range(T):
        for j in range(t + 1):
            dec = np.array([math.exp(math.fsum(gk[j + 1:t + 1, i])) for i in range(K)])
            o[t] += scale * float(np.sum(q[t] * k[j] * dec)) * v[j]
        if h0 is not None:
            lead = np.array([math.exp(math.fsum(gk[:t + 1, i])) for i in range(K)])
            o[t] += scale * (q[t] * lead) @ h0
    ST = np.zeros((K, V))
    for j in range(T):
        dec = np.array([math.exp(math.fsum(gk[j + 1:, i])) for i in range(K)])
        ST += np.outer(dec * k[j], v[j])
    if h0 is not None:
        ST += np.array([math.exp(math.fsum(gk[:, i])) for i in range(K)])[:, None] * h0
    return o, ST


def pin_gla_brute_force(lib_path=None):
    rng = np.random.default_rng(13)
    for B, T, H, K, V, h0 in [(2, 17, 2, 3, 4, True), (1, 23, 1, 4, 2, False)]:
        q = rng.standard_normal((B, T, H, K))
        k = rng.standard_normal((B, T, H, K))
        v = rng.standard_normal((B, T, H, V))
        gk = _logsigmoid(rng.standard_normal((B, T, H, K)))
        s0 = 0.5 * rng.standard_normal((B, H, K, V)) if h0 else None
        o, hT = oracle.gla_fwd(q, k, v, gk, scale=0.7, initial_state=s0, output_final_state=True, lib_path=lib_path)
        for b in range(B):
            for h in range(H):
                ob, hb = _gla_brute_force_head(q[b, :, h], k[b, :, h], v[b, :, h], gk[b, :, h], 0.7,
                                               None if s0 is None else s0[b, h])
                _close(o[b, :, h], ob)
                _close(hT[b, h], hb)


def pin_gla_reduces_to_simple_gla(lib_path=None):
    """A gate vector with all K entries equal is the head-wise gate of Simple GLA."""
    rng = np.random.default_rng(17)
    q, k, v, g, _, s0 = _inputs(rng, 2, 29, 3, 4, 5, "g", 1.0, True)
    gk = np.repeat(g[..., None], 4, axis=-1)
    o1, h1 = oracle.gla_fwd(q, k, v, gk, initial_state=s0, output_final_state=True, lib_path=lib_path)
    o2, h2 = oracle.simple_gla_fwd(q, k, v, g=g, initial_state=s0, output_final_state=True, lib_path=lib_path)
    _close(o1, o2)
    _close(h1, h2)


def _fd_grad(f, x, eps=1e-6):
    """Central finite differences of the scalar f at every element of x (in place)."""
    gr = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        gr[i] = (fp - fm) / (2 * eps)
    return gr


def pin_backward_finite_differences(lib_path=None):
    """The reverse-mode backward against central finite differences of the forward
    for L = sum(o * do) + sum(hT * dhT), every input, per-token and per-head gates,
    dense and packed."""
    rng = np.random.default_rng(19)
    for gate, cu in (("g", None), ("gamma", None), ("g", np.array([0, 2, 2, 7]))):
        B, T, H, K, V = (1, 7, 2, 3, 2) if cu is not None else (2, 5, 2, 3, 2)
        q, k, v, g, gg, s0 = _inputs(rng, B, T, H, K, V, gate, 1.0, True)
        N = len(cu) - 1 if cu is not None else B
        s0 = 0.5 * rng.standard_normal((N, H, K, V))
        do = rng.standard_normal((B, T, H, V))
        dht = rng.standard_normal((N, H, K, V))

        def loss():
            o, hT = oracle.simple_gla_fwd(q, k, v, g=g, g_gamma=gg, scale=0.8, initial_state=s0,
                                          output_final_state=True, cu_seqlens=cu, lib_path=lib_path)
            return float(np.sum(o * do) + np.sum(hT * dht))
        grads = oracle.simple_gla_bwd(q, k, v, do, g=g, g_gamma=gg, scale=0.8, initial_state=s0, dht=dht,
                                      cu_seqlens=cu, lib_path=lib_path)
        for name, x in (("dq", q), ("dk", k), ("dv", v), ("dh0", s0)):
            _close(grads[name], _fd_grad(loss, x), 1e-6)
        if g is not None:
            _close(grads["dg"], _fd_grad(loss, g), 1e-6)
        else:
            _close(grads["dg_gamma"], _fd_grad(loss, gg), 1e-6)


def pin_linearity(lib_path=None):
    rng = np.random.default_rng(8)
    q, k, v, g, _, _ = _inputs(rng, 1, 30, 2, 3, 4, h0=False)
    f = lambda q_, k_, v_, s=None: oracle.simple_gla_fwd(q_, k_, v_, g=g, scale=s, lib_path=lib_path)[0]
    base = f(q, k, v)
    v2 = rng.standard_normal(v.shape)
    _close(f(q, k, v + 2.0 * v2), base + 2.0 * f(q, k, v2))
    q2 = rng.standard_normal(q.shape)
    _close(f(q - q2, k, v), base - f(q2, k, v))
    _close(f(q, 3.0 * k, v), 3.0 * base)
    _close(f(q, k, v, 1.0 / math.sqrt(3)), base)  # default scale is 1/sqrt(K)


PINS = [pin_golden, pin_brute_force_dense, pin_brute_force_varlen, pin_closed_form_no_decay,
        pin_special_cases, pin_split_invariant, pin_varlen_equals_separate,
        pin_decode_equals_forward, pin_linearity, pin_normalized_brute_force, pin_gla_brute_force,
        pin_gla_reduces_to_simple_gla, pin_backward_finite_differences]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin, oracle_lib):
    pin()


# Plausible mistakes, planted in a copy of the oracle source: each must fail a pin.
MUTATIONS = {
    "decay_dropped": ("decay * S[i * V + j] + kt[i] * vt[j]", "S[i * V + j] + kt[i] * vt[j]"),
    "gate_sign_flipped": ("const double decay = exp(a);", "const double decay = exp(-a);"),
    "outer_product_dropped": ("decay * S[i * V + j] + kt[i] * vt[j]", "decay * S[i * V + j]"),
    "gate_of_previous_token": ("a = g[t * H + h];", "a = g[(t > t_begin ? t - 1 : t) * H + h];"),
    "key_in_readout": ("acc += qt[i] * S[i * V + j];", "acc += kt[i] * S[i * V + j];"),
    "scale_dropped": ("ot[j] = scale * acc;", "ot[j] = acc;"),
    "initial_state_ignored": ("    if (h0)\n        memcpy", "    if (0)\n        memcpy"),
    "last_token_dropped": ("for (int64_t t = t_begin; t < t_end; ++t)",
                           "for (int64_t t = t_begin; t + 1 < t_end; ++t)"),
    "gamma_of_head_zero": ("a = g_gamma[h];", "a = g_gamma[0];"),
    "gla_gate_of_key_zero": ("const double row_decay = exp(gt[i]);", "const double row_decay = exp(gt[0]);"),
    "bwd_decay_of_current_token": ("                G[e] *= a[l + 1];", "                G[e] *= a[l];"),
    "bwd_dv_uses_query": ("                acc += G[i * V + j] * kt[i];", "                acc += G[i * V + j] * qt[i];"),
    "gla_outer_product_transposed": ("row_decay * S[i * V + j] + kt[i] * vt[j]",
                                     "row_decay * S[i * V + j] + kt[j % K] * vt[i % V]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    old, new = MUTATIONS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "simple_gla_oracle.c")).read()
    assert old in src, f"mutation anchor for {name} not found"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new, 1))
    lib = str(tmp_path / f"libmutant_{name}.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", lib,
                    str(mutant), "-lm"], check=True)
    failed = []
    for pin in PINS:
        try:
            pin(lib)
        except (AssertionError, RuntimeError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name} passed every pin"


# ----------------------------------------------------------------------------- randomised shapes

from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=60, deadline=None, derandomize=True)
@given(B=st.integers(1, 2), T=st.integers(0, 20), H=st.integers(1, 3), K=st.integers(1, 5), V=st.integers(1, 5),
       gate=st.sampled_from(["g", "gamma", "none"]), h0=st.booleans(),
       scale=st.sampled_from([None, 0.25, 1.0]), seed=st.integers(0, 2**16))
def test_oracle_equals_brute_force_on_random_shapes(B, T, H, K, V, gate, h0, scale, seed, oracle_lib):
    """The brute-force parallel form against the oracle over many small shapes,
    including T = 0 and one-element head dims."""
    rng = np.random.default_rng(seed)
    q, k, v, g, gg, s0 = _inputs(rng, B, T, H, K, V, gate, 1.0, h0)
    o, hT = oracle.simple_gla_fwd(q, k, v, g=g, g_gamma=gg, scale=scale, initial_state=s0,
                                  output_final_state=True, lib_path=oracle_lib)
    ob, hb = _brute_force(q, k, v, g, gg, scale, s0)
    _close(o, ob)
    _close(hT, hb)


@settings(max_examples=25, deadline=None, derandomize=True)
@given(B=st.integers(1, 2), T=st.integers(1, 6), H=st.integers(1, 2), K=st.integers(1, 3), V=st.integers(1, 3),
       gate=st.sampled_from(["g", "gamma"]), h0=st.booleans(), with_dht=st.booleans(), seed=st.integers(0, 2**16))
def test_oracle_backward_equals_finite_differences_on_random_shapes(B, T, H, K, V, gate, h0, with_dht, seed,
                                                                    oracle_lib):
    """Reverse mode against central finite differences of the forward over many
    small shapes, with and without an initial state and an output-state gradient."""
    rng = np.random.default_rng(seed)
    q, k, v, g, gg, s0 = _inputs(rng, B, T, H, K, V, gate, 1.0, h0)
    do = rng.standard_normal((B, T, H, V))
    dht = rng.standard_normal((B, H, K, V)) if with_dht else None

    def loss():
        o, hT = oracle.simple_gla_fwd(q, k, v, g=g, g_gamma=gg, scale=0.7, initial_state=s0,
                                      output_final_state=True, lib_path=oracle_lib)
        return float(np.sum(o * do) + (np.sum(hT * dht) if dht is not None else 0.0))
    r = oracle.simple_gla_bwd(q, k, v, do, g=g, g_gamma=gg, scale=0.7, initial_state=s0, dht=dht,
                              lib_path=oracle_lib)
    for name, x in (("dq", q), ("dk", k), ("dv", v)):
        _close(r[name], _fd_grad(loss, x), 1e-6)
    if s0 is not None:
        _close(r["dh0"], _fd_grad(loss, s0), 1e-6)
    else:
        assert r["dh0"] is None
    if g is not None:
        _close(r["dg"], _fd_grad(loss, g), 1e-6)
    else:
        _close(r["dg_gamma"], _fd_grad(loss, gg), 1e-6)


@settings(max_examples=40, deadline=None, derandomize=True)
@given(B=st.integers(1, 2), T=st.integers(0, 16), H=st.integers(1, 2), K=st.integers(1, 5), V=st.integers(1, 4),
       h0=st.booleans(), seed=st.integers(0, 2**16))
def test_gla_oracle_equals_brute_force_on_random_shapes(B, T, H, K, V, h0, seed, oracle_lib):
    """GLA's per-key-decay parallel form against the oracle over many small shapes."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, K))
    k = rng.standard_normal((B, T, H, K))
    v = rng.standard_normal((B, T, H, V))
    gk = _logsigmoid(rng.standard_normal((B, T, H, K)))
    s0 = 0.5 * rng.standard_normal((B, H, K, V)) if h0 else None
    o, hT = oracle.gla_fwd(q, k, v, gk, scale=0.6, initial_state=s0, output_final_state=True, lib_path=oracle_lib)
    for b in range(B):
        for h in range(H):
            ob, hb = _gla_brute_force_head(q[b, :, h], k[b, :, h], v[b, :, h], gk[b, :, h], 0.6,
                                           None if s0 is None else s0[b, h])
            _close(o[b, :, h], ob)
            _close(hT[b, h], hb)


@settings(max_examples=40, deadline=None, derandomize=True)
@given(lens=st.lists(st.integers(0, 9), min_size=1, max_size=4), H=st.integers(1, 2), K=st.integers(1, 4),
       V=st.integers(1, 4), gate=st.sampled_from(["g", "gamma", "none"]), h0=st.booleans(),
       seed=st.integers(0, 2**16))
def test_varlen_oracle_equals_brute_force_on_random_lengths(lens, H, K, V, gate, h0, seed, oracle_lib):
    """Packed sequences of random lengths (empty ones included) against the parallel
    form of each sequence on its own span."""
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    q, k, v, g, gg, _ = _inputs(rng, 1, int(cu[-1]), H, K, V, gate, 1.0, False)
    s0 = 0.5 * rng.standard_normal((len(lens), H, K, V)) if h0 else None
    o, hT = oracle.simple_gla_fwd(q, k, v, g=g, g_gamma=gg, initial_state=s0, output_final_state=True,
                                  cu_seqlens=cu, lib_path=oracle_lib)
    ob, hb = _brute_force(q, k, v, g, gg, None, s0, cu)
    _close(o, ob)
    _close(hT, hb)
