"""fp64 CPU oracle for Simple GLA -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or executes anything here, and this
package imports nothing from the product.

The arithmetic lives in ``simple_gla_oracle.c`` (plain C, fp64, one OpenMP task
per (sequence, head)); this module only compiles it, marshals arrays to
float64 and applies the API defaults of the page "Simple GLA in
flash-linear-attention: maths and kernels" (xxqk.cn article), section 2:
``scale`` defaults to 1/sqrt(K); ``g`` and ``g_gamma`` are mutually exclusive;
with ``cu_seqlens`` the batch dimension must be 1 and ``initial_state`` must
hold ``len(cu_seqlens) - 1`` states (ValueError otherwise).

Every function here is pinned by ``tests/test_oracle_pins.py`` against
brute force, closed forms and invariants; nothing is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "simple_gla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libsgla_oracle.so")
_libs = {}


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libsgla_oracle.so`` (gcc, -fopenmp)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load(lib_path=None):
    """Load (and cache) the compiled oracle; ``lib_path`` selects another build of
    the same source (the pin tests use it to check that planted mistakes fail)."""
    path = lib_path or build()
    if path not in _libs:
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.sgla_oracle_fwd.argtypes = [P, P, P, P, P, ctypes.c_double, P, P, P,
                                        P, I64, I64, I64, I64, I64, I64, ctypes.c_int]
        lib.sgla_oracle_fwd.restype = ctypes.c_int
        lib.sgla_oracle_decode_step.argtypes = [P, P, P, P, P, ctypes.c_double, P, P,
                                                I64, I64, I64, I64, ctypes.c_int]
        lib.sgla_oracle_decode_step.restype = ctypes.c_int
        lib.sgla_oracle_gla_fwd.argtypes = [P, P, P, P, ctypes.c_double, P, P, P,
                                            P, I64, I64, I64, I64, I64, I64, ctypes.c_int]
        lib.sgla_oracle_gla_fwd.restype = ctypes.c_int
        lib.sgla_oracle_bwd.argtypes = [P, P, P, P, P, ctypes.c_double, P, P, P, P, P, P, P, P, P,
                                        P, I64, I64, I64, I64, I64, I64]
        lib.sgla_oracle_bwd.restype = ctypes.c_int
        _libs[path] = lib
    return _libs[path]


def _f64(x):
    """Any array-like (numpy, torch CPU tensor of any float dtype) -> C-contiguous float64."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: widen exactly, then hand over
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def simple_gla_fwd(q, k, v, g=None, g_gamma=None, scale=None, initial_state=None,
                   output_final_state=False, cu_seqlens=None, threads=None, lib_path=None,
                   state_v_first=False):
    """fp64 naive recurrence.  q,k [B,T,H,K]; v [B,T,H,V]; g [B,T,H]; g_gamma [H];
    initial_state [N,H,K,V] -- [N,H,V,K] with state_v_first, the transposed state
    layout of section 2 of the article (the final state is returned in the same
    layout).  Returns (o [B,T,H,V] float64, final_state or None)."""
    q, k, v, g, g_gamma, h0 = map(_f64, (q, k, v, g, g_gamma, initial_state))
    if state_v_first and h0 is not None:
        if h0.ndim != 4:
            raise ValueError("initial_state must have 4 dimensions")
        h0 = np.ascontiguousarray(h0.transpose(0, 1, 3, 2))
    if g is not None and g_gamma is not None:
        raise ValueError("only one of g and g_gamma may be given")
    if q.ndim != 4 or k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("q,k must be [B,T,H,K] and v [B,T,H,V]")
    B, T, H, K = q.shape
    V = v.shape[3]
    if g is not None and g.shape != (B, T, H):
        raise ValueError("g must be [B,T,H]")
    if g_gamma is not None and g_gamma.shape != (H,):
        raise ValueError("g_gamma must be [H]")
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
        if B != 1:
            raise ValueError("with cu_seqlens the batch size must be 1")
        N = cu.shape[0] - 1
        if N < 1 or cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
            raise ValueError("cu_seqlens must be non-decreasing from 0 to T")
    else:
        N = B
    if h0 is not None and h0.shape != (N, H, K, V):
        raise ValueError(f"initial_state must be [{N},{H},{K},{V}], got {h0.shape}")
    if scale is None:
        scale = 1.0 / math.sqrt(K)
    o = np.zeros((B, T, H, V), dtype=np.float64)
    hT = np.zeros((N, H, K, V), dtype=np.float64) if output_final_state else None
    rc = _load(lib_path).sgla_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma),
                                 float(scale), _ptr(h0), _ptr(o), _ptr(hT),
                                 _ptr(cu), N, B, T, H, K, V,
                                 int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"sgla_oracle_fwd failed with code {rc}")
    if state_v_first and hT is not None:
        hT = np.ascontiguousarray(hT.transpose(0, 1, 3, 2))
    return o, hT


def simple_gla_decode_step(q, k, v, state, g=None, g_gamma=None, scale=None, threads=None,
                           lib_path=None):
    """One recurrent step for N sequences.  q,k [N,H,K]; v [N,H,V]; g [N,H];
    state [N,H,K,V] float64 numpy array, updated IN PLACE.  Returns o [N,H,V]."""
    q, k, v, g, g_gamma = map(_f64, (q, k, v, g, g_gamma))
    if g is not None and g_gamma is not None:
        raise ValueError("only one of g and g_gamma may be given")
    if not (isinstance(state, np.ndarray) and state.dtype == np.float64
            and state.flags["C_CONTIGUOUS"]):
        raise TypeError("state must be a C-contiguous float64 numpy array (updated in place)")
    N, H, K = q.shape
    V = v.shape[2]
    if state.shape != (N, H, K, V):
        raise ValueError("state must be [N,H,K,V]")
    if scale is None:
        scale = 1.0 / math.sqrt(K)
    o = np.zeros((N, H, V), dtype=np.float64)
    rc = _load(lib_path).sgla_oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma),
                                         float(scale), _ptr(state), _ptr(o), N, H, K, V,
                                         int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"sgla_oracle_decode_step failed with code {rc}")
    return o


def simple_gla_normalized(q, k, v, g=None, g_gamma=None, initial_state=None, output_final_state=False,
                          cu_seqlens=None, threads=None, lib_path=None):
    """Normalised variant, as "relinear" runs it through fla's kernel (fla-org kernel
    integration): append a column of ones to v, run the recurrence with scale 1 --
    the state's last column is then the normaliser z and the last output column is
    q.z -- and divide the other output columns by it.  initial_state and the final
    state are the augmented [N,H,K,V+1].  Returns (o [B,T,H,V] float64, final_state)."""
    v = _f64(v)
    ones = np.ones(v.shape[:-1] + (1,), dtype=np.float64)
    o_aug, hT = simple_gla_fwd(q, k, np.concatenate([v, ones], axis=-1), g=g, g_gamma=g_gamma, scale=1.0,
                               initial_state=initial_state, output_final_state=output_final_state,
                               cu_seqlens=cu_seqlens, threads=threads, lib_path=lib_path)
    with np.errstate(divide="ignore", invalid="ignore"):  # a zero q.z gives inf / NaN, as defined
        return o_aug[..., :-1] / o_aug[..., -1:], hT


def gla_fwd(q, k, v, gk, scale=None, initial_state=None, output_final_state=False, cu_seqlens=None,
            threads=None, lib_path=None):
    """fp64 recurrence of GLA with a gate vector over the key dimension (row i of the
    state decays by exp(gk_t[i])).  q,k,gk [B,T,H,K]; v [B,T,H,V]; initial_state
    [N,H,K,V].  Returns (o [B,T,H,V] float64, final_state or None)."""
    q, k, v, gk, h0 = map(_f64, (q, k, v, gk, initial_state))
    if q.ndim != 4 or k.shape != q.shape or gk.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("q,k,gk must be [B,T,H,K] and v [B,T,H,V]")
    B, T, H, K = q.shape
    V = v.shape[3]
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
        if B != 1:
            raise ValueError("with cu_seqlens the batch size must be 1")
        N = cu.shape[0] - 1
    else:
        N = B
    if h0 is not None and h0.shape != (N, H, K, V):
        raise ValueError(f"initial_state must be [{N},{H},{K},{V}]")
    if scale is None:
        scale = 1.0 / math.sqrt(K)
    o = np.zeros((B, T, H, V), dtype=np.float64)
    hT = np.zeros((N, H, K, V), dtype=np.float64) if output_final_state else None
    rc = _load(lib_path).sgla_oracle_gla_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(gk), float(scale), _ptr(h0),
                                             _ptr(o), _ptr(hT), _ptr(cu), N, B, T, H, K, V,
                                             int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"sgla_oracle_gla_fwd failed with code {rc}")
    return o, hT


def simple_gla_bwd(q, k, v, do, g=None, g_gamma=None, scale=None, initial_state=None, dht=None, cu_seqlens=None,
                   lib_path=None):
    """fp64 reverse-mode of the recurrence (section 3's gradients).  do [B,T,H,V]; dht
    [N,H,K,V] or None.  Returns dict(dq, dk, dv, dg [B,T,H] or None, dg_gamma [H] or
    None, dh0 [N,H,K,V] or None -- dh0 only when initial_state is given)."""
    q, k, v, do, g, g_gamma, h0, dht = map(_f64, (q, k, v, do, g, g_gamma, initial_state, dht))
    B, T, H, K = q.shape
    V = v.shape[3]
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
        N = cu.shape[0] - 1
    else:
        N = B
    if scale is None:
        scale = 1.0 / math.sqrt(K)
    out = dict(dq=np.zeros((B, T, H, K)), dk=np.zeros((B, T, H, K)), dv=np.zeros((B, T, H, V)),
               dg=np.zeros((B, T, H)) if g is not None else None,
               dg_gamma=np.zeros(H) if g_gamma is not None else None,
               dh0=np.zeros((N, H, K, V)) if h0 is not None else None)
    rc = _load(lib_path).sgla_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma), float(scale), _ptr(h0),
                                         _ptr(do), _ptr(dht), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                         _ptr(out["dg"]), _ptr(out["dg_gamma"]), _ptr(out["dh0"]), _ptr(cu),
                                         N, B, T, H, K, V)
    if rc != 0:
        raise RuntimeError(f"sgla_oracle_bwd failed with code {rc}")
    return out
