"""B200 (sm_100a) Simple GLA: Python binding of libsimplegla.so.

The operator is head-wise gated linear attention as stated in "Simple GLA in
flash-linear-attention: maths and kernels" (xxqk.cn article): per head
S_t = exp(g_t) S_{t-1} + k_t v_t^T and o_t = scale * q_t^T S_t (section 1), with
the chunk_simple_gla argument conventions of section 2 and the chunked kernels
of section 3.

This module only marshals arguments: it checks tensor types and shapes, takes
device memory (outputs, workspace) from PyTorch's caching allocator, passes raw
pointers and the current CUDA stream to the C ABI declared in
``include/simple_gla.h``, and maps status codes to exceptions.  Every step of the
computation runs in the library's CUDA kernels; there is no fallback of any kind
-- a missing library or a CPU tensor is an error.

Public functions (same names as the C entry points):
  simple_gla_fwd(q, k, v, g=None, g_gamma=None, scale=None, initial_state=None,
                 output_final_state=False, chunk_size=64) -> (o, final_state|None)
  simple_gla_fwd_varlen(q, k, v, cu_seqlens, g=None, ...) -> (o, final_state|None)
  simple_gla_decode_step(q, k, v, state, g=None, g_gamma=None, scale=None,
                         state_v_first=False) -> o
  simple_gla_fused_recurrent(q, k, v, g=None, g_gamma=None, scale=None, initial_state=None,
                             output_final_state=False, cu_seqlens=None,
                             state_v_first=False) -> (o, final_state|None)
  simple_gla_chunk(q, k, v, ..., cu_seqlens=None, chunk_size=64, state_v_first=False)
  simple_gla_normalized(q, k, v, ...) / simple_gla_normalized_decode_step(...) -- the
      normalised variant through the augmented value (states [.., K, V+1])
  gla_fused_recurrent(q, k, v, gk, ...) -- GLA with a gate vector over the key dimension
  chunk_simple_gla(...)  -- the article's entry-point name; dispatches on cu_seqlens, and
      is differentiable (ChunkSimpleGLAFunction) when an input requires gradients.
  simple_gla_chunk_bwd(...), simple_gla_fused_recurrent_bwd(...) -- the gradients.
  gla_chunk(q, k, v, gk, ...) -- GLA with a vector gate, chunked form.
  fused_recurrent_simple_gla(...) -- the article's name for simple_gla_fused_recurrent.
"""
from __future__ import annotations

import ctypes
import functools
import os

import torch

from . import _lib as _lib_mod
from ._lib import (SGLA_BF16, SGLA_FP32, SGLA_OK, SglaError, lib, library_path,  # noqa: F401
                   raise_for_status)

__all__ = ["simple_gla_fwd", "simple_gla_fwd_noalloc", "simple_gla_fwd_varlen", "simple_gla_decode_step", "chunk_simple_gla",
           "simple_gla_fused_recurrent", "fused_recurrent_simple_gla", "simple_gla_chunk",
           "simple_gla_normalized", "simple_gla_normalized_decode_step", "normalized_decode_state_width",
           "gla_fused_recurrent", "simple_gla_fused_recurrent_bwd", "simple_gla_chunk_bwd", "gla_chunk", "ChunkSimpleGLAFunction",
           "simple_gla_log_decay_total", "simple_gla_state_carry", "simple_gla_chunk_final_state",
           "simple_gla_chunk_plan",
           "fwd_workspace_size", "varlen_workspace_size", "workspace_status", "noalloc_status", "library_path",
           "SglaError"]

_DTYPES = {torch.bfloat16: SGLA_BF16, torch.float32: SGLA_FP32}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _on_tensor_device(fn):
    """Run ``fn`` with the CUDA device of its tensor arguments current.  The library
    launches on the calling thread's current device and on that device's current
    stream, so a call whose tensors live on another device than the current one
    switches to theirs first; tensors on two different devices are an error (the
    kernels read only memory local to the device they run on)."""
    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        dev = None
        for t in (*args, *kwargs.values()):
            if isinstance(t, torch.Tensor) and t.is_cuda:
                if dev is None:
                    dev = t.device
                elif t.device != dev:
                    raise ValueError(f"{fn.__name__}: tensors on {dev} and {t.device}; all must be on one device")
        if dev is None or dev.index == torch.cuda.current_device():
            return fn(*args, **kwargs)
        with torch.cuda.device(dev):
            return fn(*args, **kwargs)
    return wrapper


def _check_cuda(name, t, dtype=None, ndim=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")


def fwd_workspace_size(B, T, H, K, V, chunk_size=64, dtype=torch.bfloat16) -> int:
    return int(lib().simple_gla_fwd_workspace_size(B, T, H, K, V, chunk_size, _DTYPES[dtype]))


def varlen_workspace_size(N, T_total, H, K, V, chunk_size=64, dtype=torch.bfloat16) -> int:
    return int(lib().simple_gla_fwd_varlen_workspace_size(N, T_total, H, K, V, chunk_size, _DTYPES[dtype]))


def _workspace(nbytes, device, workspace):
    if workspace is not None:
        _check_cuda("workspace", workspace, torch.uint8)
        if workspace.numel() < nbytes:
            raise ValueError(f"workspace holds {workspace.numel()} bytes, {nbytes} needed")
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _common_checks(q, k, v, g, g_gamma, initial_state):
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_cuda(name, t)
    if q.dtype not in _DTYPES:
        raise TypeError(f"q,k,v must be bfloat16 or float32, got {q.dtype}")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k and v must share one dtype")
    if g is not None and g_gamma is not None:
        raise ValueError("only one of g and g_gamma may be provided")
    _check_cuda("g", g, torch.float32)
    _check_cuda("g_gamma", g_gamma, torch.float32, 1)
    _check_cuda("initial_state", initial_state, torch.float32, 4)


def _dense_shapes(q, k, v, g, g_gamma, initial_state):
    """Checks shared by the dense forwards; returns (B, T, H, K, V).  Every tensor the
    kernels index by these sizes is checked against them, so no mis-shaped argument
    reaches the device."""
    _common_checks(q, k, v, g, g_gamma, initial_state)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("q,k must be [B,T,H,K] and v [B,T,H,V]")
    B, T, H, K = q.shape
    V = v.shape[3]
    if g is not None and tuple(g.shape) != (B, T, H):
        raise ValueError(f"g must be [B,T,H] = {(B, T, H)}, got {tuple(g.shape)}")
    if g_gamma is not None and tuple(g_gamma.shape) != (H,):
        raise ValueError(f"g_gamma must be [H] = ({H},)")
    if initial_state is not None and tuple(initial_state.shape) != (B, H, K, V):
        raise ValueError(f"initial_state must be [B,H,K,V] = {(B, H, K, V)}")
    return B, T, H, K, V


@_on_tensor_device
def simple_gla_fwd(q, k, v, g=None, g_gamma=None, scale=None, initial_state=None,
                   output_final_state=False, chunk_size=64, workspace=None):
    """Dense chunked forward.  q,k [B,T,H,K]; v [B,T,H,V]; g [B,T,H] fp32 log gates or
    g_gamma [H]; initial_state [B,H,K,V] fp32.  Returns (o [B,T,H,V], final_state)."""
    B, T, H, K, V = _dense_shapes(q, k, v, g, g_gamma, initial_state)
    dt = _DTYPES[q.dtype]
    o = torch.empty((B, T, H, V), dtype=q.dtype, device=q.device)
    ht = torch.empty((B, H, K, V), dtype=torch.float32, device=q.device) if output_final_state else None
    nbytes = int(lib().simple_gla_fwd_workspace_size(B, T, H, K, V, chunk_size, dt))
    if nbytes == 0:
        raise_for_status(_size_status(K, V, chunk_size), "simple_gla_fwd")
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().simple_gla_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma),
                              ctypes.c_float(_scale(scale)), _ptr(initial_state), _ptr(o), _ptr(ht),
                              B, T, H, K, V, chunk_size, dt, _ptr(ws), ws.numel(), _stream())
    raise_for_status(st, "simple_gla_fwd")
    return o, ht


@_on_tensor_device
def simple_gla_fwd_noalloc(q, k, v, g=None, g_gamma=None, scale=None, initial_state=None,
                           output_final_state=False, chunk_size=64):
    """simple_gla_fwd using the library's built-in 16 MiB scratch instead of a
    workspace, for callers that must not allocate device memory.  Outputs are
    still allocated here (a caller that cannot allocate calls the C entry point
    with its own output buffers).  Calls that may overlap on the GPU race on the
    shared scratch; ``noalloc_status()`` reads the device status word the last call
    left in it."""
    B, T, H, K, V = _dense_shapes(q, k, v, g, g_gamma, initial_state)
    o = torch.empty((B, T, H, V), dtype=q.dtype, device=q.device)
    ht = torch.empty((B, H, K, V), dtype=torch.float32, device=q.device) if output_final_state else None
    st = lib().simple_gla_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma),
                                      ctypes.c_float(_scale(scale)), _ptr(initial_state), _ptr(o), _ptr(ht),
                                      B, T, H, K, V, chunk_size, _DTYPES[q.dtype], _stream())
    raise_for_status(st, "simple_gla_fwd_noalloc")
    return o, ht


@_on_tensor_device
def simple_gla_fwd_varlen(q, k, v, cu_seqlens, g=None, g_gamma=None, scale=None, initial_state=None,
                          output_final_state=False, chunk_size=64, workspace=None):
    """Packed variable-length forward.  q,k [1,T,H,K] or [T,H,K]; v likewise with V;
    cu_seqlens [N+1] int64 on the device; g [1,T,H] or [T,H]; initial_state [N,H,K,V]."""
    _common_checks(q, k, v, g, g_gamma, initial_state)
    _check_cuda("cu_seqlens", cu_seqlens, torch.int64, 1)
    if q.dim() == 4:
        if q.shape[0] != 1:
            raise ValueError("with cu_seqlens the batch size must be 1 (flatten the batch first)")
        q, k, v = q[0], k[0], v[0]
        g = g[0] if g is not None else None
        squeeze = True
    else:
        squeeze = False
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
        raise ValueError("q,k must be [T,H,K] and v [T,H,V] (or with a leading batch of 1)")
    T, H, K = q.shape
    V = v.shape[2]
    N = cu_seqlens.shape[0] - 1
    if N < 1:
        raise ValueError("cu_seqlens must hold at least two entries")
    if g is not None and tuple(g.shape) != (T, H):
        raise ValueError("g must be [T,H] (or [1,T,H])")
    if g_gamma is not None and tuple(g_gamma.shape) != (H,):
        raise ValueError("g_gamma must be [H]")
    if initial_state is not None and initial_state.shape[0] != N:
        raise ValueError(f"the number of initial states must equal len(cu_seqlens) - 1 = {N}, "
                         f"got {initial_state.shape[0]}")
    if initial_state is not None and tuple(initial_state.shape) != (N, H, K, V):
        raise ValueError(f"initial_state must be [N,H,K,V] = {(N, H, K, V)}")
    dt = _DTYPES[q.dtype]
    o = torch.empty((T, H, V), dtype=q.dtype, device=q.device)
    ht = torch.empty((N, H, K, V), dtype=torch.float32, device=q.device) if output_final_state else None
    nbytes = int(lib().simple_gla_fwd_varlen_workspace_size(N, T, H, K, V, chunk_size, dt))
    if nbytes == 0:
        raise_for_status(_size_status(K, V, chunk_size), "simple_gla_fwd_varlen")
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().simple_gla_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma),
                                     ctypes.c_float(_scale(scale)), _ptr(cu_seqlens), N, T,
                                     _ptr(initial_state), _ptr(o), _ptr(ht), H, K, V, chunk_size, dt,
                                     _ptr(ws), ws.numel(), _stream())
    raise_for_status(st, "simple_gla_fwd_varlen")
    return (o.unsqueeze(0) if squeeze else o), ht


@_on_tensor_device
def simple_gla_chunk(q, k, v, g=None, g_gamma=None, scale=None, initial_state=None, output_final_state=False,
                     cu_seqlens=None, chunk_size=64, state_v_first=False, workspace=None):
    """Chunked forward with every option in one call: dense q,k [B,T,H,K] (or packed
    [1,T,H,K] / [T,H,K] with cu_seqlens), states [N,H,K,V] or, with state_v_first,
    [N,H,V,K].  Returns (o shaped like v, final_state|None)."""
    _common_checks(q, k, v, g, g_gamma, None)
    _check_cuda("initial_state", initial_state, torch.float32, 4)
    squeeze = False
    if cu_seqlens is not None:
        _check_cuda("cu_seqlens", cu_seqlens, torch.int64, 1)
        if q.dim() == 4:
            if q.shape[0] != 1:
                raise ValueError("with cu_seqlens the batch size must be 1 (flatten the batch first)")
            squeeze = True
            q, k, v = q[0], k[0], v[0]
            g = g[0] if g is not None else None
        if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
            raise ValueError("q,k must be [T,H,K] and v [T,H,V] with cu_seqlens")
        N = cu_seqlens.shape[0] - 1
        if N < 1:
            raise ValueError("cu_seqlens must hold at least two entries")
        T, H, K = q.shape
        V = v.shape[2]
        if g is not None and tuple(g.shape) != (T, H):
            raise ValueError("g must be [T,H] (or [1,T,H])")
        if initial_state is not None and initial_state.shape[0] != N:
            raise ValueError(f"the number of initial states must equal len(cu_seqlens) - 1 = {N}, "
                             f"got {initial_state.shape[0]}")
    else:
        if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
            raise ValueError("q,k must be [B,T,H,K] and v [B,T,H,V]")
        N, T, H, K = q.shape
        V = v.shape[3]
        if g is not None and tuple(g.shape) != (N, T, H):
            raise ValueError(f"g must be [B,T,H] = {(N, T, H)}")
    if g_gamma is not None and tuple(g_gamma.shape) != (H,):
        raise ValueError("g_gamma must be [H]")
    sshape = (N, H, V, K) if state_v_first else (N, H, K, V)
    if initial_state is not None and tuple(initial_state.shape) != sshape:
        raise ValueError(f"initial_state must be {sshape}")
    dt = _DTYPES[q.dtype]
    vf = 1 if state_v_first else 0
    o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    ht = torch.empty(sshape, dtype=torch.float32, device=q.device) if output_final_state else None
    nbytes = int(lib().simple_gla_chunk_workspace_size(_ptr(cu_seqlens), N, T, H, K, V, chunk_size, vf, dt))
    if nbytes == 0:
        raise_for_status(_size_status(K, V, chunk_size), "simple_gla_chunk")
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().simple_gla_chunk(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma), ctypes.c_float(_scale(scale)),
                                _ptr(initial_state), _ptr(o), _ptr(ht), _ptr(cu_seqlens), N, T, H, K, V, chunk_size,
                                vf, dt, _ptr(ws), ws.numel(), _stream())
    raise_for_status(st, "simple_gla_chunk")
    return (o.unsqueeze(0) if squeeze else o), ht


@_on_tensor_device
def simple_gla_chunk_plan(N, T, H, K, V, varlen=False, chunk_size=64, per_token_gate=True, state_v_first=False,
                          dtype=torch.bfloat16):
    """The plan a chunked forward makes for these sizes (host only, no device needed):
    {"tensor_cores", "step_tokens", "segment_steps", "max_segments", "workspace_bytes"}.
    varlen: N packed sequences in T tokens, else N sequences of T tokens."""
    if dtype not in _DTYPES:
        raise TypeError("dtype must be torch.bfloat16 or torch.float32")
    out = _lib_mod.ChunkPlan()
    st = lib().simple_gla_chunk_plan(int(bool(varlen)), int(N), int(T), int(H), int(K), int(V), int(chunk_size),
                                     int(bool(per_token_gate)), int(bool(state_v_first)), _DTYPES[dtype],
                                     ctypes.byref(out))
    raise_for_status(st, "simple_gla_chunk_plan")
    return {"tensor_cores": bool(out.tensor_cores), "step_tokens": out.step_tokens,
            "segment_steps": out.segment_steps, "max_segments": out.max_segments,
            "workspace_bytes": out.workspace_bytes}


def simple_gla_chunk_final_state(k, v, g=None, g_gamma=None, initial_state=None, cu_seqlens=None, chunk_size=64,
                                 workspace=None):
    """The final state of the chunked forward without its output (the state pass of
    section 3 alone): k [B,T,H,K], v [B,T,H,V] (or packed [1,T,H,*] / [T,H,*] with
    cu_seqlens), g [B,T,H] or g_gamma [H].  Returns final_state [N,H,K,V] fp32."""
    _common_checks(k, k, v, g, g_gamma, initial_state)
    if cu_seqlens is not None:
        _check_cuda("cu_seqlens", cu_seqlens, torch.int64, 1)
        if k.dim() == 4:
            if k.shape[0] != 1:
                raise ValueError("with cu_seqlens the batch size must be 1 (flatten the batch first)")
            k, v = k[0], v[0]
            g = g[0] if g is not None else None
        if k.dim() != 3 or v.dim() != 3 or v.shape[:2] != k.shape[:2]:
            raise ValueError("k must be [T,H,K] and v [T,H,V] with cu_seqlens")
        N = cu_seqlens.shape[0] - 1
        if N < 1:
            raise ValueError("cu_seqlens must hold at least two entries")
        T, H, K = k.shape
        V = v.shape[2]
        if g is not None and tuple(g.shape) != (T, H):
            raise ValueError("g must be [T,H] (or [1,T,H])")
    else:
        if k.dim() != 4 or v.dim() != 4 or v.shape[:3] != k.shape[:3]:
            raise ValueError("k must be [B,T,H,K] and v [B,T,H,V]")
        N, T, H, K = k.shape
        V = v.shape[3]
        if g is not None and tuple(g.shape) != (N, T, H):
            raise ValueError(f"g must be [B,T,H] = {(N, T, H)}")
    if g_gamma is not None and tuple(g_gamma.shape) != (H,):
        raise ValueError("g_gamma must be [H]")
    if initial_state is not None and tuple(initial_state.shape) != (N, H, K, V):
        raise ValueError(f"initial_state must be {(N, H, K, V)}")
    dt = _DTYPES[k.dtype]
    ht = torch.empty((N, H, K, V), dtype=torch.float32, device=k.device)
    nbytes = int(lib().simple_gla_chunk_final_state_workspace_size(_ptr(cu_seqlens), N, T, H, K, V, chunk_size, dt))
    if nbytes == 0:
        raise_for_status(_size_status(K, V, chunk_size), "simple_gla_chunk_final_state")
    ws = _workspace(nbytes, k.device, workspace)
    st = lib().simple_gla_chunk_final_state(_ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma), _ptr(initial_state), _ptr(ht),
                                            _ptr(cu_seqlens), N, T, H, K, V, chunk_size, dt, _ptr(ws), ws.numel(),
                                            _stream())
    raise_for_status(st, "simple_gla_chunk_final_state")
    return ht


class ChunkSimpleGLAFunction(torch.autograd.Function):
    """Differentiable chunked forward (the article's section 3: the training path is
    an autograd function whose backward recovers dq, dk, dv, dg and dh0).  Forward:
    simple_gla_chunk; backward: simple_gla_chunk_bwd on the saved inputs (the state
    trajectory is recomputed, not stored).  Argument marshalling only."""

    @staticmethod
    def forward(ctx, q, k, v, g, g_gamma, initial_state, scale, output_final_state, cu_seqlens, chunk_size,
                state_v_first):
        o, ht = simple_gla_chunk(q, k, v, g, g_gamma, scale, initial_state, output_final_state, cu_seqlens,
                                 chunk_size, state_v_first)
        ctx.save_for_backward(q, k, v, g, g_gamma, initial_state, cu_seqlens)
        ctx.opts = (scale, chunk_size, state_v_first)
        return o, ht

    @staticmethod
    def backward(ctx, do, dht):
        q, k, v, g, g_gamma, h0, cu = ctx.saved_tensors
        scale, chunk_size, vf = ctx.opts
        r = simple_gla_chunk_bwd(q, k, v, do.contiguous(), g=g, g_gamma=g_gamma, scale=scale, initial_state=h0,
                                 dht=None if dht is None else dht.contiguous(), cu_seqlens=cu,
                                 chunk_size=chunk_size, state_v_first=vf)
        return r["dq"], r["dk"], r["dv"], r["dg"], r["dg_gamma"], r["dh0"], None, None, None, None, None


@_on_tensor_device
def chunk_simple_gla(q, k, v, g=None, g_gamma=None, scale=None, initial_state=None,
                     output_final_state=False, cu_seqlens=None, chunk_size=64, state_v_first=False):
    """The article's entry-point name (section 2): dense, or packed when cu_seqlens is
    given; state_v_first selects the [N,H,V,K] state layout.  When gradients are
    enabled and an input requires them, the call is differentiable (backward through
    simple_gla_chunk_bwd)."""
    if torch.is_grad_enabled() and any(t is not None and t.requires_grad
                                       for t in (q, k, v, g, g_gamma, initial_state)):
        return ChunkSimpleGLAFunction.apply(q, k, v, g, g_gamma, initial_state, scale, output_final_state,
                                            cu_seqlens, chunk_size, state_v_first)
    if state_v_first:
        return simple_gla_chunk(q, k, v, g, g_gamma, scale, initial_state, output_final_state, cu_seqlens,
                                chunk_size, state_v_first=True)
    if cu_seqlens is None:
        return simple_gla_fwd(q, k, v, g, g_gamma, scale, initial_state, output_final_state, chunk_size)
    return simple_gla_fwd_varlen(q, k, v, cu_seqlens, g, g_gamma, scale, initial_state,
                                 output_final_state, chunk_size)


@_on_tensor_device
def simple_gla_decode_step(q, k, v, state, g=None, g_gamma=None, scale=None, out=None, state_v_first=False):
    """One recurrent step.  q,k [N,H,K]; v [N,H,V]; g [N,H] fp32 or g_gamma [H];
    state [N,H,K,V] fp32 ([N,H,V,K] with state_v_first) updated in place.  Returns
    o [N,H,V].  The [V,K] layout runs as a one-token simple_gla_fused_recurrent."""
    _common_checks(q, k, v, g, g_gamma, None)
    _check_cuda("state", state, torch.float32, 4)
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
        raise ValueError("q,k must be [N,H,K] and v [N,H,V]")
    N, H, K = q.shape
    V = v.shape[2]
    want = (N, H, V, K) if state_v_first else (N, H, K, V)
    if tuple(state.shape) != want:
        raise ValueError(f"state must be {'[N,H,V,K]' if state_v_first else '[N,H,K,V]'} = {want}")
    if g is not None and tuple(g.shape) != (N, H):
        raise ValueError("g must be [N,H]")
    if g_gamma is not None and tuple(g_gamma.shape) != (H,):
        raise ValueError("g_gamma must be [H]")
    o = out if out is not None else torch.empty((N, H, V), dtype=q.dtype, device=q.device)
    _check_cuda("out", o, q.dtype, 3)
    if state_v_first:
        st = lib().simple_gla_fused_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma),
                                              ctypes.c_float(_scale(scale)), _ptr(state), _ptr(o), _ptr(state),
                                              None, N, 1, H, K, V, 1, _DTYPES[q.dtype], None, _stream())
        raise_for_status(st, "simple_gla_fused_recurrent")
        return o
    st = lib().simple_gla_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma),
                                      ctypes.c_float(_scale(scale)), _ptr(state), _ptr(o), N, H, K, V,
                                      _DTYPES[q.dtype], _stream())
    raise_for_status(st, "simple_gla_decode_step")
    return o


@_on_tensor_device
def simple_gla_fused_recurrent(q, k, v, g=None, g_gamma=None, scale=None, initial_state=None,
                               output_final_state=False, cu_seqlens=None, state_v_first=False,
                               device_status=None):
    """Token-serial recurrence with the state held on chip for the whole sequence.

    Dense: q,k [B,T,H,K], v [B,T,H,V], g [B,T,H].  Packed (cu_seqlens int64 [N+1] on
    the device): q,k [1,T,H,K] or [T,H,K] and likewise v, g.  initial_state /
    final_state [N,H,K,V] fp32, [N,H,V,K] with state_v_first.  device_status: optional
    int32 CUDA tensor of one element that receives the cu_seqlens check.
    Returns (o shaped like v, final_state|None)."""
    _common_checks(q, k, v, g, g_gamma, None)
    _check_cuda("initial_state", initial_state, torch.float32, 4)
    squeeze = False
    if cu_seqlens is not None:
        _check_cuda("cu_seqlens", cu_seqlens, torch.int64, 1)
        if q.dim() == 4:
            if q.shape[0] != 1:
                raise ValueError("with cu_seqlens the batch dimension must be 1")
            squeeze = True
            q, k, v = q[0], k[0], v[0]
            g = g[0] if g is not None else None
        if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
            raise ValueError("q,k must be [T,H,K] and v [T,H,V] with cu_seqlens")
        N = cu_seqlens.numel() - 1
        if N < 1:
            raise ValueError("cu_seqlens needs at least two entries")
        T, H, K = q.shape
        V = v.shape[2]
        if g is not None and tuple(g.shape) != (T, H):
            raise ValueError(f"g must be [T,H] = {(T, H)}")
    else:
        if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
            raise ValueError("q,k must be [B,T,H,K] and v [B,T,H,V]")
        N, T, H, K = q.shape
        V = v.shape[3]
        if g is not None and tuple(g.shape) != (N, T, H):
            raise ValueError(f"g must be [B,T,H] = {(N, T, H)}")
    if g_gamma is not None and tuple(g_gamma.shape) != (H,):
        raise ValueError(f"g_gamma must be [H] = ({H},)")
    sshape = (N, H, V, K) if state_v_first else (N, H, K, V)
    if initial_state is not None and tuple(initial_state.shape) != sshape:
        raise ValueError(f"initial_state must be {sshape}")
    if device_status is not None:
        _check_cuda("device_status", device_status, torch.int32)
    o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    ht = torch.empty(sshape, dtype=torch.float32, device=q.device) if output_final_state else None
    st = lib().simple_gla_fused_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma),
                                          ctypes.c_float(_scale(scale)), _ptr(initial_state), _ptr(o), _ptr(ht),
                                          _ptr(cu_seqlens), N, T, H, K, V, 1 if state_v_first else 0,
                                          _DTYPES[q.dtype], _ptr(device_status), _stream())
    raise_for_status(st, "simple_gla_fused_recurrent")
    return (o.unsqueeze(0) if squeeze else o), ht


def _bwd_prepare(q, k, v, do, g, g_gamma, initial_state, dht, cu_seqlens, state_v_first=False):
    """Checks shared by the two backward entry points; returns (N, T, H, K, V) and the
    output tensors."""
    _common_checks(q, k, v, g, g_gamma, initial_state)
    _check_cuda("do", do, q.dtype)
    _check_cuda("dht", dht, torch.float32, 4)
    if do.shape != v.shape:
        raise ValueError(f"do must have the shape of v {tuple(v.shape)}")
    if cu_seqlens is not None:
        _check_cuda("cu_seqlens", cu_seqlens, torch.int64, 1)
        N = cu_seqlens.numel() - 1
        if N < 1:
            raise ValueError("cu_seqlens needs at least two entries")
        if q.dim() == 4 and q.shape[0] != 1:
            raise ValueError("with cu_seqlens the batch dimension must be 1")
        if q.dim() not in (3, 4):
            raise ValueError("q must be [1,T,H,K] or [T,H,K] with cu_seqlens")
        T, H, K = q.shape[-3:]
        if g is not None and g.numel() != T * H:
            raise ValueError(f"g must hold [T,H] = {(T, H)} values")
    else:
        if q.dim() != 4:
            raise ValueError("q must be [B,T,H,K]")
        N, T, H, K = q.shape
        if g is not None and tuple(g.shape) != (N, T, H):
            raise ValueError(f"g must be [B,T,H] = {(N, T, H)}")
    V = v.shape[-1]
    if k.shape != q.shape or v.shape[:-1] != q.shape[:-1]:
        raise ValueError("k must match q, and v must match q except in the last dimension")
    if g_gamma is not None and tuple(g_gamma.shape) != (H,):
        raise ValueError(f"g_gamma must be [H] = ({H},)")
    sshape = (N, H, V, K) if state_v_first else (N, H, K, V)
    for name, t in (("initial_state", initial_state), ("dht", dht)):
        if t is not None and tuple(t.shape) != sshape:
            raise ValueError(f"{name} must be {sshape}")
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               dg=torch.zeros_like(g) if g is not None else None,
               dg_gamma=torch.empty_like(g_gamma) if g_gamma is not None else None,
               dh0=torch.empty_like(initial_state) if initial_state is not None else None)
    return (N, T, H, K, V), out


@_on_tensor_device
def simple_gla_fused_recurrent_bwd(q, k, v, do, g=None, g_gamma=None, scale=None, initial_state=None, dht=None,
                                   cu_seqlens=None, state_v_first=False, workspace=None):
    """Gradients of simple_gla_fused_recurrent for the loss
    sum(o * do) + sum(final_state * dht).  Shapes as the forward; do like v; dht like
    the final state or None.  Returns dict(dq, dk, dv, dg, dg_gamma, dh0): dq, dk, dv
    in the dtype and shape of q, k, v; dg like g (None without g); dg_gamma [H] (None
    without g_gamma); dh0 like initial_state (None without it).  state_v_first: the
    states and their gradients are [N,H,V,K]."""
    (N, T, H, K, V), out = _bwd_prepare(q, k, v, do, g, g_gamma, initial_state, dht, cu_seqlens, state_v_first)
    nbytes = int(lib().simple_gla_fused_recurrent_bwd_workspace_size(_ptr(cu_seqlens), N, T, H, K))
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().simple_gla_fused_recurrent_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma), ctypes.c_float(_scale(scale)), _ptr(initial_state),
        _ptr(do), _ptr(dht), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dg_gamma"]),
        _ptr(out["dh0"]), _ptr(cu_seqlens), N, T, H, K, V, 1 if state_v_first else 0, _DTYPES[q.dtype], _ptr(ws),
        ws.numel(), _stream())
    raise_for_status(st, "simple_gla_fused_recurrent_bwd")
    return out


@_on_tensor_device
def simple_gla_chunk_bwd(q, k, v, do, g=None, g_gamma=None, scale=None, initial_state=None, dht=None,
                         cu_seqlens=None, chunk_size=64, state_v_first=False, workspace=None):
    """Gradients of simple_gla_chunk on the tensor-core path, for
    the loss sum(o * do) + sum(final_state * dht).  Arguments and result as
    simple_gla_fused_recurrent_bwd, plus chunk_size."""
    (N, T, H, K, V), out = _bwd_prepare(q, k, v, do, g, g_gamma, initial_state, dht, cu_seqlens, state_v_first)
    dt = _DTYPES[q.dtype]
    nbytes = int(lib().simple_gla_chunk_bwd_workspace_size(_ptr(cu_seqlens), N, T, H, K, V, chunk_size, dt))
    if nbytes == 0:
        raise_for_status(_size_status(K, V, chunk_size), "simple_gla_chunk_bwd")
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().simple_gla_chunk_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma), ctypes.c_float(_scale(scale)), _ptr(initial_state),
        _ptr(do), _ptr(dht), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dg_gamma"]),
        _ptr(out["dh0"]), _ptr(cu_seqlens), N, T, H, K, V, chunk_size, 1 if state_v_first else 0, dt, _ptr(ws),
        ws.numel(), _stream())
    raise_for_status(st, "simple_gla_chunk_bwd")
    return out


@_on_tensor_device
def simple_gla_normalized(q, k, v, g=None, g_gamma=None, initial_state=None, output_final_state=False,
                          cu_seqlens=None, chunk_size=64, workspace=None):
    """Normalised variant (augmented value, scale 1): o = (q^T S) / (q^T z).  Shapes as
    simple_gla_chunk; states are the augmented [N,H,K,V+1] (last column z).
    Returns (o shaped like v, final_state|None)."""
    _common_checks(q, k, v, g, g_gamma, None)
    _check_cuda("initial_state", initial_state, torch.float32, 4)
    squeeze = False
    if cu_seqlens is not None:
        _check_cuda("cu_seqlens", cu_seqlens, torch.int64, 1)
        if q.dim() == 4:
            if q.shape[0] != 1:
                raise ValueError("with cu_seqlens the batch size must be 1 (flatten the batch first)")
            squeeze = True
            q, k, v = q[0], k[0], v[0]
            g = g[0] if g is not None else None
        if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
            raise ValueError("q,k must be [T,H,K] and v [T,H,V] with cu_seqlens")
        N = cu_seqlens.shape[0] - 1
        T, H, K = q.shape
        V = v.shape[2]
    else:
        if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
            raise ValueError("q,k must be [B,T,H,K] and v [B,T,H,V]")
        N, T, H, K = q.shape
        V = v.shape[3]
    sshape = (N, H, K, V + 1)
    if initial_state is not None and tuple(initial_state.shape) != sshape:
        raise ValueError(f"initial_state must be the augmented state {sshape}")
    dt = _DTYPES[q.dtype]
    o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    ht = torch.empty(sshape, dtype=torch.float32, device=q.device) if output_final_state else None
    nbytes = int(lib().simple_gla_normalized_workspace_size(_ptr(cu_seqlens), N, T, H, K, V, chunk_size, dt))
    if nbytes == 0:
        raise_for_status(_size_status(K, V + 1, chunk_size), "simple_gla_normalized")
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().simple_gla_normalized(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma), _ptr(initial_state), _ptr(o),
                                     _ptr(ht), _ptr(cu_seqlens), N, T, H, K, V, chunk_size, dt, _ptr(ws), ws.numel(),
                                     _stream())
    raise_for_status(st, "simple_gla_normalized")
    return (o.unsqueeze(0) if squeeze else o), ht


def normalized_decode_state_width(V: int) -> int:
    """Columns of the augmented decode state: V + 1 rounded up to a multiple of 4."""
    return (V + 1 + 3) // 4 * 4


@_on_tensor_device
def simple_gla_normalized_decode_step(q, k, v, state, g=None, g_gamma=None, out=None, workspace=None):
    """One token of the normalised variant, in place on the augmented state
    [N,H,K,normalized_decode_state_width(V)] fp32 (column V is z, later ones stay 0)."""
    _common_checks(q, k, v, g, g_gamma, None)
    _check_cuda("state", state, torch.float32, 4)
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
        raise ValueError("q,k must be [N,H,K] and v [N,H,V]")
    N, H, K = q.shape
    V = v.shape[2]
    want = (N, H, K, normalized_decode_state_width(V))
    if tuple(state.shape) != want:
        raise ValueError(f"state must be {want}")
    dt = _DTYPES[q.dtype]
    o = out if out is not None else torch.empty((N, H, V), dtype=q.dtype, device=q.device)
    _check_cuda("out", o, q.dtype, 3)
    nbytes = int(lib().simple_gla_normalized_decode_workspace_size(N, H, V, dt))
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().simple_gla_normalized_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(g_gamma), _ptr(state),
                                                 _ptr(o), N, H, K, V, dt, _ptr(ws), ws.numel(), _stream())
    raise_for_status(st, "simple_gla_normalized_decode_step")
    return o


@_on_tensor_device
def gla_fused_recurrent(q, k, v, gk, scale=None, initial_state=None, output_final_state=False, cu_seqlens=None,
                        state_v_first=False, device_status=None):
    """GLA (gate vector over the key dimension), token-serial: gk fp32 log gates shaped
    like q.  Other arguments and shapes as simple_gla_fused_recurrent."""
    _common_checks(q, k, v, None, None, None)
    _check_cuda("gk", gk, torch.float32)
    _check_cuda("initial_state", initial_state, torch.float32, 4)
    if tuple(gk.shape) != tuple(q.shape):
        raise ValueError(f"gk must be shaped like q {tuple(q.shape)}, got {tuple(gk.shape)}")
    squeeze = False
    if cu_seqlens is not None:
        _check_cuda("cu_seqlens", cu_seqlens, torch.int64, 1)
        if q.dim() == 4:
            if q.shape[0] != 1:
                raise ValueError("with cu_seqlens the batch dimension must be 1")
            squeeze = True
            q, k, v, gk = q[0], k[0], v[0], gk[0]
        N = cu_seqlens.numel() - 1
        T, H, K = q.shape
        V = v.shape[2]
    else:
        if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
            raise ValueError("q,k must be [B,T,H,K] and v [B,T,H,V]")
        N, T, H, K = q.shape
        V = v.shape[3]
    sshape = (N, H, V, K) if state_v_first else (N, H, K, V)
    if initial_state is not None and tuple(initial_state.shape) != sshape:
        raise ValueError(f"initial_state must be {sshape}")
    if device_status is not None:
        _check_cuda("device_status", device_status, torch.int32)
    o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    ht = torch.empty(sshape, dtype=torch.float32, device=q.device) if output_final_state else None
    st = lib().gla_fused_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(gk), ctypes.c_float(_scale(scale)),
                                   _ptr(initial_state), _ptr(o), _ptr(ht), _ptr(cu_seqlens), N, T, H, K, V,
                                   1 if state_v_first else 0, _DTYPES[q.dtype], _ptr(device_status), _stream())
    raise_for_status(st, "gla_fused_recurrent")
    return (o.unsqueeze(0) if squeeze else o), ht


@_on_tensor_device
def gla_chunk(q, k, v, gk, scale=None, initial_state=None, output_final_state=False, cu_seqlens=None,
              workspace=None):
    """GLA (gate vector over the key dimension) in the chunked form: gk fp32 log gates
    shaped like q.  Dense q,k [B,T,H,K], v [B,T,H,V]; packed (cu_seqlens) [1,T,...] or
    [T,...].  States [N,H,K,V] fp32.  Returns (o shaped like v, final_state|None)."""
    _common_checks(q, k, v, None, None, initial_state)
    _check_cuda("gk", gk, torch.float32)
    if tuple(gk.shape) != tuple(q.shape):
        raise ValueError(f"gk must be shaped like q {tuple(q.shape)}, got {tuple(gk.shape)}")
    if cu_seqlens is not None:
        _check_cuda("cu_seqlens", cu_seqlens, torch.int64, 1)
        if q.dim() == 4 and q.shape[0] != 1:
            raise ValueError("with cu_seqlens the batch dimension must be 1")
        N = cu_seqlens.numel() - 1
        if N < 1:
            raise ValueError("cu_seqlens needs at least two entries")
        T, H, K = q.shape[-3:]
    else:
        if q.dim() != 4:
            raise ValueError("q must be [B,T,H,K]")
        N, T, H, K = q.shape
    V = v.shape[-1]
    if k.shape != q.shape or v.shape[:-1] != q.shape[:-1]:
        raise ValueError("k must match q, and v must match q except in the last dimension")
    if initial_state is not None and tuple(initial_state.shape) != (N, H, K, V):
        raise ValueError(f"initial_state must be {(N, H, K, V)}")
    dt = _DTYPES[q.dtype]
    nbytes = int(lib().gla_chunk_workspace_size(_ptr(cu_seqlens), N, T, H, K, V, dt))
    if nbytes == 0:
        raise SglaError(2, "gla_chunk: unsupported sizes (K <= 256, V <= 4096)")
    ws = _workspace(nbytes, q.device, workspace)
    o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    ht = torch.empty((N, H, K, V), dtype=torch.float32, device=q.device) if output_final_state else None
    st = lib().gla_chunk(_ptr(q), _ptr(k), _ptr(v), _ptr(gk), ctypes.c_float(_scale(scale)), _ptr(initial_state),
                         _ptr(o), _ptr(ht), _ptr(cu_seqlens), N, T, H, K, V, dt, _ptr(ws), ws.numel(), _stream())
    raise_for_status(st, "gla_chunk")
    return o, ht


@_on_tensor_device
def simple_gla_log_decay_total(g=None, g_gamma=None, T=None, H=None):
    """Total log decay per head of one slice: sum over its tokens of g [T,H] (or
    [1,T,H]), or T * g_gamma, or 0.  Returns a fp32 [H] CUDA tensor."""
    _check_cuda("g", g, torch.float32)
    _check_cuda("g_gamma", g_gamma, torch.float32, 1)
    if g is not None:
        T, H = g.shape[-2], g.shape[-1]
        dev = g.device
    elif g_gamma is not None:
        H = g_gamma.shape[0]
        dev = g_gamma.device
    else:
        dev = torch.device("cuda", torch.cuda.current_device())
    out = torch.empty(H, dtype=torch.float32, device=dev)
    st = lib().simple_gla_log_decay_total(_ptr(g), _ptr(g_gamma), int(T or 0), int(H), _ptr(out), _stream())
    raise_for_status(st, "simple_gla_log_decay_total")
    return out


@_on_tensor_device
def simple_gla_state_carry(log_decay, states, initial_state=None, rank=0):
    """State entering rank `rank`'s slice: the fold of the summaries of ranks
    0 .. rank-1 (log_decay [G,H], states [G,H,K,V] fp32) onto initial_state [H,K,V]
    (None = 0).  Returns a fp32 [H,K,V] CUDA tensor."""
    _check_cuda("log_decay", log_decay, torch.float32, 2)
    _check_cuda("states", states, torch.float32, 4)
    _check_cuda("initial_state", initial_state, torch.float32, 3)
    G, H, K, V = states.shape
    if tuple(log_decay.shape) != (G, H):
        raise ValueError(f"log_decay must be [G,H] = {(G, H)}, got {tuple(log_decay.shape)}")
    if initial_state is not None and tuple(initial_state.shape) != (H, K, V):
        raise ValueError(f"initial_state must be [H,K,V] = {(H, K, V)}, got {tuple(initial_state.shape)}")
    if not 0 <= int(rank) <= G:
        raise ValueError(f"rank must be in [0, {G}], got {rank}")
    out = torch.empty((H, K, V), dtype=torch.float32, device=states.device)
    st = lib().simple_gla_state_carry(_ptr(log_decay), _ptr(states), _ptr(initial_state), _ptr(out), int(rank), H, K,
                                      V, _stream())
    raise_for_status(st, "simple_gla_state_carry")
    return out


def fused_recurrent_simple_gla(q, k, v, g=None, g_gamma=None, scale=None, initial_state=None,
                               output_final_state=False, cu_seqlens=None, state_v_first=False):
    """The article's name (section 2) for simple_gla_fused_recurrent."""
    return simple_gla_fused_recurrent(q, k, v, g=g, g_gamma=g_gamma, scale=scale, initial_state=initial_state,
                                      output_final_state=output_final_state, cu_seqlens=cu_seqlens,
                                      state_v_first=state_v_first)


def noalloc_status() -> int:
    """Device status word the last simple_gla_fwd_noalloc call on the current device
    left in the library's built-in scratch (synchronises the current stream)."""
    out = ctypes.c_int(-1)
    raise_for_status(lib().sgla_noalloc_status(ctypes.byref(out), _stream()), "sgla_noalloc_status")
    return out.value


@_on_tensor_device
def workspace_status(workspace) -> int:
    """Device status word of the last forward that used ``workspace`` (synchronises)."""
    out = ctypes.c_int(-1)
    raise_for_status(lib().sgla_workspace_status(_ptr(workspace), ctypes.byref(out), _stream()),
                     "sgla_workspace_status")
    return out.value


def _scale(scale):
    return float("nan") if scale is None else float(scale)


def _size_status(K, V, chunk_size):
    # mirrors the library's size rules only to pick the exception type for a zero
    # workspace query; the library itself decides by returning 0
    if chunk_size <= 0 or chunk_size & (chunk_size - 1):
        return 1
    return 2
