"""ctypes loader for libsimplegla.so (the C ABI in include/simple_gla.h).

The library is built in-tree (``gated_linear_attention_local_b200/build.py``).  If
it is missing, every call raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libsimplegla.so")

SGLA_OK = 0
SGLA_ERR_INVALID_ARGUMENT = 1
SGLA_ERR_UNSUPPORTED = 2
SGLA_ERR_CUDA = 3
SGLA_ERR_WORKSPACE = 4
SGLA_ERR_DEVICE_CHECK = 5
SGLA_BF16 = 0
SGLA_FP32 = 1

# every symbol include/simple_gla.h declares, with its ctypes signature
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SIG = {
    "sgla_version": ([], ctypes.c_int),
    "sgla_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "sgla_last_cuda_error": ([], ctypes.c_char_p),
    "simple_gla_fwd_workspace_size": ([_I64, _I64, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int], ctypes.c_size_t),
    "simple_gla_fwd_varlen_workspace_size": ([_I64, _I64, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int],
                                             ctypes.c_size_t),
    "simple_gla_fwd": ([_P, _P, _P, _P, _P, _F, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int,
                        ctypes.c_int, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "simple_gla_fwd_noalloc": ([_P, _P, _P, _P, _P, _F, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int,
                                ctypes.c_int, _P], ctypes.c_int),
    "simple_gla_fwd_varlen": ([_P, _P, _P, _P, _P, _F, _P, _I64, _I64, _P, _P, _P, _I64, _I64, _I64,
                               ctypes.c_int, ctypes.c_int, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "simple_gla_decode_step": ([_P, _P, _P, _P, _P, _F, _P, _P, _I64, _I64, _I64, _I64, ctypes.c_int, _P],
                               ctypes.c_int),
    "simple_gla_chunk_workspace_size": ([_P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int, ctypes.c_int],
                                        ctypes.c_size_t),
    "simple_gla_chunk": ([_P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int,
                          ctypes.c_int, ctypes.c_int, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "simple_gla_fused_recurrent": ([_P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64,
                                    ctypes.c_int, ctypes.c_int, _P, _P], ctypes.c_int),
    "simple_gla_fused_recurrent_bwd_workspace_size": ([_P, _I64, _I64, _I64, _I64], ctypes.c_size_t),
    "simple_gla_fused_recurrent_bwd": ([_P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64,
                                        _I64, _I64, _I64, ctypes.c_int, ctypes.c_int, _P, ctypes.c_size_t, _P],
                                       ctypes.c_int),
    "simple_gla_chunk_bwd_workspace_size": ([_P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int],
                                            ctypes.c_size_t),
    "simple_gla_chunk_bwd": ([_P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64,
                              _I64, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "gla_chunk_workspace_size": ([_P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int], ctypes.c_size_t),
    "gla_chunk": ([_P, _P, _P, _P, _F, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int, _P,
                   ctypes.c_size_t, _P], ctypes.c_int),
    "simple_gla_log_decay_total": ([_P, _P, _I64, _I64, _P, _P], ctypes.c_int),
    "simple_gla_state_carry": ([_P, _P, _P, _P, ctypes.c_int, _I64, _I64, _I64, _P], ctypes.c_int),
    "simple_gla_chunk_final_state_workspace_size": ([_P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int],
                                                    ctypes.c_size_t),
    "simple_gla_chunk_final_state": ([_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int,
                                      ctypes.c_int, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "sgla_workspace_status": ([_P, ctypes.POINTER(ctypes.c_int), _P], ctypes.c_int),
    "sgla_noalloc_status": ([ctypes.POINTER(ctypes.c_int), _P], ctypes.c_int),
    "simple_gla_normalized_workspace_size": ([_P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int],
                                             ctypes.c_size_t),
    "simple_gla_normalized": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int,
                               ctypes.c_int, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "simple_gla_normalized_decode_workspace_size": ([_I64, _I64, _I64, ctypes.c_int], ctypes.c_size_t),
    "simple_gla_normalized_decode_step": ([_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, ctypes.c_int, _P,
                                           ctypes.c_size_t, _P], ctypes.c_int),
    "gla_fused_recurrent": ([_P, _P, _P, _P, _F, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int,
                             ctypes.c_int, _P, _P], ctypes.c_int),
    "sgla_selftest_wait_timeout": ([_P, _P], ctypes.c_int),
    "sgla_kernel_launch_count": ([], ctypes.c_uint64),
    "sgla_profile_begin": ([], ctypes.c_int),
    "sgla_profile_end": ([ctypes.c_char_p, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double),
                          ctypes.c_int, ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
}

_lib = None


class ChunkPlan(ctypes.Structure):
    """sgla_chunk_plan of include/simple_gla.h."""
    _fields_ = [("tensor_cores", ctypes.c_int32), ("step_tokens", ctypes.c_int32),
                ("segment_steps", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("max_segments", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64)]


_SIG["simple_gla_chunk_plan"] = ([ctypes.c_int, _I64, _I64, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_int, ctypes.c_int, ctypes.POINTER(ChunkPlan)], ctypes.c_int)


class SglaError(RuntimeError):
    def __init__(self, status, where, detail=""):
        self.status = status
        super().__init__(f"{where}: {status_name(status)}{(' (' + detail + ')') if detail else ''}")


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise ImportError(f"{library_path} is missing: build it with "
                              "`python -m gated_linear_attention_local_b200.build` (no fallback exists)")
        handle = ctypes.CDLL(library_path)
        for name, (args, res) in _SIG.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def kernel_launch_count() -> int:
    """Kernels this library has launched in the process so far."""
    return int(lib().sgla_kernel_launch_count())


def profile_begin():
    raise_for_status(lib().sgla_profile_begin(), "sgla_profile_begin")


def profile_end(max_kernels=32):
    """Stop per-kernel event recording; returns {kernel name: (launches, total ms)}."""
    names = ctypes.create_string_buffer(64 * max_kernels)
    launches = (ctypes.c_int * max_kernels)()
    total = (ctypes.c_double * max_kernels)()
    n = ctypes.c_int(0)
    raise_for_status(lib().sgla_profile_end(names, launches, total, max_kernels, ctypes.byref(n)),
                     "sgla_profile_end")
    out = {}
    for i in range(n.value):
        name = names.raw[64 * i: 64 * (i + 1)].split(b"\0", 1)[0].decode()
        out[name] = (launches[i], total[i])
    return out


def status_name(status) -> str:
    return lib().sgla_status_string(int(status)).decode()


def raise_for_status(status, where):
    status = int(status)
    if status == SGLA_OK:
        return
    if status == SGLA_ERR_INVALID_ARGUMENT:
        raise ValueError(f"{where}: {status_name(status)}")
    if status == SGLA_ERR_UNSUPPORTED:
        raise NotImplementedError(f"{where}: {status_name(status)}")
    detail = lib().sgla_last_cuda_error().decode() if status == SGLA_ERR_CUDA else ""
    raise SglaError(status, where, detail)
