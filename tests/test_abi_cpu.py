"""C ABI checks that need no GPU: the library loads, exports every entry point the
header declares, sizes its workspace, and rejects invalid calls before touching
the device (no kernel is launched by any call in this file)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from gated_linear_attention_local_b200 import _lib as L
from gated_linear_attention_local_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "simple_gla.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "defined")))


def test_header_declares_the_three_entry_points():
    names = declared_functions()
    for n in ("simple_gla_fwd", "simple_gla_fwd_varlen", "simple_gla_decode_step"):
        assert n in names


def test_header_is_plain_c(tmp_path):
    """The boundary is a C ABI: the header compiles as C (no C++ or torch types)."""
    src = tmp_path / "use_header.c"
    src.write_text('#include "simple_gla.h"\nint main(void) { return 0; }\n')
    r = subprocess.run(["gcc", "-fsyntax-only", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I",
                        os.path.join(ROOT, "include"), "-I", "/usr/local/cuda/include", str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", L.library_path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if " T " in line)
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    assert set(declared_functions()) == set(L._SIG), "binding signatures out of sync with the header"


def test_status_strings(lib):
    assert lib.sgla_status_string(0) == b"SGLA_OK"
    assert lib.sgla_status_string(1) == b"SGLA_ERR_INVALID_ARGUMENT"
    assert lib.sgla_status_string(99) == b"SGLA_UNKNOWN_STATUS"
    assert lib.sgla_version() >= 100


def test_workspace_sizes(lib):
    ws = lib.simple_gla_fwd_workspace_size
    assert ws(4, 2048, 4, 512, 512, 64, L.SGLA_BF16) > 0
    assert ws(1, 256, 2, 64, 64, 64, L.SGLA_FP32) % 256 == 0
    assert ws(1, 256, 2, 64, 64, 48, L.SGLA_FP32) == 0      # not a power of two
    assert ws(1, 256, 2, 64, 64, 256, L.SGLA_FP32) == 0     # power of two, not built
    assert ws(1, 256, 2, 1024, 64, 64, L.SGLA_FP32) == 0    # K too large
    # the varlen bound does not depend on how T_total splits
    vs = lib.simple_gla_fwd_varlen_workspace_size
    assert vs(8, 18062, 16, 128, 128, 64, L.SGLA_BF16) >= ws(1, 18062, 16, 128, 128, 64, L.SGLA_BF16)
    assert vs(0, 100, 16, 128, 128, 64, L.SGLA_BF16) == 0



def test_size_limits_on_the_host(lib):
    """The largest accepted sizes are accepted and one past them is refused as
    unsupported, before anything is launched (grid y/z bound for H, int32 token
    indices inside the kernels)."""
    ws = lib.simple_gla_fwd_workspace_size
    assert ws(1, 64, 65535, 64, 64, 64, L.SGLA_BF16) > 0
    assert ws(1, 64, 65536, 64, 64, 64, L.SGLA_BF16) == 0
    assert ws(1, 2**31 - 1, 1, 64, 64, 64, L.SGLA_BF16) > 0
    assert ws(2, 2**30, 1, 64, 64, 64, L.SGLA_BF16) == 0          # B x T = 2^31 tokens
    assert ws(1, 64, 1, 512, 512, 64, L.SGLA_BF16) > 0
    assert ws(1, 64, 1, 8, 8, 16, L.SGLA_FP32) > 0                 # smallest head dims, smallest chunk
    assert lib.simple_gla_fwd_varlen_workspace_size(2, 2**31, 1, 64, 64, 64, L.SGLA_BF16) == 0

FAKE = 1 << 20  # an aligned non-NULL address: every call below must return before using it


def _fwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=None, g_gamma=None, scale=float("nan"), h0=None, o=FAKE, hT=None,
             B=1, T=64, H=2, K=64, V=64, C=64, dtype=L.SGLA_BF16, ws=FAKE, wsb=1 << 30, stream=None)
    a.update(kw)
    return lib.simple_gla_fwd(a["q"], a["k"], a["v"], a["g"], a["g_gamma"], a["scale"], a["h0"], a["o"],
                              a["hT"], a["B"], a["T"], a["H"], a["K"], a["V"], a["C"], a["dtype"], a["ws"],
                              a["wsb"], a["stream"])


def test_invalid_calls_are_rejected_on_the_host(lib):
    assert _fwd(lib, g=FAKE, g_gamma=FAKE) == L.SGLA_ERR_INVALID_ARGUMENT   # both gates
    assert _fwd(lib, C=48) == L.SGLA_ERR_INVALID_ARGUMENT                    # not a power of two
    assert _fwd(lib, C=256) == L.SGLA_ERR_UNSUPPORTED
    assert _fwd(lib, K=520) == L.SGLA_ERR_UNSUPPORTED
    assert _fwd(lib, V=60) == L.SGLA_ERR_UNSUPPORTED
    assert _fwd(lib, q=None) == L.SGLA_ERR_INVALID_ARGUMENT
    assert _fwd(lib, q=FAKE + 2) == L.SGLA_ERR_INVALID_ARGUMENT             # misaligned
    assert _fwd(lib, H=0) == L.SGLA_ERR_INVALID_ARGUMENT
    assert _fwd(lib, H=65536) == L.SGLA_ERR_UNSUPPORTED
    assert _fwd(lib, B=2, T=2**30) == L.SGLA_ERR_UNSUPPORTED               # 2^31 tokens
    assert _fwd(lib, B=-1) == L.SGLA_ERR_INVALID_ARGUMENT
    assert _fwd(lib, dtype=7) == L.SGLA_ERR_INVALID_ARGUMENT
    assert _fwd(lib, ws=None) == L.SGLA_ERR_WORKSPACE
    assert _fwd(lib, wsb=16) == L.SGLA_ERR_WORKSPACE
    assert _fwd(lib, ws=FAKE + 16) == L.SGLA_ERR_INVALID_ARGUMENT           # workspace not 256-aligned
    r = lib.simple_gla_fwd_varlen(FAKE, FAKE, FAKE, None, None, 1.0, None, 2, 100, None, FAKE, None,
                                  2, 64, 64, 64, L.SGLA_BF16, FAKE, 1 << 30, None)
    assert r == L.SGLA_ERR_INVALID_ARGUMENT                                  # cu_seqlens missing
    r = lib.simple_gla_fwd_varlen(FAKE, FAKE, FAKE, None, None, 1.0, FAKE, 0, 100, None, FAKE, None,
                                  2, 64, 64, 64, L.SGLA_BF16, FAKE, 1 << 30, None)
    assert r == L.SGLA_ERR_INVALID_ARGUMENT                                  # N == 0
    d = lib.simple_gla_decode_step
    assert d(FAKE, FAKE, FAKE, FAKE, FAKE, 1.0, FAKE, FAKE, 4, 2, 64, 64, 0, None) == L.SGLA_ERR_INVALID_ARGUMENT
    assert d(FAKE, FAKE, FAKE, None, None, 1.0, FAKE, FAKE, 4, 2, 64, 66, 0, None) == L.SGLA_ERR_UNSUPPORTED
    assert d(FAKE, FAKE, FAKE, None, None, 1.0, None, FAKE, 4, 2, 64, 64, 0, None) == L.SGLA_ERR_INVALID_ARGUMENT


def test_chunk_workspace_grows_with_the_vk_layout(lib):
    kv = lib.simple_gla_chunk_workspace_size(None, 4, 2048, 4, 128, 128, 64, 0, L.SGLA_BF16)
    vk = lib.simple_gla_chunk_workspace_size(None, 4, 2048, 4, 128, 128, 64, 1, L.SGLA_BF16)
    assert kv == lib.simple_gla_fwd_workspace_size(4, 2048, 4, 128, 128, 64, L.SGLA_BF16)
    assert vk >= kv + 2 * 4 * 4 * 128 * 128 * 4  # two [K,V] state copies
    assert lib.simple_gla_chunk_workspace_size(None, 4, 2048, 4, 128, 130, 64, 1, L.SGLA_BF16) == 0


def test_fused_recurrent_validation_on_the_host(lib):
    f = lib.simple_gla_fused_recurrent

    def call(q=FAKE, g=None, gg=None, h0=None, hT=None, cu=None, N=4, T=8, H=2, K=64, V=64, vf=0,
             dt=L.SGLA_BF16, status=None):
        return f(q, FAKE, FAKE, g, gg, 1.0, h0, FAKE, hT, cu, N, T, H, K, V, vf, dt, status, None)

    assert call(g=FAKE, gg=FAKE) == L.SGLA_ERR_INVALID_ARGUMENT       # both gates
    assert call(K=520) == L.SGLA_ERR_UNSUPPORTED                      # K above 512
    assert call(K=264, dt=L.SGLA_FP32) == L.SGLA_ERR_UNSUPPORTED      # fp32 K above 256
    assert call(V=68) == L.SGLA_ERR_UNSUPPORTED                       # bf16 V not a multiple of 8
    assert call(K=60) == L.SGLA_ERR_UNSUPPORTED                       # bf16 K not a multiple of 8
    assert call(q=FAKE + 8) == L.SGLA_ERR_INVALID_ARGUMENT            # q not 16-byte aligned
    assert call(h0=FAKE + 8) == L.SGLA_ERR_INVALID_ARGUMENT           # state not 16-byte aligned
    assert call(cu=FAKE, N=0) == L.SGLA_ERR_INVALID_ARGUMENT          # packed with no sequence
    assert call(q=None) == L.SGLA_ERR_INVALID_ARGUMENT                # tokens but no q
    assert call(dt=7) == L.SGLA_ERR_INVALID_ARGUMENT                  # unknown dtype
    assert call(N=0) == L.SGLA_OK                                     # nothing to do, nothing launched


def test_fused_recurrent_bwd_validation_on_the_host(lib):
    f = lib.simple_gla_fused_recurrent_bwd
    ws_need = lib.simple_gla_fused_recurrent_bwd_workspace_size(None, 4, 8, 2, 64)
    assert ws_need >= 2 * 4 * 8 * 2 * 64 * 4 + 4 * 2 * 4   # fp32 dq, dk and one scalar per (sequence, head)
    assert lib.simple_gla_fused_recurrent_bwd_workspace_size(None, 4, 8, 0, 64) == 0

    def call(q=FAKE, g=None, gg=None, h0=None, dht=None, dg=None, dgg=None, dh0=None, cu=None, N=4, T=8, H=2,
             K=64, V=64, dt=L.SGLA_BF16, ws=FAKE, nws=None):
        return f(q, FAKE, FAKE, g, gg, 1.0, h0, FAKE, dht, FAKE, FAKE, FAKE, dg, dgg, dh0, cu, N, T, H, K, V, 0, dt, ws,
                 ws_need if nws is None else nws, None)

    assert call(g=FAKE, gg=FAKE) == L.SGLA_ERR_INVALID_ARGUMENT       # both gates
    assert call(K=520) == L.SGLA_ERR_UNSUPPORTED                      # K above 512
    assert call(V=4100) == L.SGLA_ERR_UNSUPPORTED                     # V above 4096
    assert call(dg=FAKE) == L.SGLA_ERR_INVALID_ARGUMENT               # dg without g
    assert call(g=FAKE, dgg=FAKE) == L.SGLA_ERR_INVALID_ARGUMENT      # dg_gamma without g_gamma
    assert call(dh0=FAKE) == L.SGLA_ERR_INVALID_ARGUMENT              # dh0 without an initial state
    assert call(q=FAKE + 1) == L.SGLA_ERR_INVALID_ARGUMENT            # q not aligned to its element
    assert call(q=None) == L.SGLA_ERR_INVALID_ARGUMENT                # tokens but no q
    assert call(cu=FAKE, N=0) == L.SGLA_ERR_INVALID_ARGUMENT          # packed with no sequence
    assert call(nws=ws_need - 4) == L.SGLA_ERR_WORKSPACE              # workspace too small
    assert call(ws=None) == L.SGLA_ERR_WORKSPACE                      # no workspace
    assert call(ws=FAKE + 16) == L.SGLA_ERR_INVALID_ARGUMENT          # workspace not 256-byte aligned
    assert call(dt=7) == L.SGLA_ERR_INVALID_ARGUMENT                  # unknown dtype


def test_gla_chunk_validation_on_the_host(lib):
    f = lib.gla_chunk
    need = lib.gla_chunk_workspace_size(None, 4, 64, 2, 64, 64, L.SGLA_BF16)
    # q~, k~ (bf16) and the 32 x 32 score blocks of 2 chunks per sequence, plus row decays
    assert need >= 2 * 4 * 64 * 2 * 64 * 2 + 8 * 2 * 32 * 32 * 2 + 8 * 2 * 64 * 4
    assert lib.gla_chunk_workspace_size(None, 4, 64, 2, 264, 64, L.SGLA_BF16) == 0   # K above 256
    assert lib.gla_chunk_workspace_size(None, 4, 64, 2, 60, 64, L.SGLA_BF16) == 0    # bf16 K not a multiple of 8

    def call(q=FAKE, gk=FAKE, cu=None, N=4, T=64, K=64, V=64, dt=L.SGLA_BF16, ws=FAKE, nws=None):
        return f(q, FAKE, FAKE, gk, 1.0, None, FAKE, None, cu, N, T, 2, K, V, dt, ws, need if nws is None else nws,
                 None)

    assert call(K=264) == L.SGLA_ERR_UNSUPPORTED
    assert call(V=68) == L.SGLA_ERR_UNSUPPORTED                       # bf16 V not a multiple of 8
    assert call(q=FAKE + 8) == L.SGLA_ERR_INVALID_ARGUMENT            # q not 16-byte aligned
    assert call(gk=None) == L.SGLA_ERR_INVALID_ARGUMENT               # tokens but no gate
    assert call(cu=FAKE, N=0) == L.SGLA_ERR_INVALID_ARGUMENT          # packed with no sequence
    assert call(nws=need - 1) == L.SGLA_ERR_WORKSPACE
    assert call(ws=FAKE + 16) == L.SGLA_ERR_INVALID_ARGUMENT          # workspace not 256-byte aligned
    assert call(dt=7) == L.SGLA_ERR_INVALID_ARGUMENT


def test_binding_refuses_cpu_tensors():
    import gated_linear_attention_local_b200 as sg
    x = torch.zeros(1, 8, 1, 16)
    with pytest.raises(TypeError):
        sg.simple_gla_fwd(x, x, x)
    with pytest.raises(TypeError):
        sg.simple_gla_decode_step(x[0], x[0], x[0], torch.zeros(1, 8, 16, 16))
    # every other entry point: no CPU path, the call fails before reaching the library
    calls = [
        lambda: sg.simple_gla_chunk(x, x, x),
        lambda: sg.simple_gla_fused_recurrent(x, x, x),
        lambda: sg.simple_gla_normalized(x, x, x),
        lambda: sg.gla_fused_recurrent(x, x, x, x),
        lambda: sg.gla_chunk(x, x, x, x),
        lambda: sg.simple_gla_chunk_bwd(x, x, x, x),
        lambda: sg.simple_gla_fused_recurrent_bwd(x, x, x, x),
        lambda: sg.chunk_simple_gla(x.clone().requires_grad_(True), x, x),
    ]
    for call in calls:
        with pytest.raises(TypeError):
            call()


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(L, "library_path", str(tmp_path / "missing.so"))
    monkeypatch.setattr(L, "_lib", None)
    with pytest.raises(ImportError):
        L.lib()


class _OnDevice(torch.Tensor):
    """A CPU tensor that reports itself as living on a given CUDA device (only the
    binding's device check looks at it; nothing reaches the library)."""

    @property
    def is_cuda(self):
        return True

    @property
    def device(self):
        return self._dev


def _on(dev, *shape):
    t = torch.Tensor._make_subclass(_OnDevice, torch.zeros(*shape))
    t._dev = torch.device(dev)
    return t


def test_binding_refuses_tensors_on_two_devices():
    import gated_linear_attention_local_b200 as sg
    q0 = _on("cuda:0", 1, 8, 2, 16)
    g1 = _on("cuda:1", 1, 8, 2)
    calls = [
        lambda: sg.simple_gla_fwd(q0, q0, q0, g=g1),
        lambda: sg.chunk_simple_gla(q0, q0, q0, g=g1),
        lambda: sg.simple_gla_decode_step(*[_on("cuda:0", 8, 2, 16)] * 3, _on("cuda:1", 8, 2, 16, 16)),
        lambda: sg.simple_gla_chunk_bwd(q0, q0, q0, q0, g=g1),
        lambda: sg.gla_chunk(q0, q0, q0, _on("cuda:1", 1, 8, 2, 16)),
        lambda: sg.simple_gla_state_carry(_on("cuda:0", 2, 2), _on("cuda:1", 2, 2, 16, 16)),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="one device"):
            call()


def test_every_compute_entry_point_has_a_binding_of_the_same_name():
    import gated_linear_attention_local_b200 as sg
    text = open(HEADER).read()
    names = re.findall(r"SGLA_API\s+sgla_status\s+(\w+)\s*\(", text)
    compute = [n for n in names if not n.startswith("sgla_")]
    assert {"simple_gla_fwd", "simple_gla_fwd_varlen", "simple_gla_decode_step"} <= set(compute)
    missing = [n for n in compute if not callable(getattr(sg, n, None))]
    assert not missing, missing


def test_chunk_plan_of_the_measured_workloads(lib):
    """The plan the chunked forward makes for the measured workloads, read on the host:
    the path, the step, the segment length the cost model picks (one segment per
    sequence at K = V = 512, four per sequence on the long per-head-decay workload, and
    the length that balances the walk started under the state pass on the packed
    batch), and the workspace against the size queries."""
    import gated_linear_attention_local_b200 as sg
    p = sg.simple_gla_chunk_plan(4, 2048, 4, 512, 512)  # dense_prefill
    assert p["tensor_cores"] and p["step_tokens"] == 128
    assert p["segment_steps"] == 16 and p["max_segments"] == 4
    assert p["workspace_bytes"] == sg.fwd_workspace_size(4, 2048, 4, 512, 512)
    p = sg.simple_gla_chunk_plan(1, 65536, 32, 128, 128, per_token_gate=False)  # long_gamma
    assert p["segment_steps"] == 128 and p["max_segments"] == 4
    p = sg.simple_gla_chunk_plan(8, 18062, 16, 128, 128, varlen=True)  # varlen_prefill
    assert p["segment_steps"] == 20
    assert p["workspace_bytes"] == sg.varlen_workspace_size(8, 18062, 16, 128, 128)
    p = sg.simple_gla_chunk_plan(1, 256, 2, 64, 64, dtype=torch.float32)  # tiny_fp32
    assert not p["tensor_cores"] and p["step_tokens"] == 64


def test_chunk_plan_agrees_with_the_workspace_query(lib):
    """Over random sizes: the plan's workspace is what simple_gla_chunk_workspace_size
    reports (per-token gate, either state layout), its segments cover every chunk of a
    dense batch exactly, and a packed plan bounds the segments any split can need."""
    import random

    import gated_linear_attention_local_b200 as sg
    rng = random.Random(5)
    for _ in range(300):
        varlen = rng.random() < 0.5
        N = rng.randint(1, 48)
        T = rng.randint(0, 300000)
        H = rng.choice([1, 2, 4, 16, 32])
        K, V = rng.choice([(64, 64), (128, 128), (128, 64), (256, 128), (512, 512), (96, 40)])
        chunk = rng.choice([16, 32, 64, 128])
        vf = rng.random() < 0.3
        dtype = rng.choice([torch.bfloat16, torch.float32])
        p = sg.simple_gla_chunk_plan(N, T, H, K, V, varlen=varlen, chunk_size=chunk, state_v_first=vf,
                                     dtype=dtype)
        cu = ctypes.c_void_p(8) if varlen else None  # the size query only tests it against NULL
        want = lib.simple_gla_chunk_workspace_size(cu, N, T, H, K, V, chunk, int(vf), sg._DTYPES[dtype])
        assert p["workspace_bytes"] == want
        C, L = p["step_tokens"], p["segment_steps"]
        assert C in (16, 32, 64, 128) and L >= 1
        if varlen:
            # every sequence of n tokens needs ceil(ceil(n / C) / L) segments; the sum over
            # any split of T tokens into N sequences is at most T // (C L) + N
            assert p["max_segments"] == T // (C * L) + N
        else:
            assert p["max_segments"] == N * -(-(-(-T // C)) // L)


def test_chunk_plan_rejects_what_the_forward_rejects(lib):
    import gated_linear_attention_local_b200 as sg
    with pytest.raises(ValueError):
        sg.simple_gla_chunk_plan(1, 256, 2, 64, 64, chunk_size=48)
    with pytest.raises(NotImplementedError):
        sg.simple_gla_chunk_plan(1, 256, 2, 64, 64, chunk_size=256)
    with pytest.raises(ValueError):
        sg.simple_gla_chunk_plan(0, 256, 2, 64, 64, varlen=True)
    assert lib.simple_gla_chunk_plan(0, 1, 256, 2, 64, 64, 64, 1, 0, L.SGLA_BF16, None) == L.SGLA_ERR_INVALID_ARGUMENT
