"""Host-only checks of the C ABI (no GPU needed).

The library must load, export every entry point include/kda.h declares, and
reject bad arguments on the host before touching the GPU: these calls pass
null or misaligned pointers and must return the documented status without
any CUDA call being made.
"""
import ctypes
import os
import re

import pytest

import gated_delta_rule_60_b200 as kda
from gated_delta_rule_60_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def _declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(", text)
    return names


def test_header_declares_entry_points():
    names = _declared_symbols()
    for must in ("kda_chunk_fwd", "kda_decode_step", "kda_stream_status",
                 "kda_status_string", "kda_chunk_fwd_workspace_size",
                 "kda_version"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings_and_version(lib):
    assert kda.kda_version() >= 10000
    for s in range(7):
        assert kda.kda_status_string(s)
    assert kda.kda_status_string(99) == "unknown status"


def test_workspace_size_is_host_only(lib):
    assert lib.kda_chunk_fwd_workspace_size(0, 0, 1, 128, 128, 0) == 0
    assert lib.kda_chunk_fwd_workspace_size(1, 64, 2, 16, 16, 1) == 0
    ws = lib.kda_chunk_fwd_workspace_size(1, 8192, 96, 128, 128, 0)
    assert ws >= 0


def _segment_workspace(G, seg0, T, H):
    # G start states, G transfer matrices and G end states of 128 x 128 fp32
    # per head, plus one bf16 row of M^T q per token and head after segment 0
    return 3 * G * H * 128 * 128 * 4 + (T - seg0) * H * 128 * 2


def test_segment_plans_of_the_long_context_workloads(lib):
    """The segment plans the long-sequence path picks on a 148-SM B200, read
    back through the workspace they need: at 2^20 tokens, 16 heads five equal
    segments of 209,728 tokens (the last one 209,664; 144 CTAs in the local
    pass, one wave); at 8 heads eighteen segments of 55,200 tokens with
    segment 0 twice as long.  Below 8,192 tokens, with several sequences,
    and when the heads alone fill the SMs there is no split."""
    ws = lambda N, T, H: lib.kda_chunk_fwd_workspace_size(N, T, H, 128, 128, 0)
    T = 1 << 20
    assert ws(1, T, 16) == _segment_workspace(5, 209728, T, 16)
    assert 4 * 209728 + 209664 == T
    assert ws(1, T, 8) == _segment_workspace(18, 2 * 55200, T, 8)
    assert 2 * 55200 + 16 * 55200 + 54976 == T
    assert ws(1, 8191, 2) == 0
    assert ws(2, 1 << 15, 2) == 0
    assert ws(1, T, 96) == 0 and ws(1, T, 148) == 0


def _call_fwd(lib, **over):
    args = dict(q=16, k=16, v=16, g=16, beta=16, h0=None, cu=None, N=1, T=32,
                H=2, dk=16, dv=16, dt=1, o=16, hT=None, ws=None, wsb=0,
                stream=None)
    args.update(over)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.kda_chunk_fwd(P(args["q"]), P(args["k"]), P(args["v"]),
                             P(args["g"]), P(args["beta"]), P(args["h0"]),
                             P(args["cu"]), args["N"], args["T"], args["H"],
                             args["dk"], args["dv"], args["dt"], P(args["o"]),
                             P(args["hT"]), P(args["ws"]), args["wsb"],
                             P(args["stream"]))


def test_chunk_fwd_host_validation(lib):
    E = binding
    assert _call_fwd(lib, q=None) == E.KDA_ERR_INVALID_ARGUMENT
    assert _call_fwd(lib, o=None) == E.KDA_ERR_INVALID_ARGUMENT
    assert _call_fwd(lib, k=24) == E.KDA_ERR_INVALID_ARGUMENT      # misaligned
    assert _call_fwd(lib, h0=8) == E.KDA_ERR_INVALID_ARGUMENT
    assert _call_fwd(lib, N=-1) == E.KDA_ERR_INVALID_ARGUMENT
    assert _call_fwd(lib, H=0) == E.KDA_ERR_INVALID_ARGUMENT
    assert _call_fwd(lib, T=-5) == E.KDA_ERR_INVALID_ARGUMENT
    assert _call_fwd(lib, N=3, T=32) == E.KDA_ERR_INVALID_ARGUMENT  # 32 % 3
    assert _call_fwd(lib, dk=48, dv=48) == E.KDA_ERR_UNSUPPORTED
    assert _call_fwd(lib, dk=16, dv=32) == E.KDA_ERR_UNSUPPORTED
    assert _call_fwd(lib, dt=7) == E.KDA_ERR_UNSUPPORTED
    assert _call_fwd(lib, N=0, T=0) == E.KDA_OK                    # nothing to do
    assert _call_fwd(lib, N=0, T=4) == E.KDA_ERR_INVALID_ARGUMENT
    assert _call_fwd(lib, N=1 << 16, H=1 << 15, T=1 << 16) == E.KDA_ERR_INVALID_ARGUMENT
    # the tensor-core path takes tokens as signed 32-bit TMA coordinates
    assert _call_fwd(lib, T=1 << 31, dk=128, dv=128, dt=0) == E.KDA_ERR_UNSUPPORTED


def test_chunk_fwd_workspace_validation(lib):
    # one 1M-token sequence on 8 heads is split into segments, which need scratch
    T, H = 1 << 20, 8
    need = lib.kda_chunk_fwd_workspace_size(1, T, H, 128, 128, 0)
    assert need > 0
    st = _call_fwd(lib, T=T, H=H, dk=128, dv=128, dt=0, ws=None, wsb=0)
    assert st == binding.KDA_ERR_WORKSPACE
    st = _call_fwd(lib, T=T, H=H, dk=128, dv=128, dt=0, ws=256, wsb=need - 1)
    assert st == binding.KDA_ERR_WORKSPACE
    st = _call_fwd(lib, T=T, H=H, dk=128, dv=128, dt=0, ws=128, wsb=need)   # not 256-aligned
    assert st == binding.KDA_ERR_WORKSPACE
    # many heads fill the GPU without splitting: no scratch
    assert lib.kda_chunk_fwd_workspace_size(1, 8192, 96, 128, 128, 0) == 0


def test_decode_host_validation(lib):
    P = ctypes.c_void_p
    ok = [P(16)] * 7
    def call(ptrs, B=2, H=2, dk=16, dv=16, dt=1):
        return lib.kda_decode_step(*ptrs, B, H, dk, dv, dt, None)
    bad = list(ok); bad[5] = None
    assert call(bad) == binding.KDA_ERR_INVALID_ARGUMENT
    bad = list(ok); bad[0] = P(20)
    assert call(bad) == binding.KDA_ERR_INVALID_ARGUMENT
    assert call(ok, dk=100, dv=100) == binding.KDA_ERR_UNSUPPORTED
    assert call(ok, B=-1) == binding.KDA_ERR_INVALID_ARGUMENT
    assert call(ok, B=0) == binding.KDA_OK
    assert call(ok, B=1 << 16, H=1 << 15) == binding.KDA_ERR_INVALID_ARGUMENT  # 2^31 units


def test_binding_fails_loudly_without_library(tmp_path):
    saved = binding._lib
    binding._lib = None
    try:
        with pytest.raises(ImportError):
            binding.load_library(str(tmp_path / "missing.so"))
    finally:
        binding._lib = saved


def test_binding_refuses_host_tensors(lib):
    """No CPU path: host tensors are rejected before the library is called."""
    import torch
    T, H, d = 32, 2, 16
    q = torch.zeros(T, H, d)
    beta = torch.zeros(T, H)
    with pytest.raises(ValueError, match="must be on"):
        binding.kda_chunk_fwd(q, q, q, q, beta)
    with pytest.raises(ValueError, match="must be on"):
        binding.kda_decode_step(q[:2], q[:2], q[:2], q[:2], beta[:2],
                                torch.zeros(2, H, d, d))


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(ImportError, match="not built"):
        binding.load_library(str(tmp_path / "libkda.so"))


def test_noalloc_refuses_oversized_scratch_on_the_host(lib):
    """Scratch beyond the static 16 MiB array (the 1M-token, 16-head shape)
    is refused before any device access; the pointers are never used."""
    T, H = 1 << 20, 16
    assert lib.kda_chunk_fwd_workspace_size(1, T, H, 128, 128, 0) > 16 << 20
    P = ctypes.c_void_p
    st = lib.kda_chunk_fwd_noalloc(P(256), P(256), P(256), P(256), P(256), None, None,
                                   1, T, H, 128, 128, 0, P(256), None, None)
    assert st == binding.KDA_ERR_WORKSPACE
    # argument errors still win over the scratch check
    st = lib.kda_chunk_fwd_noalloc(None, P(256), P(256), P(256), P(256), None, None,
                                   1, T, H, 128, 128, 0, P(256), None, None)
    assert st == binding.KDA_ERR_INVALID_ARGUMENT


def test_selftest_limit_is_checked_on_the_host(lib):
    assert lib.kda_selftest_wait_timeout(0, None) == binding.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_selftest_wait_timeout((1 << 32) + 1, None) == binding.KDA_ERR_INVALID_ARGUMENT


def test_prefill_stall_diagnostic_checks_its_arguments(lib):
    """Invalid requests are refused on the host and arm nothing."""
    assert lib.kda_debug_range_prefill(-1) == binding.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_debug_range_read(None, 24) == binding.KDA_ERR_INVALID_ARGUMENT
    buf = (ctypes.c_float * 8)()
    assert lib.kda_debug_range_read(buf, 8) == binding.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_debug_stall_prefill(-1, 1000) == binding.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_debug_stall_prefill(0, 0) == binding.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_debug_stall_prefill(0, (1 << 32) + 1) == binding.KDA_ERR_INVALID_ARGUMENT


def test_prologue_arguments_checked_on_the_host(lib):
    """Unsupported head sizes and dtypes, bad counts and NULL pointers are
    refused before any launch (the pointers below are never dereferenced)."""
    P = ctypes.c_void_p
    args = lambda d, H, N, T, dt, x=P(256): (x, P(256), P(256), P(256), P(256), P(256), P(256),
                                             None, N, T, H, d, dt, P(256), P(256), P(256),
                                             P(256), None)
    assert lib.kda_prologue(*args(48, 2, 1, 64, binding.KDA_BF16)) == binding.KDA_ERR_UNSUPPORTED
    assert lib.kda_prologue(*args(128, 2, 1, 64, 7)) == binding.KDA_ERR_UNSUPPORTED
    assert lib.kda_prologue(*args(128, 0, 1, 64, binding.KDA_BF16)) == binding.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_prologue(*args(128, 70000, 1, 64, binding.KDA_BF16)) == binding.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_prologue(*args(128, 2, 3, 64, binding.KDA_BF16)) == binding.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_prologue(*args(128, 2, 1, 64, binding.KDA_BF16, None)) == binding.KDA_ERR_INVALID_ARGUMENT
    assert lib.kda_prologue(*args(128, 2, 0, 0, binding.KDA_BF16)) == binding.KDA_OK


def test_gated_prefill_needs_z(lib):
    P = ctypes.c_void_p
    st = lib.kda_chunk_fwd_gated(P(256), P(256), P(256), P(256), P(256), None, None, 1, 64, 2,
                                 128, 128, binding.KDA_BF16, None, P(256), None, None, 0, None)
    assert st == binding.KDA_ERR_INVALID_ARGUMENT


def test_backward_workspace_and_arguments(lib):
    """The backward's workspace grows with the chunk checkpoints; a missing or
    short workspace is refused before any launch."""
    ws = lib.kda_chunk_bwd_workspace_size(2, 100, 3, 64, 64, binding.KDA_FP32)
    assert ws == (3 * ((100 + 15) // 16 + 2) + 2 * 3 * 16) * 64 * 64 * 4
    assert lib.kda_chunk_bwd_workspace_size(2, 100, 3, 48, 48, binding.KDA_FP32) == 0
    P = ctypes.c_void_p
    args = [P(256)] * 5 + [None, None, 1, 64, 2, 64, 64, binding.KDA_FP32, P(256), None] + \
        [P(256)] * 5 + [None]
    assert lib.kda_chunk_bwd(*args, None, 0, None) == binding.KDA_ERR_WORKSPACE
    assert lib.kda_chunk_bwd(*args, P(512), 16, None) == binding.KDA_ERR_WORKSPACE


def test_softplus_entry_points_checked_on_the_host(lib):
    """The unbounded-gate prefill and decode refuse unsupported head sizes and
    dtypes, bad counts, and NULL or misaligned pointers before any launch
    (the pointers below are never dereferenced)."""
    P = ctypes.c_void_p
    INV, UNS, OK = binding.KDA_ERR_INVALID_ARGUMENT, binding.KDA_ERR_UNSUPPORTED, binding.KDA_OK

    def fwd(N=1, T=64, H=2, d=128, dt=binding.KDA_BF16, q=256, cu=None, o=256):
        p = lambda x: None if x is None else P(x)
        return lib.kda_chunk_fwd_softplus(p(q), P(256), P(256), P(256), P(256), None, p(cu),
                                          N, T, H, d, d, dt, p(o), None, None)

    assert fwd(d=48) == UNS and fwd(dt=7) == UNS
    assert fwd(H=0) == INV and fwd(N=-1) == INV and fwd(T=-1) == INV
    assert fwd(N=0, T=64) == INV and fwd(N=0, T=0) == OK
    assert fwd(N=3, T=64) == INV                  # equal lengths need T % N == 0
    assert fwd(q=None) == INV and fwd(o=None) == INV and fwd(q=258) == INV
    assert fwd(cu=260) == INV                     # misaligned cu_seqlens

    def dec(B=4, H=2, d=64, dt=binding.KDA_FP32, S=256):
        p = lambda x: None if x is None else P(x)
        return lib.kda_decode_step_softplus(P(256), P(256), P(256), P(256), P(256), p(S),
                                            P(256), B, H, d, d, dt, None)

    assert dec(d=48) == UNS and dec(dt=7) == UNS
    assert dec(B=-1) == INV and dec(H=0) == INV
    assert dec(B=0) == OK
    assert dec(S=None) == INV and dec(S=264) == INV


def test_binding_has_every_entry_point_under_its_c_name(lib):
    """The Python binding mirrors the C ABI name for name, and the package
    exports each of them."""
    for name in _declared_symbols():
        assert callable(getattr(binding, name, None)), name
        assert getattr(kda, name) is getattr(binding, name), name


def test_backward_workspace_query_through_the_binding(lib):
    import torch
    assert binding.kda_chunk_bwd_workspace_size(2, 100, 3, 64, 64, torch.float32) == \
        lib.kda_chunk_bwd_workspace_size(2, 100, 3, 64, 64, binding.KDA_FP32) > 0
