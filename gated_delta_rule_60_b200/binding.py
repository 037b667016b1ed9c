"""Thin ctypes binding of libkda (include/kda.h).

Argument marshalling only: every function here checks tensor placement,
dtype, shape and contiguity, passes raw device pointers and the current CUDA
stream to the C ABI, and turns a non-OK status into an exception.  All of the
operator's arithmetic runs in libkda's CUDA kernels; there is no fallback of
any kind, and importing a function from here on a machine without the built
library raises immediately.

The Python names are the C names.  As in the C ABI, the tensors of a call
must live on the current CUDA device (select it with torch.cuda.set_device or
a torch.cuda.device context); stream=None means that device's current stream.
"""
import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda.so")

KDA_OK = 0
KDA_ERR_INVALID_ARGUMENT = 1
KDA_ERR_UNSUPPORTED = 2
KDA_ERR_WORKSPACE = 3
KDA_ERR_CUDA = 4
KDA_ERR_TIMEOUT = 5
KDA_ERR_BAD_SEQLENS = 6

KDA_BF16 = 0
KDA_FP32 = 1

_DTYPES = {torch.bfloat16: KDA_BF16, torch.float32: KDA_FP32}

_lib = None


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, kda_status_string(status),
                                                 status))


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libkda.so (built in-tree by gated_delta_rule_60_b200/build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            "libkda.so is not built at %s; run `python -m "
            "gated_delta_rule_60_b200.build` (nvcc, sm_100a)" % path)
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.kda_chunk_fwd_workspace_size.restype = sz
    lib.kda_chunk_fwd_workspace_size.argtypes = [i32, i64, i32, i32, i32, ctypes.c_int]
    lib.kda_chunk_fwd.restype = ctypes.c_int
    lib.kda_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32,
                                  i32, ctypes.c_int, vp, vp, vp, sz, vp]
    lib.kda_chunk_fwd_gated.restype = ctypes.c_int
    lib.kda_chunk_fwd_gated.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32,
                                        i32, ctypes.c_int, vp, vp, vp, vp, sz, vp]
    lib.kda_chunk_fwd_noalloc.restype = ctypes.c_int
    lib.kda_chunk_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32,
                                          i32, ctypes.c_int, vp, vp, vp]
    lib.kda_decode_step.restype = ctypes.c_int
    lib.kda_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                    i32, ctypes.c_int, vp]
    lib.kda_stream_status.restype = ctypes.c_int
    lib.kda_stream_status.argtypes = [vp]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_version.restype = i32
    lib.kda_version.argtypes = []
    lib.kda_selftest_wait_timeout.restype = ctypes.c_int
    lib.kda_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
    lib.kda_chunk_bwd_workspace_size.restype = sz
    lib.kda_chunk_bwd_workspace_size.argtypes = [i32, i64, i32, i32, i32, ctypes.c_int]
    lib.kda_chunk_bwd.restype = ctypes.c_int
    lib.kda_chunk_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32,
                                  ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.kda_chunk_fwd_softplus.restype = ctypes.c_int
    lib.kda_chunk_fwd_softplus.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32,
                                           i32, ctypes.c_int, vp, vp, vp]
    lib.kda_decode_step_softplus.restype = ctypes.c_int
    lib.kda_decode_step_softplus.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                             i32, ctypes.c_int, vp]
    lib.kda_prologue.restype = ctypes.c_int
    lib.kda_prologue.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32,
                                 ctypes.c_int, vp, vp, vp, vp, vp]
    lib.kda_debug_stall_prefill.restype = ctypes.c_int
    lib.kda_debug_stall_prefill.argtypes = [i32, ctypes.c_uint64]
    lib.kda_debug_range_prefill.restype = ctypes.c_int
    lib.kda_debug_range_prefill.argtypes = [i32]
    lib.kda_debug_range_read.restype = ctypes.c_int
    lib.kda_debug_range_read.argtypes = [ctypes.POINTER(ctypes.c_float), sz]
    _lib = lib
    return lib


def kda_status_string(status: int) -> str:
    return load_library().kda_status_string(int(status)).decode()


def kda_version() -> int:
    return int(load_library().kda_version())


def kda_chunk_fwd_workspace_size(N: int, T_tot: int, H: int, dk: int, dv: int,
                                 dtype: torch.dtype) -> int:
    return int(load_library().kda_chunk_fwd_workspace_size(
        int(N), int(T_tot), int(H), int(dk), int(dv), _DTYPES[dtype]))


def kda_chunk_bwd_workspace_size(N: int, T_tot: int, H: int, dk: int, dv: int,
                                 dtype: torch.dtype) -> int:
    return int(load_library().kda_chunk_bwd_workspace_size(
        int(N), int(T_tot), int(H), int(dk), int(dv), _DTYPES[dtype]))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t: torch.Tensor, name: str, dtype, shape, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.device.type != "cuda" or (device is not None and t.device != device):
        raise ValueError("%s must be on %s, got %s" % (name, device or "cuda", t.device))
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape),
                                                            tuple(t.shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def kda_chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                  g: torch.Tensor, beta: torch.Tensor,
                  h0: Optional[torch.Tensor] = None,
                  cu_seqlens: Optional[torch.Tensor] = None, *,
                  num_seqs: Optional[int] = None,
                  o: Optional[torch.Tensor] = None,
                  hT: Optional[torch.Tensor] = None,
                  output_final_state: bool = True,
                  workspace: Optional[torch.Tensor] = None,
                  stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked KDA prefill.  Returns (o [T_tot,H,dv], hT [N,H,dk,dv] or None).

    q, k, g [T_tot, H, dk]; v [T_tot, H, dv]; beta [T_tot, H] share one dtype
    (bf16 or fp32); h0 fp32 [N, H, dk, dv] or None; cu_seqlens int32 [N+1] on
    the device, or None with num_seqs equal-length sequences (default 1).
    """
    lib = load_library()
    dev = q.device
    T_tot, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DTYPES:
        raise TypeError("unsupported dtype %s" % dt)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32, (cu_seqlens.numel(),), dev)
        N = cu_seqlens.numel() - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    for t, name, shp in ((q, "q", (T_tot, H, dk)), (k, "k", (T_tot, H, dk)),
                         (g, "g", (T_tot, H, dk)), (v, "v", (T_tot, H, dv)),
                         (beta, "beta", (T_tot, H))):
        _check(t, name, dt, shp, dev)
    if h0 is not None:
        _check(h0, "h0", torch.float32, (N, H, dk, dv), dev)
    if o is None:
        o = torch.empty(T_tot, H, dv, dtype=dt, device=dev)
    _check(o, "o", dt, (T_tot, H, dv), dev)
    if hT is None and output_final_state:
        hT = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    if hT is not None:
        _check(hT, "hT", torch.float32, (N, H, dk, dv), dev)
    ws_need = kda_chunk_fwd_workspace_size(N, T_tot, H, dk, dv, dt)
    if ws_need and workspace is None:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                           _ptr(h0), _ptr(cu_seqlens), N, T_tot, H, dk, dv,
                           _DTYPES[dt], _ptr(o), _ptr(hT), _ptr(workspace),
                           ws_bytes, _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd")
    return o, hT


def kda_chunk_fwd_gated(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                        g: torch.Tensor, beta: torch.Tensor, z: torch.Tensor,
                        h0: Optional[torch.Tensor] = None,
                        cu_seqlens: Optional[torch.Tensor] = None, *,
                        num_seqs: Optional[int] = None,
                        o: Optional[torch.Tensor] = None,
                        hT: Optional[torch.Tensor] = None,
                        output_final_state: bool = True,
                        workspace: Optional[torch.Tensor] = None,
                        stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """kda_chunk_fwd with the output gate fused into the output store:
    o = (S^T q) * sigmoid(z), z [T_tot, H, dv] in the inputs' dtype."""
    lib = load_library()
    dev = q.device
    T_tot, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DTYPES:
        raise TypeError("unsupported dtype %s" % dt)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32, (cu_seqlens.numel(),), dev)
        N = cu_seqlens.numel() - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    for t, name, shp in ((q, "q", (T_tot, H, dk)), (k, "k", (T_tot, H, dk)),
                         (g, "g", (T_tot, H, dk)), (v, "v", (T_tot, H, dv)),
                         (beta, "beta", (T_tot, H)), (z, "z", (T_tot, H, dv))):
        _check(t, name, dt, shp, dev)
    if h0 is not None:
        _check(h0, "h0", torch.float32, (N, H, dk, dv), dev)
    if o is None:
        o = torch.empty(T_tot, H, dv, dtype=dt, device=dev)
    _check(o, "o", dt, (T_tot, H, dv), dev)
    if hT is None and output_final_state:
        hT = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    if hT is not None:
        _check(hT, "hT", torch.float32, (N, H, dk, dv), dev)
    ws_need = kda_chunk_fwd_workspace_size(N, T_tot, H, dk, dv, dt)
    if ws_need and workspace is None:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.kda_chunk_fwd_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                 _ptr(h0), _ptr(cu_seqlens), N, T_tot, H, dk, dv,
                                 _DTYPES[dt], _ptr(z), _ptr(o), _ptr(hT), _ptr(workspace),
                                 ws_bytes, _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_gated")
    return o, hT


def kda_chunk_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                          g: torch.Tensor, beta: torch.Tensor,
                          h0: Optional[torch.Tensor] = None,
                          cu_seqlens: Optional[torch.Tensor] = None, *,
                          o: torch.Tensor, hT: Optional[torch.Tensor] = None,
                          num_seqs: Optional[int] = None,
                          stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """kda_chunk_fwd for callers that cannot allocate device memory: o (and
    hT, if wanted) must be given; the long-sequence scratch comes from the
    library's static device array, so nothing here allocates."""
    lib = load_library()
    dev = q.device
    T_tot, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DTYPES:
        raise TypeError("unsupported dtype %s" % dt)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32, (cu_seqlens.numel(),), dev)
        N = cu_seqlens.numel() - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    for t, name, shp in ((q, "q", (T_tot, H, dk)), (k, "k", (T_tot, H, dk)),
                         (g, "g", (T_tot, H, dk)), (v, "v", (T_tot, H, dv)),
                         (beta, "beta", (T_tot, H)), (o, "o", (T_tot, H, dv))):
        _check(t, name, dt, shp, dev)
    if h0 is not None:
        _check(h0, "h0", torch.float32, (N, H, dk, dv), dev)
    if hT is not None:
        _check(hT, "hT", torch.float32, (N, H, dk, dv), dev)
    st = lib.kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                   _ptr(h0), _ptr(cu_seqlens), N, T_tot, H, dk, dv,
                                   _DTYPES[dt], _ptr(o), _ptr(hT), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_noalloc")
    return o, hT


def kda_decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                    g: torch.Tensor, beta: torch.Tensor, S: torch.Tensor, *,
                    o: Optional[torch.Tensor] = None,
                    stream=None, _softplus: bool = False) -> torch.Tensor:
    """One KDA decode step; S [B,H,dk,dv] fp32 is updated in place.
    Returns o [B, H, dv] (dtype of q)."""
    lib = load_library()
    dev = q.device
    B, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DTYPES:
        raise TypeError("unsupported dtype %s" % dt)
    for t, name, shp in ((q, "q", (B, H, dk)), (k, "k", (B, H, dk)),
                         (g, "g", (B, H, dk)), (v, "v", (B, H, dv)),
                         (beta, "beta", (B, H))):
        _check(t, name, dt, shp, dev)
    _check(S, "S", torch.float32, (B, H, dk, dv), dev)
    if o is None:
        o = torch.empty(B, H, dv, dtype=dt, device=dev)
    _check(o, "o", dt, (B, H, dv), dev)
    fn = lib.kda_decode_step_softplus if _softplus else lib.kda_decode_step
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o), B, H, dk, dv,
            _DTYPES[dt], _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode_step" + ("_softplus" if _softplus else ""))
    return o


def kda_decode_step_softplus(q, k, v, g, beta, S, *, o=None, stream=None) -> torch.Tensor:
    """kda_decode_step with the unbounded gate log a = -softplus(g)."""
    return kda_decode_step(q, k, v, g, beta, S, o=o, stream=stream, _softplus=True)


def kda_chunk_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                  beta: torch.Tensor, dO: torch.Tensor, h0: Optional[torch.Tensor] = None,
                  cu_seqlens: Optional[torch.Tensor] = None, dhT: Optional[torch.Tensor] = None,
                  *, num_seqs: Optional[int] = None, stream=None) -> dict:
    """Gradient of the prefill for L = <dO, O> + <dhT, hT>: returns a dict of
    dq, dk, dg [T_tot, H, dk], dv [T_tot, H, dv], dbeta [T_tot, H] (dtype of
    q) and dh0 [N, H, dk, dv] fp32."""
    lib = load_library()
    dev = q.device
    T_tot, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DTYPES:
        raise TypeError("unsupported dtype %s" % dt)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32, (cu_seqlens.numel(),), dev)
        N = cu_seqlens.numel() - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    for t, name, shp in ((q, "q", (T_tot, H, dk)), (k, "k", (T_tot, H, dk)),
                         (g, "g", (T_tot, H, dk)), (v, "v", (T_tot, H, dv)),
                         (beta, "beta", (T_tot, H)), (dO, "dO", (T_tot, H, dv))):
        _check(t, name, dt, shp, dev)
    for t, name in ((h0, "h0"), (dhT, "dhT")):
        if t is not None:
            _check(t, name, torch.float32, (N, H, dk, dv), dev)
    out = {"dq": torch.empty(T_tot, H, dk, dtype=dt, device=dev),
           "dk": torch.empty(T_tot, H, dk, dtype=dt, device=dev),
           "dv": torch.empty(T_tot, H, dv, dtype=dt, device=dev),
           "dg": torch.empty(T_tot, H, dk, dtype=dt, device=dev),
           "dbeta": torch.empty(T_tot, H, dtype=dt, device=dev),
           "dh0": torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)}
    ws_n = int(lib.kda_chunk_bwd_workspace_size(N, T_tot, H, dk, dv, _DTYPES[dt]))
    ws = torch.empty(max(ws_n, 256), dtype=torch.uint8, device=dev)
    st = lib.kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                           _ptr(cu_seqlens), N, T_tot, H, dk, dv, _DTYPES[dt], _ptr(dO),
                           _ptr(dhT), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                           _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["dh0"]), _ptr(ws),
                           ws.numel(), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_bwd")
    return out


def kda_chunk_fwd_softplus(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                           g: torch.Tensor, beta: torch.Tensor,
                           h0: Optional[torch.Tensor] = None,
                           cu_seqlens: Optional[torch.Tensor] = None, *,
                           num_seqs: Optional[int] = None,
                           o: Optional[torch.Tensor] = None,
                           hT: Optional[torch.Tensor] = None,
                           output_final_state: bool = True,
                           stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked prefill with the unbounded gate log a = -softplus(g) (fp32
    CUDA-core path, any supported head size, bf16 or fp32 inputs)."""
    lib = load_library()
    dev = q.device
    T_tot, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DTYPES:
        raise TypeError("unsupported dtype %s" % dt)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32, (cu_seqlens.numel(),), dev)
        N = cu_seqlens.numel() - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    for t, name, shp in ((q, "q", (T_tot, H, dk)), (k, "k", (T_tot, H, dk)),
                         (g, "g", (T_tot, H, dk)), (v, "v", (T_tot, H, dv)),
                         (beta, "beta", (T_tot, H))):
        _check(t, name, dt, shp, dev)
    if h0 is not None:
        _check(h0, "h0", torch.float32, (N, H, dk, dv), dev)
    if o is None:
        o = torch.empty(T_tot, H, dv, dtype=dt, device=dev)
    _check(o, "o", dt, (T_tot, H, dv), dev)
    if hT is None and output_final_state:
        hT = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    if hT is not None:
        _check(hT, "hT", torch.float32, (N, H, dk, dv), dev)
    st = lib.kda_chunk_fwd_softplus(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                    _ptr(h0), _ptr(cu_seqlens), N, T_tot, H, dk, dv,
                                    _DTYPES[dt], _ptr(o), _ptr(hT), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_softplus")
    return o, hT


def kda_selftest_wait_timeout(limit_cycles: int, stream=None) -> None:
    """Let one bounded wait run out on the GPU (no fault): afterwards
    kda_stream_status() reports KDA_ERR_TIMEOUT."""
    st = load_library().kda_selftest_wait_timeout(int(limit_cycles), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_selftest_wait_timeout")


def kda_prologue(xq: torch.Tensor, xk: torch.Tensor, xv: torch.Tensor,
                 wq: torch.Tensor, wk: torch.Tensor, wv: torch.Tensor,
                 beta_raw: torch.Tensor, cu_seqlens: Optional[torch.Tensor] = None, *,
                 num_seqs: Optional[int] = None,
                 stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor]:
    """Short-conv prologue: (q, k, v, beta) for kda_chunk_fwd from the raw
    projections xq, xk, xv [T_tot, H, d], taps w* [H, d, 4] fp32 and
    beta_raw [T_tot, H] (see include/kda.h)."""
    lib = load_library()
    dev = xq.device
    T_tot, H, d = xq.shape
    dt = xq.dtype
    if dt not in _DTYPES:
        raise TypeError("unsupported dtype %s" % dt)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32, (cu_seqlens.numel(),), dev)
        N = cu_seqlens.numel() - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    for t, name in ((xq, "xq"), (xk, "xk"), (xv, "xv")):
        _check(t, name, dt, (T_tot, H, d), dev)
    for t, name in ((wq, "wq"), (wk, "wk"), (wv, "wv")):
        _check(t, name, torch.float32, (H, d, 4), dev)
    _check(beta_raw, "beta_raw", dt, (T_tot, H), dev)
    q, k, v = (torch.empty(T_tot, H, d, dtype=dt, device=dev) for _ in range(3))
    beta = torch.empty(T_tot, H, dtype=dt, device=dev)
    st = lib.kda_prologue(_ptr(xq), _ptr(xk), _ptr(xv), _ptr(wq), _ptr(wk), _ptr(wv),
                          _ptr(beta_raw), _ptr(cu_seqlens), N, T_tot, H, d, _DTYPES[dt],
                          _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _stream_handle(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_prologue")
    return q, k, v, beta


def kda_debug_stall_prefill(step: int, limit_cycles: int) -> None:
    """Make the next tensor-core kda_chunk_fwd call stall its scan at state
    step `step` on a wait that nothing completes, bounded by limit_cycles
    (no fault: the kernel reports KDA_ERR_TIMEOUT, drains and returns)."""
    st = load_library().kda_debug_stall_prefill(int(step), int(limit_cycles))
    if st != KDA_OK:
        raise KdaError(st, "kda_debug_stall_prefill")


RANGE_ROWS = ("Kr", "Qr", "Kh", "Z")
RANGE_COLS = ("max_abs", "min_nonzero_abs", "subnormal", "zero", "nonfinite", "count")


def kda_debug_range_prefill(step: int) -> None:
    """Make CTA 0 of the next tensor-core kda_chunk_fwd call record the
    magnitudes of its scaled operands (Kr, Qr, Kh in bf16) and of Z = Kh^T T
    (fp32, before the delta rescale) at state step `step`."""
    st = load_library().kda_debug_range_prefill(int(step))
    if st != KDA_OK:
        raise KdaError(st, "kda_debug_range_prefill")


def kda_debug_range_read() -> dict:
    """The record of kda_debug_range_prefill: {row: {column: value}}."""
    buf = (ctypes.c_float * (len(RANGE_ROWS) * len(RANGE_COLS)))()
    st = load_library().kda_debug_range_read(buf, len(buf))
    if st != KDA_OK:
        raise KdaError(st, "kda_debug_range_read")
    n = len(RANGE_COLS)
    return {r: {c: float(buf[i * n + j]) for j, c in enumerate(RANGE_COLS)}
            for i, r in enumerate(RANGE_ROWS)}


def kda_stream_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(load_library().kda_stream_status(_stream_handle(stream)))
