"""fp64 CPU oracle for the KDA operator (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package.  It is independent of the CUDA library: it imports nothing from
gated_delta_rule_60_b200 and the library imports nothing from here.

The arithmetic lives in kda_oracle.c (a token-by-token fp64 recurrence); this
module only marshals numpy arrays through ctypes.  Every function takes the
exact values the GPU receives, widened to fp64, so input rounding is not
counted as kernel error.

The steps just before and after the operator (short-conv prologue, output
gate) are plain numpy in layer_ops.py.

Recurrence, per head (pages: "Kimi K3 发布核实与 Moonshot AI 主干架构演变" §3
"KDA 为什么不同于 MLA" and "K3 对 Kimi Linear 的进一步修改" bullet 1):
    a_t = exp(-5 * sigmoid(g_t));  S = Diag(a_t) S
    u_t = beta_t (v_t - S^T k_t);  S = S + k_t u_t^T;  o_t = S^T q_t
"""
import ctypes
import os

import numpy as np

from . import build as _build
from .layer_ops import l2_normalize, output_gate, prologue, short_conv  # noqa: F401

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.kda_oracle_forward.restype = ctypes.c_int
        lib.kda_oracle_forward.argtypes = [
            dp, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
            ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.POINTER(ctypes.c_uint8), dp, dp]
        lib.kda_oracle_forward_gate.restype = ctypes.c_int
        lib.kda_oracle_forward_gate.argtypes = \
            lib.kda_oracle_forward.argtypes + [ctypes.c_int]
        lib.kda_oracle_log_alpha_softplus.restype = ctypes.c_double
        lib.kda_oracle_log_alpha_softplus.argtypes = [ctypes.c_double]
        lib.kda_oracle_decode.restype = ctypes.c_int
        lib.kda_oracle_decode.argtypes = [
            dp, dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, dp]
        lib.kda_oracle_log_alpha.restype = ctypes.c_double
        lib.kda_oracle_log_alpha.argtypes = [ctypes.c_double]
        lib.kda_oracle_backward.restype = ctypes.c_int
        lib.kda_oracle_backward.argtypes = [
            dp, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
            ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, dp, dp, dp, dp, dp, dp, dp, dp]
        _lib = lib
    return _lib


def _f64(x):
    """Contiguous fp64 numpy copy of a numpy array or CPU torch tensor."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, ctype=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def log_alpha(g: float) -> float:
    """log a = -5 * sigmoid(g) for one scalar, in fp64."""
    return _load().kda_oracle_log_alpha(float(g))


GATES = {"sigmoid5": 0, "softplus": 1}


def log_alpha_softplus(g: float) -> float:
    """log a = -softplus(g), the unbounded gate K3 replaced, in fp64."""
    return _load().kda_oracle_log_alpha_softplus(float(g))


def forward(q, k, v, g, beta, cu_seqlens, h0=None, unit_mask=None,
            want_o=True, gate="sigmoid5"):
    """Token-by-token fp64 prefill.

    q, k, g: [T_tot, H, dk]; v: [T_tot, H, dv]; beta: [T_tot, H];
    cu_seqlens: [N+1] integers; h0: [N, H, dk, dv] or None (= zeros);
    unit_mask: bool [N, H] or None (= every unit).  gate: "sigmoid5" for K3's
    log a = -5 sigmoid(g), "softplus" for Kimi Linear's unbounded
    log a = -softplus(g) (the variant the pages contrast it with).  Returns
    (o, hT) as fp64 numpy arrays [T_tot, H, dv] and [N, H, dk, dv]; entries of
    units that the mask skips are NaN.
    """
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    cu = np.ascontiguousarray(np.asarray(
        cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
        dtype=np.int64))
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    N = cu.shape[0] - 1
    assert k.shape == (T_tot, H, dk) and g.shape == (T_tot, H, dk)
    assert v.shape == (T_tot, H, dv) and beta.shape == (T_tot, H)
    h0a = None if h0 is None else _f64(h0)
    if h0a is not None:
        assert h0a.shape == (N, H, dk, dv)
    mask = None
    if unit_mask is not None:
        mask = np.ascontiguousarray(np.asarray(unit_mask, dtype=np.uint8)
                                    .reshape(N * H))
    o = np.full((T_tot, H, dv), np.nan) if want_o else None
    hT = np.full((N, H, dk, dv), np.nan)
    rc = _load().kda_oracle_forward_gate(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0a),
        _ptr(cu, ctypes.c_int64), N, T_tot, H, dk, dv,
        _ptr(mask, ctypes.c_uint8), _ptr(o), _ptr(hT), GATES[gate])
    if rc != 0:
        raise ValueError("kda_oracle_forward: malformed cu_seqlens or OOM")
    return o, hT


def backward(q, k, v, g, beta, cu_seqlens, h0=None, d_o=None, d_hT=None):
    """fp64 gradient of the prefill, by the chain rule through the token
    recurrence in reverse.

    For L = <d_o, o> + <d_hT, hT> (either term may be None = zero) returns a
    dict of numpy arrays: dq, dk, dg [T_tot, H, dk], dv [T_tot, H, dv],
    dbeta [T_tot, H] and dh0 [N, H, dk, dv] (the gradient with respect to the
    initial state, zero or not).
    """
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    cu = np.ascontiguousarray(np.asarray(
        cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
        dtype=np.int64))
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    N = cu.shape[0] - 1
    assert k.shape == (T_tot, H, dk) and g.shape == (T_tot, H, dk)
    assert v.shape == (T_tot, H, dv) and beta.shape == (T_tot, H)
    h0a = None if h0 is None else _f64(h0)
    doa = None if d_o is None else _f64(d_o)
    dha = None if d_hT is None else _f64(d_hT)
    if h0a is not None:
        assert h0a.shape == (N, H, dk, dv)
    if doa is not None:
        assert doa.shape == (T_tot, H, dv)
    if dha is not None:
        assert dha.shape == (N, H, dk, dv)
    out = {"dq": np.zeros((T_tot, H, dk)), "dk": np.zeros((T_tot, H, dk)),
           "dv": np.zeros((T_tot, H, dv)), "dg": np.zeros((T_tot, H, dk)),
           "dbeta": np.zeros((T_tot, H)), "dh0": np.zeros((N, H, dk, dv))}
    rc = _load().kda_oracle_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0a),
        _ptr(cu, ctypes.c_int64), N, T_tot, H, dk, dv, _ptr(doa), _ptr(dha),
        _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
        _ptr(out["dbeta"]), _ptr(out["dh0"]))
    if rc != 0:
        raise ValueError("kda_oracle_backward: malformed cu_seqlens or OOM")
    return out


def decode(q, k, v, g, beta, S):
    """One fp64 decode step: q,k,g [B,H,dk], v [B,H,dv], beta [B,H],
    S [B,H,dk,dv].  Returns (o [B,H,dv], S_new) without touching S."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    S = _f64(S).copy()
    B, H, dk = q.shape
    dv = v.shape[2]
    assert S.shape == (B, H, dk, dv)
    o = np.empty((B, H, dv))
    rc = _load().kda_oracle_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                   _ptr(beta), _ptr(S), B, H, dk, dv, _ptr(o))
    if rc != 0:
        raise MemoryError("kda_oracle_decode")
    return o, S


def threads() -> int:
    """OpenMP threads the oracle will use (OMP_NUM_THREADS, else all cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        try:
            return max(1, int(env))
        except ValueError:
            pass
    return os.cpu_count() or 1
