"""fp64 definitions of the steps just before and just after the KDA operator
(test infrastructure only, like the rest of this package; numpy).

Prologue (page "Kimi K3 模型架构解析：KDA、AttnRes 与 Stable LatentMoE", §二.3:
KDA runs 96 heads of 128 state channels together with a length-4 short
convolution for local token mixing).  Readings where the pages are silent:
the convolution is causal and depthwise (one 4-tap filter per head and
channel, tap 0 on the current token), it is applied to the q, k and v
projections, it restarts at every sequence start (zero history), and no
activation follows it; q and k are then L2-normalised per (token, head) and
beta = sigmoid of its raw projection.  The gate g stays raw: the operator
applies log a = -5 sigmoid(g) itself.

Output gate (page "Kimi K3 发布核实与 Moonshot AI 主干架构演变", §3 "K3 对 Kimi
Linear 的进一步修改", bullet 2: the low-rank output gate became an
input-dependent full-rank channel gate).  Reading: o'_t = o_t * sigmoid(z_t)
per value channel, with z_t [H, dv] the full-rank projection of the layer
input (computed outside); no normalisation (the pages name none).
"""
import numpy as np

CONV_TAPS = 4


def _f64(x):
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def sigmoid(x):
    """1 / (1 + e^-x) for any real x, +-inf included, without overflow."""
    x = _f64(x)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def short_conv(x, w, cu_seqlens):
    """Causal depthwise convolution per sequence.

    x [T_tot, H, d]; w [H, d, 4] (w[..., j] multiplies the token j steps
    back); cu_seqlens [N+1].  y_t = sum_j w[..., j] * x_{t-j}, where tokens
    before the start of t's sequence count as zero.
    """
    x, w = _f64(x), _f64(w)
    cu = [int(c) for c in cu_seqlens]
    T, H, d = x.shape
    assert w.shape == (H, d, CONV_TAPS)
    y = np.zeros_like(x)
    for n in range(len(cu) - 1):
        s, e = cu[n], cu[n + 1]
        for t in range(s, e):
            for j in range(CONV_TAPS):
                if t - j >= s:
                    y[t] += w[:, :, j] * x[t - j]
    return y


def l2_normalize(x):
    """x / ||x|| over the last axis; an all-zero row stays zero."""
    x = _f64(x)
    n = np.linalg.norm(x, axis=-1, keepdims=True)
    return x / np.where(n > 0, n, 1.0)


def prologue(xq, xk, xv, wq, wk, wv, beta_raw, cu_seqlens):
    """The operator's inputs from the raw projections:
    q = l2(conv(xq)), k = l2(conv(xk)), v = conv(xv), beta = sigmoid(beta_raw)."""
    q = l2_normalize(short_conv(xq, wq, cu_seqlens))
    k = l2_normalize(short_conv(xk, wk, cu_seqlens))
    v = short_conv(xv, wv, cu_seqlens)
    return q, k, v, sigmoid(beta_raw)


def output_gate(o, z):
    """o * sigmoid(z), elementwise; o and z [T_tot, H, dv]."""
    o, z = _f64(o), _f64(z)
    assert o.shape == z.shape
    return o * sigmoid(z)
