"""Shared helpers for the libkda tests: device transfer, oracle calls, the
tolerance metric.

Tolerance metric (both sides see the same seeded inputs; the oracle gets the
exact values the GPU receives, widened to fp64):
    err(x, ref) = max |x - ref| / max |ref|
bf16 inputs with fp32 accumulation: err(o) <= 2e-2, err(hT) <= 1e-2.
fp32 test mode: err(o) <= 1e-5, err(hT) <= 1e-5.
"""
import numpy as np
import torch

import oracle

TOL_BF16_O = 2e-2
TOL_BF16_S = 1e-2
TOL_FP32 = 1e-5


def tolerances(dtype):
    if dtype == torch.bfloat16:
        return TOL_BF16_O, TOL_BF16_S
    return TOL_FP32, TOL_FP32


def rel_err(x, ref) -> float:
    x = np.asarray(x.detach().cpu().double().numpy() if hasattr(x, "detach") else x,
                   dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    mask = ~np.isnan(ref)
    denom = np.max(np.abs(ref[mask])) if mask.any() else 0.0
    diff = np.max(np.abs(x[mask] - ref[mask])) if mask.any() else 0.0
    if denom == 0.0:
        return float(diff)
    return float(diff / denom)


def to_device(inp, device="cuda"):
    out = {
        "q": inp.q.to(device), "k": inp.k.to(device), "v": inp.v.to(device),
        "g": inp.g.to(device), "beta": inp.beta.to(device),
        "h0": None if inp.h0 is None else inp.h0.to(device),
        "cu_seqlens": inp.cu_seqlens.to(device),
    }
    return out


def oracle_forward(inp, unit_mask=None):
    return oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta,
                          inp.cu_seqlens, inp.h0, unit_mask=unit_mask)
