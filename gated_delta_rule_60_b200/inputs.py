"""Seeded synthetic inputs for the KDA operator.

This module draws random numbers and nothing else: it holds none of the
operator's arithmetic, so the tests, the benchmark and the fp64 oracle can all
take their inputs from it.  By default everything is drawn on the CPU with a
seeded ``torch.Generator`` and returned as CPU tensors; with ``device`` set,
make_prefill, make_decode_step and make_layer draw with that device's
generator instead (same distributions, a different random stream) and return
tensors there.

Distributions (the workloads of the KDA operator description):
  q, k ~ N(0, 1), then L2-normalised per (token, head) over the key channels;
  v ~ N(0, 1);  g ~ N(0, 1) per key channel (the raw gate: the operator applies
  log a = -5 * sigmoid(g) itself);  beta = sigmoid(N(0, 1)) per (token, head);
  h0 ~ N(0, std^2) in fp32 when a carried state is requested.
Values are drawn in fp32 and rounded to the requested dtype (bf16 rounding is
round-to-nearest-even); states stay fp32.
"""
from dataclasses import dataclass
from typing import List, Optional

import torch


@dataclass
class PrefillInputs:
    q: torch.Tensor            # [T_tot, H, dk]
    k: torch.Tensor            # [T_tot, H, dk]
    v: torch.Tensor            # [T_tot, H, dv]
    g: torch.Tensor            # [T_tot, H, dk]
    beta: torch.Tensor         # [T_tot, H]
    h0: Optional[torch.Tensor]  # [N, H, dk, dv] fp32 or None
    cu_seqlens: torch.Tensor   # [N+1] int32

    @property
    def lengths(self) -> List[int]:
        cu = self.cu_seqlens.tolist()
        return [cu[i + 1] - cu[i] for i in range(len(cu) - 1)]


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    n = x.norm(dim=-1, keepdim=True)
    return x / torch.where(n > 0, n, torch.ones_like(n))


def cu_from_lengths(lengths) -> torch.Tensor:
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32)


def make_prefill(lengths, H: int, dk: int, dv: int, dtype=torch.bfloat16,
                 seed: int = 0, h0_std: Optional[float] = None,
                 device=None) -> PrefillInputs:
    """Packed varlen prefill inputs for sequences of the given lengths.

    With ``device`` set, the numbers are drawn by that device's generator
    (same distributions, a different random stream) and stay there; this is
    for large benchmark inputs that would be slow to draw on the CPU."""
    dev = torch.device("cpu") if device is None else torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(int(seed))
    T = int(sum(lengths))
    N = len(lengths)
    kw = dict(generator=gen, device=dev)

    def draw_unit(*shape):
        return _unit_rows(torch.randn(*shape, **kw)).to(dtype)

    q = draw_unit(T, H, dk)
    k = draw_unit(T, H, dk)
    v = torch.randn(T, H, dv, **kw).to(dtype)
    g = torch.randn(T, H, dk, **kw).to(dtype)
    beta = torch.sigmoid(torch.randn(T, H, **kw)).to(dtype)
    h0 = None
    if h0_std is not None:
        h0 = torch.randn(N, H, dk, dv, **kw) * float(h0_std)
    return PrefillInputs(q, k, v, g, beta, h0, cu_from_lengths(lengths).to(dev))


def draw_lengths(n: int, lo: int, hi: int, seed: int) -> List[int]:
    """n integer lengths uniform on [lo, hi] (both ends inclusive)."""
    gen = torch.Generator().manual_seed(int(seed))
    return torch.randint(lo, hi + 1, (n,), generator=gen).tolist()


@dataclass
class DecodeInputs:
    q: torch.Tensor     # [B, H, dk]
    k: torch.Tensor     # [B, H, dk]
    v: torch.Tensor     # [B, H, dv]
    g: torch.Tensor     # [B, H, dk]
    beta: torch.Tensor  # [B, H]


def make_decode_step(B: int, H: int, dk: int, dv: int, dtype=torch.bfloat16,
                     seed: int = 0, device=None) -> DecodeInputs:
    """One token per (sequence, head) with the prefill distributions."""
    dev = torch.device("cpu") if device is None else torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(int(seed))
    kw = dict(generator=gen, device=dev)
    q = _unit_rows(torch.randn(B, H, dk, **kw))
    k = _unit_rows(torch.randn(B, H, dk, **kw))
    v = torch.randn(B, H, dv, **kw)
    g = torch.randn(B, H, dk, **kw)
    beta = torch.sigmoid(torch.randn(B, H, **kw))
    return DecodeInputs(q.to(dtype), k.to(dtype), v.to(dtype), g.to(dtype),
                        beta.to(dtype))


def make_state(B: int, H: int, dk: int, dv: int, std: float, seed: int
               ) -> torch.Tensor:
    gen = torch.Generator().manual_seed(int(seed))
    return torch.randn(B, H, dk, dv, generator=gen) * float(std)


@dataclass
class LayerInputs:
    """Raw projections of a KDA layer (before the short-conv prologue)."""
    xq: torch.Tensor            # [T_tot, H, d]
    xk: torch.Tensor            # [T_tot, H, d]
    xv: torch.Tensor            # [T_tot, H, d]
    wq: torch.Tensor            # [H, d, 4] fp32 filter taps
    wk: torch.Tensor
    wv: torch.Tensor
    beta_raw: torch.Tensor      # [T_tot, H]
    g: torch.Tensor             # [T_tot, H, d] raw gate
    z: torch.Tensor             # [T_tot, H, d] raw output-gate projection
    cu_seqlens: torch.Tensor    # [N+1] int32


def make_layer(lengths, H: int, d: int, dtype=torch.bfloat16, seed: int = 0,
               w_std: float = 0.5, device=None) -> LayerInputs:
    """Raw projections x ~ N(0, 1), filter taps ~ N(0, w_std^2) (fp32),
    beta_raw, g, z ~ N(0, 1); drawn in fp32, rounded to dtype (taps stay fp32)."""
    dev = torch.device("cpu") if device is None else torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(int(seed))
    T = int(sum(lengths))
    kw = dict(generator=gen, device=dev)
    xq, xk, xv = (torch.randn(T, H, d, **kw).to(dtype) for _ in range(3))
    wq, wk, wv = (torch.randn(H, d, 4, **kw) * float(w_std) for _ in range(3))
    beta_raw = torch.randn(T, H, **kw).to(dtype)
    g = torch.randn(T, H, d, **kw).to(dtype)
    z = torch.randn(T, H, d, **kw).to(dtype)
    return LayerInputs(xq, xk, xv, wq, wk, wv, beta_raw, g, z, cu_from_lengths(lengths).to(dev))
