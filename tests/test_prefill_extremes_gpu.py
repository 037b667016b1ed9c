"""GPU parity of the tensor-core prefill (bf16, d = 128) at the extremes of
the bounded gate, against the fp64 oracle, every unit checked.

The gate is log a = -5 sigmoid(g) (page "Kimi K3 发布核实与 Moonshot AI 主干架构演
变", §3 "K3 对 Kimi Linear 的进一步修改", bullet 1): its bound of -5 per token is
what keeps the reciprocal decay scaling of a 16-token tile inside the BF16
exponent range.  These cases drive the kernel's scaled operands to that bound
and to the opposite regime:

* maximal decay, g = +30 or g = +inf everywhere: log a = -5 on every channel,
  so a 16-token tile spans |b| = 80 and the scaled keys reach e^{+-75..80};
* mixed extremes, g drawn from {-inf, -30, 0, +30, +inf}: channels that never
  decay next to channels that decay maximally, inside one tile;
* slow decay, g - 6, g - 9, g - 12 over 4,096+ tokens with a carried state:
  the state keeps thousands of tokens, so rounding in the bf16 copy of the
  state that the chunk products read would build up if it compounded;
* no-op padding tokens (beta = 0, g = -inf) through the tensor-core kernel:
  they must leave the state exactly unchanged.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_60_b200 import binding, inputs
from kda_testutil import oracle_forward, rel_err, to_device, tolerances

pytestmark = pytest.mark.gpu

D = 128


def run(inp):
    d = to_device(inp)
    o, hT = binding.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                  d["h0"], d["cu_seqlens"])
    assert binding.kda_stream_status() == binding.KDA_OK
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
    return o, hT


def check(inp, o, hT):
    o_ref, h_ref = oracle_forward(inp)
    tol_o, tol_s = tolerances(torch.bfloat16)
    eo, es = rel_err(o, o_ref), rel_err(hT, h_ref)
    assert eo <= tol_o and es <= tol_s, (eo, es)
    return eo, es


def with_gate(inp, g):
    return inputs.PrefillInputs(inp.q, inp.k, inp.v, g.to(inp.g.dtype), inp.beta,
                                inp.h0, inp.cu_seqlens)


# lengths with full 32-token steps, partial last steps and an empty sequence
LENGTHS = [300, 33, 0, 96, 17]


@pytest.mark.parametrize("gval", [30.0, float("inf")])
def test_maximal_decay(gval):
    inp = inputs.make_prefill(LENGTHS, 3, D, D, torch.bfloat16, seed=300,
                              h0_std=0.02)
    inp = with_gate(inp, torch.full(inp.g.shape, gval))
    o, hT = run(inp)
    check(inp, o, hT)


def test_mixed_extreme_gates():
    inp = inputs.make_prefill(LENGTHS, 3, D, D, torch.bfloat16, seed=301,
                              h0_std=0.02)
    levels = torch.tensor([-float("inf"), -30.0, 0.0, 30.0, float("inf")])
    gen = torch.Generator().manual_seed(302)
    idx = torch.randint(0, len(levels), inp.g.shape, generator=gen)
    inp = with_gate(inp, levels[idx])
    o, hT = run(inp)
    check(inp, o, hT)


def test_mixed_extremes_per_channel():
    """Each key channel keeps one extreme gate for the whole sequence, so
    never-decaying channels accumulate next to maximally decaying ones."""
    inp = inputs.make_prefill([700, 64], 2, D, D, torch.bfloat16, seed=303,
                              h0_std=0.02)
    levels = torch.tensor([-float("inf"), -30.0, 0.0, 30.0, float("inf")])
    gen = torch.Generator().manual_seed(304)
    per_ch = levels[torch.randint(0, len(levels), (1, 2, D), generator=gen)]
    inp = with_gate(inp, per_ch.expand_as(inp.g).clone())
    o, hT = run(inp)
    check(inp, o, hT)


@pytest.mark.parametrize("shift", [6.0, 9.0, 12.0])
def test_slow_decay_long_memory(shift):
    inp = inputs.make_prefill([4096 + 45, 1000], 2, D, D, torch.bfloat16,
                              seed=310 + int(shift), h0_std=0.02)
    inp = with_gate(inp, inp.g.float() - shift)
    o, hT = run(inp)
    check(inp, o, hT)


def test_noop_padding_tokens_tensor_core_path():
    """beta = 0 and g = -inf (a = 1) are exact no-ops: appending such tokens
    leaves hT unchanged and, with q = 0 there, their outputs are zero."""
    inp = inputs.make_prefill([75], 2, D, D, torch.bfloat16, seed=320, h0_std=0.02)
    o, hT = run(inp)
    pad = 53
    z = lambda x: torch.cat([x, torch.zeros((pad,) + tuple(x.shape[1:]), dtype=x.dtype)])
    gp = torch.cat([inp.g, torch.full((pad,) + tuple(inp.g.shape[1:]), -float("inf"),
                                      dtype=inp.g.dtype)])
    padded = inputs.PrefillInputs(z(inp.q), z(inp.k), z(inp.v), gp, z(inp.beta),
                                  inp.h0, inputs.cu_from_lengths([75 + pad]))
    o2, h2 = run(padded)
    assert torch.equal(o2[:75], o)
    assert int(torch.count_nonzero(o2[75:])) == 0
    # the padding only re-associates fp32 sums of the state; no decay, no write
    assert rel_err(h2, hT.cpu().double().numpy()) <= 1e-6
    check(padded, o2, h2)
