"""GPU parity of the unbounded-gate variant (log a = -softplus(g), the Kimi
Linear gate that K3 replaced) against the fp64 oracle's softplus gate.

Cases where the bounded gate's range argument no longer holds: large g (a
16-token tile decays by e^{-320} or more), g = +inf (full forgetting), g =
-inf (no decay), mixed per element, slow decay over long sequences, and the
decode step (one token of the same recurrence)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_60_b200 import binding, inputs
from kda_testutil import rel_err, to_device, tolerances

pytestmark = pytest.mark.gpu


def run(inp):
    d = to_device(inp)
    o, hT = binding.kda_chunk_fwd_softplus(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                           d["h0"], d["cu_seqlens"])
    assert binding.kda_stream_status() == binding.KDA_OK
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
    return o, hT


def check(inp, o, hT):
    o_ref, h_ref = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens,
                                  inp.h0, gate="softplus")
    tol_o, tol_s = tolerances(inp.q.dtype)
    eo, es = rel_err(o, o_ref), rel_err(hT, h_ref)
    assert eo <= tol_o and es <= tol_s, (eo, es)


def with_gate(inp, g):
    return inputs.PrefillInputs(inp.q, inp.k, inp.v, g.to(inp.g.dtype), inp.beta,
                                inp.h0, inp.cu_seqlens)


@pytest.mark.parametrize("dtype,d", [(torch.float32, 16), (torch.float32, 128),
                                     (torch.bfloat16, 128), (torch.bfloat16, 64)])
def test_softplus_gate_normal(dtype, d):
    inp = inputs.make_prefill([1, 15, 16, 17, 0, 70], 2, d, d, dtype, seed=500 + d,
                              h0_std=0.02)
    o, hT = run(inp)
    check(inp, o, hT)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_softplus_gate_beyond_the_bounded_range(dtype):
    """g = 20 gives log a = -20 per token: a 16-token tile spans e^{-320},
    far outside what reciprocal scaling could hold in fp32 or bf16."""
    inp = inputs.make_prefill([40, 33], 2, 128, 128, dtype, seed=510, h0_std=0.02)
    o, hT = run(with_gate(inp, torch.full(inp.g.shape, 20.0)))
    check(with_gate(inp, torch.full(inp.g.shape, 20.0)), o, hT)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_softplus_gate_mixed_extremes(dtype):
    inp = inputs.make_prefill([64, 19], 2, 32, 32, dtype, seed=520, h0_std=0.02)
    levels = torch.tensor([-float("inf"), -30.0, -3.0, 0.0, 3.0, 30.0, float("inf")])
    gen = torch.Generator().manual_seed(521)
    g = levels[torch.randint(0, len(levels), inp.g.shape, generator=gen)]
    case = with_gate(inp, g)
    o, hT = run(case)
    check(case, o, hT)


def test_softplus_full_forgetting_token_by_token():
    """g = +inf forgets everything at every token: each token's output is
    beta (q . k) v of that token alone (the oracle's pinned closed form)."""
    inp = inputs.make_prefill([20], 2, 16, 16, torch.float32, seed=530, h0_std=0.02)
    case = with_gate(inp, torch.full(inp.g.shape, float("inf")))
    o, hT = run(case)
    qk = (inp.q.double() * inp.k.double()).sum(-1)
    want = inp.beta.double()[..., None] * qk[..., None] * inp.v.double()
    assert rel_err(o, want.numpy()) <= 1e-5


def test_softplus_slow_decay_long_sequence():
    inp = inputs.make_prefill([3000], 1, 64, 64, torch.float32, seed=540, h0_std=0.02)
    case = with_gate(inp, inp.g - 8.0)
    o, hT = run(case)
    check(case, o, hT)


@pytest.mark.parametrize("dtype,d", [(torch.float32, 128), (torch.bfloat16, 128),
                                     (torch.float32, 16)])
def test_softplus_decode_is_one_token_prefill(dtype, d):
    B, H = 3, 2
    x = inputs.make_decode_step(B, H, d, d, dtype, seed=550 + d)
    S = inputs.make_state(B, H, d, d, std=0.5, seed=551)
    # the decode step of B sequences = the prefill of B one-token sequences
    o_ref, S_ref = oracle.forward(x.q.reshape(B, H, d), x.k, x.v, x.g, x.beta,
                                  list(range(B + 1)), S, gate="softplus")
    Sd = S.cuda()
    o = binding.kda_decode_step_softplus(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.g.cuda(),
                                         x.beta.cuda(), Sd)
    assert binding.kda_stream_status() == binding.KDA_OK
    tol_o, tol_s = tolerances(dtype)
    assert rel_err(o, o_ref) <= tol_o
    assert rel_err(Sd, S_ref) <= 1e-5
