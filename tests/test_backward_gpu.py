"""GPU parity of the prefill's gradient (kda_chunk_bwd) against the fp64
backward oracle (itself pinned by finite differences, the adjoint identity and
closed forms).

Tolerance.  fp32 arithmetic: every gradient entry is a sum of O(d) products
per token carried through up to a few hundred tokens of reverse recurrence,
so fp32 round-off stays near 1e-6 of the largest entry; 1e-4 of the largest
entry leaves a wide margin and still fails any dropped or mis-signed term
(those move entries by O(1) of the largest).  bf16 storage: inputs, dO and
outputs are bf16, so each gradient carries one output rounding (2^-9 relative)
on top of the fp32 error: 1e-2 of the largest entry."""
import pytest
import torch

import oracle
from gated_delta_rule_60_b200 import binding, inputs
from kda_testutil import rel_err

pytestmark = pytest.mark.gpu


def _case(lengths, H, d, dtype, seed, with_h0=True, with_dhT=True):
    inp = inputs.make_prefill(lengths, H, d, d, dtype, seed=seed,
                              h0_std=0.02 if with_h0 else None)
    gen = torch.Generator().manual_seed(seed + 1)
    T = sum(lengths)
    dO = torch.randn(T, H, d, generator=gen).to(dtype)
    dhT = torch.randn(len(lengths), H, d, d, generator=gen) * 0.1 if with_dhT else None
    return inp, dO, dhT


def _run(inp, dO, dhT):
    c = lambda t: None if t is None else t.cuda()
    out = binding.kda_chunk_bwd(c(inp.q), c(inp.k), c(inp.v), c(inp.g), c(inp.beta), c(dO),
                                c(inp.h0), c(inp.cu_seqlens), c(dhT))
    assert binding.kda_stream_status() == binding.KDA_OK
    return out


def _check(inp, dO, dhT, out, tol):
    ref = oracle.backward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.h0,
                          d_o=dO, d_hT=dhT)
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        err = rel_err(out[name], ref[name])
        assert err <= tol, (name, err)


@pytest.mark.parametrize("d", [16, 32, 128])
def test_backward_fp32_varlen(d):
    """Sequences of 1, 17, 0 and 40 tokens: partial chunks, an empty sequence
    (dh0 = dhT there), several checkpoints."""
    inp, dO, dhT = _case([1, 17, 0, 40], 2, d, torch.float32, seed=600 + d)
    _check(inp, dO, dhT, _run(inp, dO, dhT), 1e-4)


def test_backward_fp32_no_h0_no_dhT():
    inp, dO, _ = _case([33, 50], 2, 64, torch.float32, seed=620, with_h0=False,
                       with_dhT=False)
    _check(inp, dO, None, _run(inp, dO, None), 1e-4)


def test_backward_bf16_d128():
    inp, dO, dhT = _case([70, 45], 2, 128, torch.bfloat16, seed=630)
    _check(inp, dO, dhT, _run(inp, dO, dhT), 1e-2)


def test_backward_longer_sequence():
    """300 tokens: 19 chunks, so the reverse sweep reloads many checkpoints."""
    inp, dO, dhT = _case([300], 1, 32, torch.float32, seed=640)
    _check(inp, dO, dhT, _run(inp, dO, dhT), 1e-4)
