"""The segment-parallel scheme of the long-sequence prefill, checked on the CPU
with the oracle as the only arithmetic of the operator (no GPU, no library
code).

For value inputs V and start state S0, the state after the tokens of a
segment is linear in (S0, V): with v = 0 each token maps S to
(I - beta k k^T) Diag(a) S, a left multiplication, so

    S_end = M_s S_start + R_s,   S_t = M_{s,t} S_start + R_{s,t}

where R comes from running the segment from S0 = 0 and M from running it
from S0 = I with v = 0 (its final state is M_s, its outputs are
M_{s,t}^T q_t).  Hence, for every token t of segment s,

    o_t = o_t(zero start) + S_start^T (M_{s,t}^T q_t)

and the start states chain as S_{s+1} = M_s S_s + R_s.  The library's
long-sequence path runs exactly these pieces: segment 0 from the real h0,
every later segment from zero and from the identity (one local pass), the
chain of start states (the combine, whose last state is hT), and the
correction o_t += S_start^T (M_{s,t}^T q_t) with M_{s,t}^T q_t kept in a bf16
scratch and bf16 operands on the tensor cores.

Two checks, on a sequence under slow decay (so that state crosses segment
boundaries) with a doubled first segment and a ragged last one:
  * exact: the composed result equals one oracle run over the whole
    sequence to fp64 round-off;
  * with the path's roundings emulated (o of the zero-start run stored in
    bf16, M^T q and S_start as bf16 operands, fp32 sums and an fp32 combine,
    the result rounded to bf16): within the bf16 tolerance of the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_60_b200 import inputs


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.bfloat16).to(torch.float64).numpy()


def _f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _exact(x):
    return x


def _case(T, H, d, seed, shift):
    inp = inputs.make_prefill([T], H, d, d, torch.bfloat16, seed=seed, h0_std=0.02)
    g = (inp.g.double() - shift).to(torch.bfloat16).double()
    q, k, v, beta = (x.double().numpy() for x in (inp.q, inp.k, inp.v, inp.beta))
    return q, k, v, g.numpy(), beta, inp.h0.double().numpy()


def segmented(q, k, v, g, beta, h0, bounds, rb=_exact, acc=_exact):
    """The long-sequence path's composition for one sequence (N = 1)."""
    T, H, d = q.shape
    o = np.zeros((T, H, d))
    a, b = bounds[0], bounds[1]
    cu = np.array([0, b - a])
    o[a:b], S = oracle.forward(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], cu, h0)
    o[a:b] = rb(o[a:b])
    S = S[0]                                                  # [H, d, d]
    eye = np.broadcast_to(np.eye(d), (1, H, d, d)).copy()
    for a, b in zip(bounds[1:-1], bounds[2:]):
        cu = np.array([0, b - a])
        o_zero, R = oracle.forward(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], cu, None)
        Mq, M = oracle.forward(q[a:b], k[a:b], np.zeros_like(v[a:b]), g[a:b], beta[a:b],
                               cu, eye)
        for h in range(H):
            corr = acc(rb(Mq[:, h]) @ rb(S[h]))               # (S_start^T M^T q)^T per token
            o[a:b, h] = rb(acc(rb(o_zero[:, h]) + corr))
        S = acc(np.einsum("hij,hjk->hik", M[0], S) + R[0])    # S_{s+1} = M_s S_s + R_s
    return o, S[None]


def _rel(x, ref):
    return float(np.max(np.abs(x - ref)) / np.max(np.abs(ref)))


BOUNDS = [0, 256, 384, 512, 640, 700]      # segment 0 doubled, last one ragged


@pytest.mark.parametrize("shift", [0.0, 6.0, 9.0])
def test_segment_composition_equals_one_run(shift):
    q, k, v, g, beta, h0 = _case(700, 2, 32, seed=21, shift=shift)
    o, hT = segmented(q, k, v, g, beta, h0, BOUNDS)
    o_ref, h_ref = oracle.forward(q, k, v, g, beta, np.array([0, 700]), h0)
    assert _rel(o, o_ref) < 1e-11, _rel(o, o_ref)
    assert _rel(hT, h_ref) < 1e-11, _rel(hT, h_ref)


def test_state_crosses_the_segment_boundaries():
    """Under g - 9 the carried state is a large part of the later segments'
    outputs, so the composition is tested, not bypassed: dropping the
    correction leaves errors far beyond the tolerance."""
    q, k, v, g, beta, h0 = _case(700, 2, 32, seed=21, shift=9.0)
    o_ref, _ = oracle.forward(q, k, v, g, beta, np.array([0, 700]), h0)
    cu = np.array([0, 700 - 256])
    o_zero, _ = oracle.forward(q[256:], k[256:], v[256:], g[256:], beta[256:], cu, None)
    assert _rel(o_zero, o_ref[256:]) > 0.2


@pytest.mark.parametrize("shift", [6.0, 9.0])
def test_segment_path_roundings_within_bf16_tolerance(shift):
    q, k, v, g, beta, h0 = _case(700, 2, 32, seed=22, shift=shift)
    o, hT = segmented(q, k, v, g, beta, h0, BOUNDS, rb=_bf16, acc=_f32)
    o_ref, h_ref = oracle.forward(q, k, v, g, beta, np.array([0, 700]), h0)
    eo, eh = _rel(o, o_ref), _rel(hT, h_ref)
    assert eo <= 2e-2 and eh <= 1e-2, (eo, eh)
