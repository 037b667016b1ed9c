"""GPU parity of the steps around the operator against the fp64 layer oracle
(oracle/layer_ops.py): the short-conv prologue on its own, and the prologue
followed by the operator against the oracle's prologue followed by the
oracle's recurrence.

Tolerances.  Prologue alone: fp32 arithmetic, outputs rounded to the storage
type, so max|err| <= 2^-8 max|ref| in bf16 (half an ulp of the rounding plus
fp32 noise) and <= 1e-5 in fp32.  Prologue then operator: the operator's own
tolerances (2e-2 / 1e-2 bf16); the bf16 rounding of q, k, v, beta between the
two GPU steps is inside that budget (the oracle chain never rounds)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import layer_ops
from gated_delta_rule_60_b200 import binding, inputs
from kda_testutil import rel_err, tolerances

pytestmark = pytest.mark.gpu

LENGTHS = [1, 2, 3, 0, 5, 17, 130, 64]


def _prologue(li):
    d = {n: getattr(li, n).cuda() for n in ("xq", "xk", "xv", "wq", "wk", "wv", "beta_raw",
                                              "cu_seqlens")}
    out = binding.kda_prologue(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"],
                               d["beta_raw"], d["cu_seqlens"])
    assert binding.kda_stream_status() == binding.KDA_OK
    return out


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.bfloat16, 16),
                                     (torch.float32, 128), (torch.float32, 32)])
def test_prologue_matches_layer_oracle(dtype, d):
    li = inputs.make_layer(LENGTHS, 3, d, dtype, seed=400 + d)
    q, k, v, beta = _prologue(li)
    rq, rk, rv, rb = layer_ops.prologue(li.xq, li.xk, li.xv, li.wq, li.wk, li.wv,
                                        li.beta_raw, li.cu_seqlens.tolist())
    tol = 2.0 ** -8 if dtype == torch.bfloat16 else 1e-5
    for got, ref in ((q, rq), (k, rk), (v, rv), (beta, rb)):
        assert rel_err(got, ref) <= tol, rel_err(got, ref)
    # q and k rows are unit vectors up to the output rounding
    nq = q.float().norm(dim=-1).cpu().numpy()
    assert np.all(np.abs(nq - 1.0) <= (2e-2 if dtype == torch.bfloat16 else 1e-5))


def test_prologue_restarts_at_sequence_starts():
    """Changing the last token of one sequence leaves the next sequence's
    outputs bitwise unchanged (the convolution does not cross the boundary)."""
    li = inputs.make_layer([40, 37], 2, 128, torch.bfloat16, seed=420)
    q1, k1, v1, _ = _prologue(li)
    for x in (li.xq, li.xk, li.xv):
        x[39] = 7.0
    q2, k2, v2, _ = _prologue(li)
    for a, b in ((q1, q2), (k1, k2), (v1, v2)):
        assert torch.equal(a[40:], b[40:])
        assert not torch.equal(a[39], b[39])


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_prologue_then_operator_matches_oracle_chain(dtype, d):
    li = inputs.make_layer([300, 0, 77, 45], 2, d, dtype, seed=430 + d)
    q, k, v, beta = _prologue(li)
    g = li.g.cuda()
    o, hT = binding.kda_chunk_fwd(q, k, v, g, beta, None, li.cu_seqlens.cuda())
    assert binding.kda_stream_status() == binding.KDA_OK
    rq, rk, rv, rb = layer_ops.prologue(li.xq, li.xk, li.xv, li.wq, li.wk, li.wv,
                                        li.beta_raw, li.cu_seqlens.tolist())
    o_ref, h_ref = oracle.forward(rq, rk, rv, li.g, rb, li.cu_seqlens)
    tol_o, tol_s = tolerances(dtype)
    if dtype == torch.float32:
        tol_o = tol_s = 1e-4      # fp32 rounding of the prologue's outputs feeds the operator
    assert rel_err(o, o_ref) <= tol_o and rel_err(hT, h_ref) <= tol_s


def test_prologue_reports_malformed_seqlens():
    li = inputs.make_layer([32, 32], 2, 64, torch.float32, seed=440)
    d = {n: getattr(li, n).cuda() for n in ("xq", "xk", "xv", "wq", "wk", "wv", "beta_raw")}
    bad = torch.tensor([0, 40, 30], dtype=torch.int32, device="cuda")
    binding.kda_prologue(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"],
                         d["beta_raw"], bad)
    assert binding.kda_stream_status() == binding.KDA_ERR_BAD_SEQLENS
    assert binding.kda_stream_status() == binding.KDA_OK


def _gated_case(lengths, H, d, dtype, seed, h0_std=0.02):
    inp = inputs.make_prefill(lengths, H, d, d, dtype, seed=seed, h0_std=h0_std)
    z = inputs.make_layer(lengths, H, d, dtype, seed=seed + 1).z
    return inp, z


@pytest.mark.parametrize("dtype,d,lengths", [
    (torch.bfloat16, 128, [1, 31, 32, 33, 0, 100, 257]),   # tensor-core path, ragged steps
    (torch.float32, 32, [5, 16, 0, 40]),                    # fp32 CUDA-core path
    (torch.bfloat16, 64, [7, 50])])
def test_fused_output_gate_matches_oracle(dtype, d, lengths):
    """o * sigmoid(z) fused into the output store equals the oracle's output
    gate applied to the oracle's operator output; hT is the ungated state,
    bitwise the same as without the gate."""
    inp, z = _gated_case(lengths, 2, d, dtype, seed=450 + d)
    dd = {n: getattr(inp, n).cuda() for n in ("q", "k", "v", "g", "beta", "h0", "cu_seqlens")}
    o, hT = binding.kda_chunk_fwd_gated(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                                        z.cuda(), dd["h0"], dd["cu_seqlens"])
    assert binding.kda_stream_status() == binding.KDA_OK
    o_ref, h_ref = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.h0)
    tol_o, tol_s = tolerances(dtype)
    assert rel_err(o, layer_ops.output_gate(o_ref, z)) <= tol_o
    assert rel_err(hT, h_ref) <= tol_s
    _, hT_plain = binding.kda_chunk_fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                                        dd["h0"], dd["cu_seqlens"])
    assert torch.equal(hT, hT_plain)


def test_fused_output_gate_on_the_segmented_path():
    """One long sequence per head (split into segments, three launches): the
    gate is applied by the launches that write o."""
    T, H = 16384 + 77, 2
    inp, z = _gated_case([T], H, 128, torch.bfloat16, seed=470)
    dd = {n: getattr(inp, n).cuda() for n in ("q", "k", "v", "g", "beta", "h0", "cu_seqlens")}
    o, hT = binding.kda_chunk_fwd_gated(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                                        z.cuda(), dd["h0"], dd["cu_seqlens"])
    assert binding.kda_stream_status() == binding.KDA_OK
    o_ref, h_ref = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.h0)
    assert rel_err(o, layer_ops.output_gate(o_ref, z)) <= 2e-2
    assert rel_err(hT, h_ref) <= 1e-2


def test_gate_extremes():
    """z = +inf passes o through, z = -inf zeroes it."""
    inp, _ = _gated_case([70], 2, 128, torch.bfloat16, seed=480)
    dd = {n: getattr(inp, n).cuda() for n in ("q", "k", "v", "g", "beta", "h0", "cu_seqlens")}
    o_plain, _ = binding.kda_chunk_fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                                       dd["h0"], dd["cu_seqlens"])
    zp = torch.full_like(dd["q"], float("inf"))
    o1, _ = binding.kda_chunk_fwd_gated(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], zp,
                                        dd["h0"], dd["cu_seqlens"])
    o0, _ = binding.kda_chunk_fwd_gated(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], -zp,
                                        dd["h0"], dd["cu_seqlens"])
    assert binding.kda_stream_status() == binding.KDA_OK
    assert torch.equal(o1, o_plain)
    assert int(torch.count_nonzero(o0)) == 0
