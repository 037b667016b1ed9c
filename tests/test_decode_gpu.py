"""GPU parity of kda_decode_step against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_60_b200 import binding, inputs
from kda_testutil import rel_err, tolerances

pytestmark = pytest.mark.gpu


def _step_inputs(B, H, d, dtype, seed):
    x = inputs.make_decode_step(B, H, d, d, dtype, seed)
    return x


@pytest.mark.parametrize("d", [16, 32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_one_step(d, dtype):
    B, H = 3, 5
    x = _step_inputs(B, H, d, dtype, seed=100 + d)
    S = inputs.make_state(B, H, d, d, std=0.5, seed=7)
    o_ref, S_ref = oracle.decode(x.q, x.k, x.v, x.g, x.beta, S)
    Sd = S.cuda()
    o = binding.kda_decode_step(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.g.cuda(),
                                x.beta.cuda(), Sd)
    assert binding.kda_stream_status() == binding.KDA_OK
    tol_o, tol_s = tolerances(dtype)
    assert rel_err(o, o_ref) <= tol_o
    assert rel_err(Sd, S_ref) <= tol_s
    # the state is fp32 and the inputs are exact: only fp32 rounding remains
    assert rel_err(Sd, S_ref) <= 1e-5


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_many_steps(dtype):
    """20 chained steps on 7 x 3 heads (a ragged head count)."""
    B, H, d = 7, 3, 128
    S = inputs.make_state(B, H, d, d, std=0.02, seed=8)
    Sd = S.cuda()
    S_ref = S.double().numpy()
    tol_o, tol_s = tolerances(dtype)
    for s in range(20):
        x = _step_inputs(B, H, d, dtype, seed=5000 + s)
        o_ref, S_ref = oracle.decode(x.q, x.k, x.v, x.g, x.beta, S_ref)
        o = binding.kda_decode_step(x.q.cuda(), x.k.cuda(), x.v.cuda(),
                                    x.g.cuda(), x.beta.cuda(), Sd)
        assert rel_err(o, o_ref) <= tol_o, s
    assert rel_err(Sd, S_ref) <= tol_s


def test_decode_full_size_sampled():
    """256 x 96 heads (the batched-decode workload) for 3 steps; the oracle
    checks a seeded sample of 40 (sequence, head) units one by one."""
    B, H, d = 256, 96, 128
    S = inputs.make_state(B, H, d, d, std=0.05, seed=9)
    Sd = S.cuda()
    rng = np.random.default_rng(0)
    units = [(int(b), int(h)) for b, h in zip(rng.integers(0, B, 40),
                                              rng.integers(0, H, 40))]
    units += [(0, 0), (B - 1, H - 1)]
    S_ref = {u: S[u[0], u[1]].double().numpy()[None, None] for u in units}
    for s in range(3):
        x = _step_inputs(B, H, d, torch.bfloat16, seed=5000 + s)
        o = binding.kda_decode_step(x.q.cuda(), x.k.cuda(), x.v.cuda(),
                                    x.g.cuda(), x.beta.cuda(), Sd)
        oc = o.float().cpu()
        for (b, h) in units:
            sl = (slice(b, b + 1), slice(h, h + 1))
            o_ref, S_ref[(b, h)] = oracle.decode(
                x.q[sl], x.k[sl], x.v[sl], x.g[sl], x.beta[sl], S_ref[(b, h)])
            assert rel_err(oc[b, h], o_ref[0, 0]) <= 2e-2
    Sc = Sd.cpu()
    for (b, h) in units:
        assert rel_err(Sc[b, h], S_ref[(b, h)][0, 0]) <= 1e-2


def test_decode_empty_batch_is_noop():
    q = torch.zeros(0, 2, 16, device="cuda")
    S = torch.zeros(0, 2, 16, 16, device="cuda")
    o = binding.kda_decode_step(q, q, q, q, torch.zeros(0, 2, device="cuda"), S)
    assert o.shape == (0, 2, 16)


def test_batched_decode_workload_from_prefill_state():
    """The batched-decode workload as specified: 256 sequences x 96 heads,
    the state built by a 512-token kda_chunk_fwd prefill of every sequence,
    then 128 chained kda_decode_step calls with fresh inputs each step.  The
    oracle follows a seeded sample of (sequence, head) units through the same
    prefill and all 128 steps, checking o at every step and the state at the
    end.  Inputs are drawn on the device (the benchmark's generator) and the
    oracle receives copies of the sampled units' values."""
    from gated_delta_rule_60_b200 import workloads
    B, H, d = workloads.DECODE_B, workloads.DECODE_H, workloads.DECODE_D
    P = workloads.DECODE_PREFILL
    pre = inputs.make_prefill([P] * B, H, d, d, torch.bfloat16, workloads.DECODE_SEED,
                              device="cuda")
    S = torch.empty(B, H, d, d, dtype=torch.float32, device="cuda")
    binding.kda_chunk_fwd(pre.q, pre.k, pre.v, pre.g, pre.beta, None, pre.cu_seqlens,
                          hT=S)
    assert binding.kda_stream_status() == binding.KDA_OK
    rng = np.random.default_rng(4)
    units = sorted({(int(b), int(h)) for b, h in zip(rng.integers(0, B, 14),
                                                     rng.integers(0, H, 14))}
                   | {(0, 0), (B - 1, H - 1)})
    S_ref = {}
    for (b, h) in units:
        tok = slice(b * P, (b + 1) * P)
        sl = lambda x: x[tok, h:h + 1].cpu()
        _, hT = oracle.forward(sl(pre.q), sl(pre.k), sl(pre.v), sl(pre.g),
                               sl(pre.beta), [0, P], None)
        S_ref[(b, h)] = hT
    del pre
    Sc = S.cpu()
    for (b, h) in units:
        assert rel_err(Sc[b, h], S_ref[(b, h)][0, 0]) <= 1e-2
    for s in range(workloads.DECODE_STEPS):
        x = inputs.make_decode_step(B, H, d, d, torch.bfloat16,
                                    workloads.DECODE_STEP_SEED0 + s, device="cuda")
        o = binding.kda_decode_step(x.q, x.k, x.v, x.g, x.beta, S)
        oc = o.float().cpu()
        for (b, h) in units:
            sl = lambda t: t[b:b + 1, h:h + 1].cpu()
            o_ref, S_ref[(b, h)] = oracle.decode(sl(x.q), sl(x.k), sl(x.v), sl(x.g),
                                                 sl(x.beta), S_ref[(b, h)])
            assert rel_err(oc[b, h], o_ref[0, 0]) <= 2e-2, (s, b, h)
    assert binding.kda_stream_status() == binding.KDA_OK
    Sc = S.cpu()
    for (b, h) in units:
        assert rel_err(Sc[b, h], S_ref[(b, h)][0, 0]) <= 1e-2, (b, h)
