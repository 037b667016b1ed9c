"""GPU parity of kda_chunk_fwd against the fp64 oracle, plus metamorphic
properties that need no oracle (split-carry, varlen packing, determinism,
no-op padding, decode = prefill)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_60_b200 import binding, inputs, workloads
from kda_testutil import oracle_forward, rel_err, to_device, tolerances

pytestmark = pytest.mark.gpu


def run(inp, **kw):
    d = to_device(inp)
    o, hT = binding.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                  d["h0"], d["cu_seqlens"], **kw)
    assert binding.kda_stream_status() == binding.KDA_OK
    return o, hT


def check(inp, o, hT, unit_mask=None, tol=None):
    o_ref, h_ref = oracle_forward(inp, unit_mask)
    tol_o, tol_s = tol or tolerances(inp.q.dtype)
    eo, es = rel_err(o, o_ref), rel_err(hT, h_ref)
    assert eo <= tol_o and es <= tol_s, (eo, es)
    return eo, es


def test_tiny_fp32_workload():
    """The tiny fp32 workload (B=1, H=2, T=64, d=16) against the oracle at
    1e-5, and its bf16 cast at the bf16 tolerance."""
    inp = workloads.TINY.make()
    o, hT = run(inp)
    check(inp, o, hT)
    b = inputs.make_prefill([64], 2, 16, 16, torch.bfloat16, workloads.TINY.seed)
    o, hT = run(b)
    check(b, o, hT)


@pytest.mark.parametrize("d", [16, 32, 64, 128])
def test_fp32_varlen_partial_chunks(d):
    lengths = [1, 15, 16, 17, 0, 33, 70]
    inp = inputs.make_prefill(lengths, 3, d, d, torch.float32, seed=20 + d,
                              h0_std=0.02)
    o, hT = run(inp)
    check(inp, o, hT)


@pytest.mark.parametrize("d", [16, 32, 64])
def test_bf16_small_heads(d):
    inp = inputs.make_prefill([5, 40, 0, 64], 2, d, d, torch.bfloat16, seed=30 + d,
                              h0_std=0.02)
    o, hT = run(inp)
    check(inp, o, hT)


def test_bf16_d128_varlen_full_oracle():
    """bf16, d = 128 (the tensor-core path) on several tiles and ragged
    tails, every unit checked."""
    lengths = [1, 15, 16, 17, 100, 0, 300, 257]
    inp = inputs.make_prefill(lengths, 3, 128, 128, torch.bfloat16, seed=40,
                              h0_std=0.02)
    o, hT = run(inp)
    check(inp, o, hT)


@pytest.mark.parametrize("n_seq", [40, 600])
def test_bf16_d128_many_sequences(n_seq):
    """Many short sequences in one call: chains run longest first up to 512
    sequences and in index order beyond; both orders must give every
    (sequence, head) its own result."""
    gen = np.random.default_rng(44 + n_seq)
    lengths = gen.integers(0, 41, size=n_seq).tolist()
    inp = inputs.make_prefill(lengths, 1, 128, 128, torch.bfloat16, seed=44,
                              h0_std=0.02)
    o, hT = run(inp)
    check(inp, o, hT)


def test_bf16_d128_step_boundaries():
    """Sequence lengths around the 32-token state steps, packed next to each
    other: full steps leave through the staged tile stores, partial last steps
    through masked stores that must not touch the next sequence's rows."""
    lengths = [31, 32, 33, 63, 64, 65, 96, 1]
    inp = inputs.make_prefill(lengths, 2, 128, 128, torch.bfloat16, seed=42,
                              h0_std=0.02)
    o, hT = run(inp)
    check(inp, o, hT)


def test_bf16_d128_no_h0_no_hT():
    inp = inputs.make_prefill([48, 31], 2, 128, 128, torch.bfloat16, seed=41)
    o, hT = run(inp, output_final_state=False)
    assert hT is None
    o_ref, _ = oracle_forward(inp)
    assert rel_err(o, o_ref) <= 2e-2


def test_k3_prefill_sampled_heads():
    """The K3-shaped workload (H=96, T=8192, d=128, bf16, S0=0) in the launch
    configuration the benchmark times; the oracle checks 6 seeded heads."""
    w = workloads.K3_PREFILL
    inp = w.make()
    o, hT = run(inp)
    mask = np.zeros((1, w.H), dtype=bool)
    mask[0, np.random.default_rng(1).choice(w.H, 4, replace=False)] = True
    mask[0, 0] = mask[0, w.H - 1] = True
    check(inp, o, hT, unit_mask=mask)


def test_varlen_h0_workload_sampled():
    """24 packed sequences (256..8192 tokens), h0 ~ N(0, 0.02^2): oracle on a
    seeded sample of units including the shortest and longest sequence."""
    w = workloads.VARLEN
    inp = w.make()
    o, hT = run(inp)
    L = np.array(inp.lengths)
    rng = np.random.default_rng(2)
    mask = np.zeros((len(L), w.H), dtype=bool)
    for n in (int(L.argmin()), int(L.argmax())):
        mask[n, rng.integers(0, w.H)] = True
    for _ in range(6):
        mask[rng.integers(0, len(L)), rng.integers(0, w.H)] = True
    check(inp, o, hT, unit_mask=mask)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_split_carry(dtype):
    """One call over T tokens equals two calls split at a non-multiple of 16,
    with the first call's hT passed as the second call's h0."""
    d = 128
    inp = inputs.make_prefill([200], 2, d, d, dtype, seed=50, h0_std=0.02)
    o, hT = run(inp)
    cut = 77
    first = inputs.PrefillInputs(inp.q[:cut], inp.k[:cut], inp.v[:cut],
                                 inp.g[:cut], inp.beta[:cut], inp.h0,
                                 inputs.cu_from_lengths([cut]))
    o1, h1 = run(first)
    second = inputs.PrefillInputs(inp.q[cut:], inp.k[cut:], inp.v[cut:],
                                  inp.g[cut:], inp.beta[cut:], h1.cpu(),
                                  inputs.cu_from_lengths([200 - cut]))
    o2, h2 = run(second)
    tol_o, tol_s = tolerances(dtype)
    ref_o = o.float().cpu().double().numpy()
    assert rel_err(torch.cat([o1, o2]), ref_o) <= tol_o
    assert rel_err(h2, hT.cpu().double().numpy()) <= tol_s


def test_varlen_equals_separate_calls():
    lengths = [33, 0, 128, 7]
    inp = inputs.make_prefill(lengths, 2, 128, 128, torch.bfloat16, seed=60,
                              h0_std=0.02)
    o, hT = run(inp)
    cu = inp.cu_seqlens.tolist()
    for n, L in enumerate(lengths):
        s, e = cu[n], cu[n + 1]
        one = inputs.PrefillInputs(inp.q[s:e], inp.k[s:e], inp.v[s:e],
                                   inp.g[s:e], inp.beta[s:e], inp.h0[n:n + 1],
                                   inputs.cu_from_lengths([L]))
        o1, h1 = run(one)
        # packing is bookkeeping: each sequence's chain sees the same work
        assert torch.equal(o1, o[s:e])
        assert torch.equal(h1, hT[n:n + 1])


def test_deterministic():
    inp = inputs.make_prefill([300, 45], 4, 128, 128, torch.bfloat16, seed=70,
                              h0_std=0.02)
    o1, h1 = run(inp)
    o2, h2 = run(inp)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


def test_noop_padding_tokens():
    """Tokens with beta = 0 and g = -inf (alpha = 1) leave the state exactly
    unchanged, so appending them does not change hT."""
    inp = inputs.make_prefill([37], 2, 128, 128, torch.float32, seed=80,
                              h0_std=0.02)
    o, hT = run(inp)
    pad = 21
    z = lambda x: torch.cat([x, torch.zeros((pad,) + tuple(x.shape[1:]), dtype=x.dtype)])
    gp = torch.cat([inp.g, torch.full((pad,) + tuple(inp.g.shape[1:]), -float("inf"))])
    padded = inputs.PrefillInputs(z(inp.q), z(inp.k), z(inp.v), gp, z(inp.beta),
                                  inp.h0, inputs.cu_from_lengths([37 + pad]))
    o2, h2 = run(padded)
    assert rel_err(h2, hT.cpu().double().numpy()) <= 1e-6
    # q = 0 on the padding rows, so their reads are exactly zero
    assert int(torch.count_nonzero(o2[37:])) == 0
    assert torch.equal(o2[:37], o)


def test_decode_equals_prefill():
    """T decode steps from h0 give the same outputs and state as a prefill of
    those T tokens."""
    T, H, d = 40, 3, 128
    for dtype in (torch.float32, torch.bfloat16):
        inp = inputs.make_prefill([T], H, d, d, dtype, seed=90, h0_std=0.02)
        o, hT = run(inp)
        S = inp.h0.clone().cuda()
        outs = []
        for t in range(T):
            sl = slice(t, t + 1)
            outs.append(binding.kda_decode_step(
                inp.q[sl].cuda(), inp.k[sl].cuda(), inp.v[sl].cuda(),
                inp.g[sl].cuda(), inp.beta[sl].cuda(), S))
        tol_o, tol_s = tolerances(dtype)
        assert rel_err(torch.cat(outs), o.float().cpu().double().numpy()) <= tol_o
        assert rel_err(S, hT.cpu().double().numpy()) <= tol_s


@pytest.mark.parametrize("dtype,dim", [(torch.float32, 16), (torch.bfloat16, 128)])
def test_bad_seqlens_reported_not_faulted(dtype, dim):
    inp = inputs.make_prefill([32, 32], 2, dim, dim, dtype, seed=95)
    d = to_device(inp)
    bad = torch.tensor([0, 40, 30], dtype=torch.int32, device="cuda")
    o = torch.zeros(64, 2, dim, dtype=dtype, device="cuda")
    binding.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None, bad, o=o)
    assert binding.kda_stream_status() == binding.KDA_ERR_BAD_SEQLENS
    assert binding.kda_stream_status() == binding.KDA_OK  # cleared


def test_long_sequence_segmented():
    """One long sequence per head with few heads takes the segment-parallel
    path (local pass, combine, final pass).  A ragged last segment and a
    carried state; every unit checked against the oracle."""
    T, H = 16384 + 77, 2
    assert binding.kda_chunk_fwd_workspace_size(1, T, H, 128, 128, torch.bfloat16) > 0
    inp = inputs.make_prefill([T], H, 128, 128, torch.bfloat16, seed=96, h0_std=0.02)
    o, hT = run(inp)
    check(inp, o, hT)


def test_long_sequence_segmented_long_first_segment():
    """A shape whose segment plan gives segment 0 twice the length of the
    others on a 148-SM part (12 heads, 52,901 tokens: twelve segments, the last
    one ragged), with a carried state; every unit checked against the
    oracle."""
    T, H = 52901, 12
    assert binding.kda_chunk_fwd_workspace_size(1, T, H, 128, 128, torch.bfloat16) > 0
    inp = inputs.make_prefill([T], H, 128, 128, torch.bfloat16, seed=97, h0_std=0.02)
    o, hT = run(inp)
    check(inp, o, hT)


def test_long_1m_workload_sampled():
    """The long-context workload (T = 1,048,576, H = 16, bf16, S0 = 0): the
    oracle runs 2 seeded heads over the full length."""
    w = workloads.LONG
    inp = w.make()
    o, hT = run(inp)
    mask = np.zeros((1, w.H), dtype=bool)
    mask[0, np.random.default_rng(3).choice(w.H, 2, replace=False)] = True
    check(inp, o, hT, unit_mask=mask)


@pytest.mark.parametrize("with_h0", [True, False])
def test_all_empty_batch_writes_hT(with_h0):
    """No tokens at all but a final state asked for: the token pointers may be
    NULL, and hT must be h0 (or zero) for every (sequence, head)."""
    N, H, d = 3, 2, 128
    h0 = torch.randn(N, H, d, d, device="cuda") if with_h0 else None
    hT = torch.full((N, H, d, d), 7.0, device="cuda")
    cu = torch.zeros(N + 1, dtype=torch.int32, device="cuda")
    lib = binding.load_library()
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = lib.kda_chunk_fwd(None, None, None, None, None, P(h0), P(cu), N, 0, H, d, d,
                           binding.KDA_BF16, None, P(hT), None, 0, None)
    assert st == binding.KDA_OK
    assert binding.kda_stream_status() == binding.KDA_OK
    assert torch.equal(hT, h0 if with_h0 else torch.zeros_like(hT))


def test_bad_seqlens_on_the_segmented_path():
    """One long sequence per head runs split into segments; a cu_seqlens whose
    last entry is not T_tot must still be reported, with nothing written."""
    T, H = 16384 + 77, 2
    assert binding.kda_chunk_fwd_workspace_size(1, T, H, 128, 128, torch.bfloat16) > 0
    inp = inputs.make_prefill([T], H, 128, 128, torch.bfloat16, seed=98)
    d = to_device(inp)
    bad = torch.tensor([0, T - 1], dtype=torch.int32, device="cuda")
    o = torch.zeros(T, H, 128, dtype=torch.bfloat16, device="cuda")
    hT = torch.zeros(1, H, 128, 128, dtype=torch.float32, device="cuda")
    binding.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None, bad, o=o, hT=hT)
    assert binding.kda_stream_status() == binding.KDA_ERR_BAD_SEQLENS
    assert binding.kda_stream_status() == binding.KDA_OK
    assert int(torch.count_nonzero(o)) == 0 and int(torch.count_nonzero(hT)) == 0
