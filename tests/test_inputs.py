"""The seeded synthetic inputs (CPU): the distributions, sizes and seeds that
the tests and the benchmark rely on, as the workload recipe states them.

  q, k ~ N(0, 1), L2-normalised per (token, head);  v, g ~ N(0, 1);
  beta = sigmoid(N(0, 1));  h0 ~ N(0, 0.02^2) fp32;  drawn in fp32 and
  rounded to the storage dtype;  varlen lengths uniform integers on
  [256, 8192];  seeds 1000 + workload index.
"""
import math

import pytest
import torch

from gated_delta_rule_60_b200 import inputs, workloads


def test_prefill_distributions_and_rounding():
    inp = inputs.make_prefill([300, 0, 77], 8, 128, 64, torch.bfloat16, seed=5, h0_std=0.02)
    T = 377
    assert inp.q.shape == inp.k.shape == inp.g.shape == (T, 8, 128)
    assert inp.v.shape == (T, 8, 64) and inp.beta.shape == (T, 8)
    assert inp.h0.shape == (3, 8, 128, 64) and inp.h0.dtype == torch.float32
    assert inp.cu_seqlens.dtype == torch.int32 and inp.cu_seqlens.tolist() == [0, 300, 300, 377]
    assert inp.lengths == [300, 0, 77]
    for t in (inp.q, inp.k, inp.v, inp.g, inp.beta):
        assert t.dtype == torch.bfloat16
    # unit rows up to bf16 rounding of each component
    for t in (inp.q, inp.k):
        n = t.float().norm(dim=-1)
        assert torch.all((n - 1).abs() < 1e-2)
    b = inp.beta.float()
    assert torch.all((b > 0) & (b < 1))
    # N(0, 1) moments over ~96k (v) and ~386k (g) draws: well inside 5 sigma
    for t in (inp.v.float(), inp.g.float()):
        assert abs(t.mean().item()) < 5 / math.sqrt(t.numel())
        assert abs(t.std().item() - 1) < 0.02
    assert abs(inp.h0.std().item() - 0.02) < 0.001
    # sigmoid(N(0,1)) has mean 1/2 by symmetry
    assert abs(b.mean().item() - 0.5) < 0.01


def test_same_seed_same_inputs_other_seed_other_inputs():
    a = inputs.make_prefill([40, 9], 2, 16, 16, torch.float32, seed=7, h0_std=0.1)
    b = inputs.make_prefill([40, 9], 2, 16, 16, torch.float32, seed=7, h0_std=0.1)
    c = inputs.make_prefill([40, 9], 2, 16, 16, torch.float32, seed=8, h0_std=0.1)
    for n in ("q", "k", "v", "g", "beta", "h0"):
        assert torch.equal(getattr(a, n), getattr(b, n))
        assert not torch.equal(getattr(a, n), getattr(c, n))


def test_fp32_inputs_are_the_bf16_draws_before_rounding():
    a = inputs.make_prefill([33], 2, 32, 32, torch.float32, seed=3)
    b = inputs.make_prefill([33], 2, 32, 32, torch.bfloat16, seed=3)
    for n in ("q", "k", "v", "g", "beta"):
        assert torch.equal(getattr(a, n).to(torch.bfloat16), getattr(b, n))


def test_lengths_uniform_inclusive():
    xs = inputs.draw_lengths(20000, 3, 7, seed=1)
    assert min(xs) == 3 and max(xs) == 7
    for v in range(3, 8):
        assert abs(xs.count(v) / 20000 - 0.2) < 0.02


def test_workloads_as_specified():
    assert [w.seed for w in workloads.ALL_PREFILL] == [1000, 1001, 1002, 1003]
    w = workloads.K3_PREFILL
    assert (w.H, w.dk, w.dv, w.dtype, w.T_tot, w.h0_std) == (96, 128, 128, torch.bfloat16,
                                                             8192, None)
    w = workloads.TINY
    assert (w.H, w.dk, w.dtype, w.T_tot) == (2, 16, torch.float32, 64)
    w = workloads.LONG
    assert (w.H, w.dk, w.T_tot, len(w.lengths)) == (16, 128, 1 << 20, 1)
    w = workloads.VARLEN
    assert len(w.lengths) == 24 and all(256 <= L <= 8192 for L in w.lengths)
    assert w.h0_std == 0.02 and w.H == 96
    assert w.T_tot == 104165                    # the drawn lengths of seed 1002
    assert (workloads.DECODE_B, workloads.DECODE_H, workloads.DECODE_D) == (256, 96, 128)
    assert (workloads.DECODE_PREFILL, workloads.DECODE_STEPS) == (512, 128)
    assert workloads.DECODE_STEP_SEED0 == 5000


def test_decode_and_layer_inputs():
    x = inputs.make_decode_step(4, 3, 64, 32, torch.bfloat16, seed=2)
    assert x.q.shape == (4, 3, 64) and x.v.shape == (4, 3, 32) and x.beta.shape == (4, 3)
    assert torch.all((x.k.float().norm(dim=-1) - 1).abs() < 1e-2)
    S = inputs.make_state(2, 3, 16, 16, 0.05, seed=3)
    assert S.shape == (2, 3, 16, 16) and S.dtype == torch.float32
    li = inputs.make_layer([500, 12], 4, 32, torch.bfloat16, seed=4)
    assert li.xq.shape == (512, 4, 32) and li.wq.shape == (4, 32, 4)
    assert li.wq.dtype == torch.float32 and li.z.dtype == torch.bfloat16
    assert abs(torch.cat([li.wq, li.wk, li.wv]).std().item() - 0.5) < 0.03
    assert li.cu_seqlens.tolist() == [0, 500, 512]
