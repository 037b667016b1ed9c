"""The step algebra of the tensor-core prefill, checked on the CPU against the
oracle (no GPU, no library code).

The tensor-core prefill advances each (sequence, head) state in steps of two
16-token tiles and forms every intra-step product with exponents centred on
the end of the first tile.  Per key channel, with b_r the cumulative
log-decay from the start of the step (rows r = 0..31) and m = b_15:

    eps = e^m,  delta = e^{b_31 - m},  gamma = eps * delta = e^{b_31}
    Kr = K e^{b - m},  Qr = Q e^{b - m},  Kh = K e^{m - b}
    Ke = Kr Diag(eps) = K e^b,  Qe = Qr Diag(eps) = Q e^b
    A_kk = Kr Kh^T,  A_qk = Qr Kh^T        (entry (r, i): sum_c x_rc k_ic e^{b_rc - b_ic})
    T = (I + Diag(beta) strict_lower(A_kk))^-1 Diag(beta)
    P = causal(A_qk) T,  Z = Diag(delta) Kh^T T
    W = V - Ke S0
    S_next = Diag(gamma) S0 + Z W,  O = Qe S0 + P W

A partial last step is padded with exact no-op tokens (q = k = v = 0,
beta = 0, log-decay 0), and every sequence restarts its steps.  This is the
unrolled recurrence of the pages ("Kimi K3 发布核实与 Moonshot AI 主干架构演变",
§3 "KDA 为什么不同于 MLA": decay, delta correction, read of the updated state;
item 3: recurrent across chunks, parallel within a chunk) regrouped, with the
reciprocal scaling of "K3 对 Kimi Linear 的进一步修改", bullet 1, applied per
16-token tile.

Two checks:
  * exact arithmetic (fp64, no rounding): the step form equals the
    token-by-token oracle to fp64 round-off for normal, maximal, mixed and
    slow decay, across sequence restarts and partial steps;
  * the kernel's precision plan (fp64 stands in for its fp32 accumulators;
    bf16 rounding at every tensor-core operand: Kr, Qr, Kh, Ke, Qe, the
    causal A_qk, T, P, Diag(delta) Z, the bf16 copy of S0 and -(Ke S0); the
    state itself stays wide): within the bf16 tolerance of the oracle, also
    on a 4,160-token sequence under slow decay (g - 12), where the state
    carries thousands of tokens through the bf16 copy the products read.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_60_b200 import inputs

STEP, TILE = 32, 16


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.bfloat16).to(torch.float64).numpy()


def _f32(x):
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float32).astype(np.float64)


def _exact(x):
    return x


def step(q, k, v, g, beta, S0, rb=_exact, acc=_exact, centre=TILE - 1):
    """One step of up to 32 tokens of one head.  rb rounds a tensor-core
    operand, acc rounds an accumulator (both identity for exact arithmetic).
    centre is the row whose cumulative log-decay is the reference m (None:
    m = 0, the absolute scaling e^{+-b} from the start of the step)."""
    L, dk = q.shape
    dv = v.shape[1]
    pad = STEP - L
    if pad:
        # exact no-op tokens: nothing is written, nothing decays
        q = np.vstack([q, np.zeros((pad, dk))])
        k = np.vstack([k, np.zeros((pad, dk))])
        v = np.vstack([v, np.zeros((pad, dv))])
        beta = np.concatenate([beta, np.zeros(pad)])
    with np.errstate(over="ignore"):
        l = -5.0 / (1.0 + np.exp(-g))
    l = np.vstack([l, np.zeros((pad, dk))])
    b = np.cumsum(l, axis=0)                                  # [32, dk]
    m = np.zeros(dk) if centre is None else b[centre]
    eps, delta, gamma = np.exp(m), np.exp(b[-1] - m), np.exp(b[-1])
    Kr, Qr, Kh = rb(k * np.exp(b - m)), rb(q * np.exp(b - m)), rb(k * np.exp(m - b))
    # The 32 x 32 products also form the non-causal entries (i > r), growth
    # factors up to e^155 that may overflow the fp32 accumulator; the kernel
    # never reads them, and the masks below select instead of multiplying.
    with np.errstate(over="ignore", invalid="ignore"):
        A_kk, A_qk = acc(Kr @ Kh.T), acc(Qr @ Kh.T)
    strict = np.tril(np.ones((STEP, STEP), dtype=bool), -1)
    causal = np.tril(np.ones((STEP, STEP), dtype=bool))
    A_kk = np.where(strict, A_kk, 0.0)
    A_qk = np.where(causal, A_qk, 0.0)
    T = acc(np.linalg.solve(np.eye(STEP) + beta[:, None] * A_kk, np.diag(beta)))
    Tb = rb(T)
    P = rb(acc(rb(A_qk) @ Tb))
    Z = rb(delta[:, None] * acc(Kh.T @ Tb))                    # [dk, 32]
    Ke, Qe = rb(Kr * eps), rb(Qr * eps)
    S0b = rb(S0)
    neg_KeS = rb(-acc(Ke @ S0b))
    O = acc(acc(Qe @ S0b) + P @ v + P @ neg_KeS)
    S = acc(gamma[:, None] * S0 + Z @ v + Z @ neg_KeS)
    return O[:L], S


def forward(q, k, v, g, beta, cu, h0, rb=_exact, acc=_exact, centre=TILE - 1):
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    N = len(cu) - 1
    o = np.zeros((T_tot, H, dv))
    hT = np.zeros((N, H, dk, dv))
    for n in range(N):
        for h in range(H):
            S = np.zeros((dk, dv)) if h0 is None else np.array(h0[n, h], dtype=np.float64)
            for s in range(int(cu[n]), int(cu[n + 1]), STEP):
                e = min(s + STEP, int(cu[n + 1]))
                o[s:e, h], S = step(q[s:e, h], k[s:e, h], v[s:e, h], g[s:e, h],
                                    beta[s:e, h], S, rb, acc, centre)
            hT[n, h] = S
    return o, hT


def _case(lengths, H, d, seed, gate, h0_std=0.02):
    inp = inputs.make_prefill(lengths, H, d, d, torch.bfloat16, seed=seed, h0_std=h0_std)
    g = inp.g.double()
    if gate == "max_decay":
        g = torch.full_like(g, 30.0)
        g[::3] = float("inf")
    elif gate == "mixed":
        vals = torch.tensor([float("inf"), -float("inf"), 30.0, -30.0, 0.0], dtype=torch.float64)
        gen = torch.Generator().manual_seed(seed)
        g = vals[torch.randint(0, 5, g.shape, generator=gen)]
    elif gate.startswith("slow"):
        g = g - float(gate[4:])
    g = g.to(torch.bfloat16).double()
    arrs = [x.double().numpy() for x in (inp.q, inp.k, inp.v)]
    h0 = None if inp.h0 is None else inp.h0.double().numpy()
    return arrs + [g.numpy(), inp.beta.double().numpy(), inp.cu_seqlens.numpy(), h0]


def _rel(x, ref):
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-300))


@pytest.mark.parametrize("gate", ["normal", "max_decay", "mixed", "slow6", "slow12"])
def test_step_form_equals_recurrence_exactly(gate):
    # restarts, partial steps on either side of the tile boundary, an empty sequence
    q, k, v, g, beta, cu, h0 = _case([0, 7, 16, 45, 97], 2, 32, seed=11, gate=gate)
    o, hT = forward(q, k, v, g, beta, cu, h0)
    o_ref, h_ref = oracle.forward(q, k, v, g, beta, cu, h0)
    assert np.isfinite(o).all() and np.isfinite(hT).all()
    assert _rel(o, o_ref) < 1e-11, _rel(o, o_ref)
    assert _rel(hT, h_ref) < 1e-11, _rel(hT, h_ref)


@pytest.mark.parametrize("gate", ["normal", "max_decay", "mixed"])
def test_precision_plan_within_bf16_tolerance(gate):
    q, k, v, g, beta, cu, h0 = _case([45, 130, 300], 2, 128, seed=12, gate=gate)
    o, hT = forward(q, k, v, g, beta, cu, h0, rb=_bf16, acc=_f32)
    o_ref, h_ref = oracle.forward(q, k, v, g, beta, cu, h0)
    assert np.isfinite(o).all() and np.isfinite(hT).all()
    eo, eh = _rel(o, o_ref), _rel(hT, h_ref)
    assert eo <= 2e-2 and eh <= 1e-2, (eo, eh)
    # the plan's own level (about 4e-3 and 2.5e-3 for these seeds), far inside
    # the tolerance: a lost bit of operand precision would show here first
    assert eo <= 6e-3 and eh <= 4e-3, (eo, eh)


def test_centring_is_what_keeps_the_step_in_range():
    """The converse: the same plan with absolute scaling (m = 0) under maximal
    decay needs K e^{-b} up to e^{160} over a 32-token step, past the bf16
    maximum (e^88.7); the step then yields non-finite values or misses the
    tolerance by far."""
    q, k, v, g, beta, cu, h0 = _case([45, 130], 1, 128, seed=14, gate="max_decay")
    with np.errstate(all="ignore"):
        o, hT = forward(q, k, v, g, beta, cu, h0, rb=_bf16, acc=_f32, centre=None)
    o_ref, h_ref = oracle.forward(q, k, v, g, beta, cu, h0)
    bad = not (np.isfinite(o).all() and np.isfinite(hT).all())
    assert bad or _rel(o, o_ref) > 2e-2 or _rel(hT, h_ref) > 1e-2
    # while the centred plan is fine on the same inputs
    o, hT = forward(q, k, v, g, beta, cu, h0, rb=_bf16, acc=_f32)
    assert _rel(o, o_ref) <= 6e-3 and _rel(hT, h_ref) <= 4e-3


def test_precision_plan_under_slow_decay_over_thousands_of_tokens():
    """g - 12 keeps about 0.99997 of the state per token, so S carries
    thousands of tokens; only the correction products see the bf16 copy of
    S, the state stays wide, and the error does not compound."""
    q, k, v, g, beta, cu, h0 = _case([4160], 1, 128, seed=13, gate="slow12")
    o, hT = forward(q, k, v, g, beta, cu, h0, rb=_bf16, acc=_f32)
    o_ref, h_ref = oracle.forward(q, k, v, g, beta, cu, h0)
    eo, eh = _rel(o, o_ref), _rel(hT, h_ref)
    assert eo <= 2e-2 and eh <= 1e-2, (eo, eh)
    assert eo <= 6e-3 and eh <= 4e-3, (eo, eh)
    # and the error of the last 32-token step is no larger than that of a step
    # in the first tenth of the sequence (times two): no growth with length
    def step_err(s):
        return float(np.max(np.abs(o[s:s + 32] - o_ref[s:s + 32])) / np.max(np.abs(o_ref)))
    early = max(step_err(s) for s in range(0, 416, 32))
    assert step_err(4128) <= 2 * early + 1e-6, (step_err(4128), early)
