"""Numerics of longer state steps (64 and 128 tokens) with per-32-token-block
scaling: the design study behind the prefill's next lever (fewer, longer
serial steps).  No kernel of the library runs this form yet; this test is the
evidence that its precision plan holds, checked on the CPU against the oracle.

A step of L = 32 B tokens (B blocks of two 16-token tiles) from start state
S0, with b_r the cumulative log-decay from the start of the step:

  * the diagonal block p of A_kk = [beta_r k_r . k_i e^{b_r - b_i}] and of
    A_qk is formed as in the 32-token step, centred on m_p = b at the end of
    the block's first tile, so both scaled operands stay within one
    16-token tile's range (|exponent| <= 80 with the -5 gate bound);
  * an off-diagonal block (row block p after column block q) splits
    e^{b_r - b_i} = e^{b_r - b_e} e^{b_e - b_i} at the boundary e before block
    p: both factors are <= 1, so they can only underflow, and only for
    contributions below e^-87 of the largest, which fp32 drops anyway;
  * T = (I + Diag(beta) strict_lower(A_kk))^-1 Diag(beta) (L x L),
    P = causal(A_qk) T, Z = (K e^{b_last - b})^T T, W = V - (K e^b) S0,
    S_next = Diag(e^{b_last}) S0 + Z W, O = (Q e^b) S0 + P W.

Checked: exact in fp64 against the oracle; with bf16 rounding at every
tensor-core operand (fp32 accumulators, the state kept wide) within the
bf16 tolerance of the oracle, with no non-finite value, for steps of 32, 64
and 128 tokens under normal, maximal and weak decay.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_60_b200 import inputs

TILE, BLOCK = 16, 32


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.bfloat16).to(torch.float64).numpy()


def _f32(x):
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float32).astype(np.float64)


def _exact(x):
    return x


def _pair_products(X, K, b, L, rb, acc, strict):
    """[x_r . k_i e^{b_r - b_i}] for i < r (strict) or i <= r, by blocks."""
    out = np.zeros((L, L))
    for p in range(L // BLOCK):
        rows = slice(p * BLOCK, (p + 1) * BLOCK)
        m = b[p * BLOCK + TILE - 1]                     # centre of the diagonal block
        with np.errstate(over="ignore", invalid="ignore"):
            d = acc(rb(X[rows] * np.exp(b[rows] - m)) @ rb(K[rows] * np.exp(m - b[rows])).T)
        mask = np.tril(np.ones((BLOCK, BLOCK), dtype=bool), -1 if strict else 0)
        out[rows, rows] = np.where(mask, d, 0.0)
        if p:
            e = b[p * BLOCK - 1]                        # boundary before block p
            cols = slice(0, p * BLOCK)
            out[rows, cols] = acc(rb(X[rows] * np.exp(b[rows] - e)) @
                                  rb(K[cols] * np.exp(e - b[cols])).T)
    return out


def step(q, k, v, g, beta, S0, L, rb=_exact, acc=_exact):
    n, dk = q.shape
    dv = v.shape[1]
    pad = L - n
    z = lambda w: np.zeros((pad, w))
    if pad:
        q, k, v = np.vstack([q, z(dk)]), np.vstack([k, z(dk)]), np.vstack([v, z(dv)])
        beta = np.concatenate([beta, np.zeros(pad)])
    with np.errstate(over="ignore"):
        l = -5.0 / (1.0 + np.exp(-g))
    b = np.cumsum(np.vstack([l, z(dk)]), axis=0)
    A_kk = _pair_products(k, k, b, L, rb, acc, strict=True)
    A_qk = _pair_products(q, k, b, L, rb, acc, strict=False)
    T = acc(np.linalg.solve(np.eye(L) + beta[:, None] * A_kk, np.diag(beta)))
    Tb = rb(T)
    P = rb(acc(rb(A_qk) @ Tb))
    Z = rb(acc(rb(k * np.exp(b[-1] - b)).T @ Tb))
    S0b = rb(S0)
    neg_KeS = rb(-acc(rb(k * np.exp(b)) @ S0b))
    O = acc(acc(rb(q * np.exp(b)) @ S0b) + P @ v + P @ neg_KeS)
    S = acc(np.exp(b[-1])[:, None] * S0 + Z @ v + Z @ neg_KeS)
    return O[:n], S


def forward(q, k, v, g, beta, h0, L, rb=_exact, acc=_exact):
    T, dv = q.shape[0], v.shape[1]
    o = np.zeros((T, dv))
    S = h0.copy()
    for s in range(0, T, L):
        e = min(s + L, T)
        o[s:e], S = step(q[s:e], k[s:e], v[s:e], g[s:e], beta[s:e], S, L, rb, acc)
    return o, S


def _case(T, gate, seed):
    inp = inputs.make_prefill([T], 1, 128, 128, torch.bfloat16, seed=seed, h0_std=0.02)
    g = inp.g.double()
    if gate == "max_decay":
        g = torch.full_like(g, 30.0)
    elif gate == "weak":
        g = g - 6.0
    g = g.to(torch.bfloat16).double()
    x = [t[:, 0].double().numpy() for t in (inp.q, inp.k, inp.v)]
    return x + [g[:, 0].numpy(), inp.beta[:, 0].double().numpy(), inp.h0[0, 0].double().numpy()]


def _ref(q, k, v, g, beta, h0):
    T = q.shape[0]
    o, hT = oracle.forward(q[:, None], k[:, None], v[:, None], g[:, None], beta[:, None],
                           np.array([0, T]), h0[None, None])
    return o[:, 0], hT[0, 0]


def _rel(x, ref):
    return float(np.max(np.abs(x - ref)) / np.max(np.abs(ref)))


@pytest.mark.parametrize("L", [32, 64, 128])
@pytest.mark.parametrize("gate", ["normal", "max_decay", "weak"])
def test_blocked_long_step_exact(L, gate):
    q, k, v, g, beta, h0 = _case(300, gate, seed=61)
    o, hT = forward(q, k, v, g, beta, h0, L)
    o_ref, h_ref = _ref(q, k, v, g, beta, h0)
    assert _rel(o, o_ref) < 1e-10 and _rel(hT, h_ref) < 1e-10, (_rel(o, o_ref), _rel(hT, h_ref))


@pytest.mark.parametrize("L", [32, 64, 128])
@pytest.mark.parametrize("gate", ["normal", "max_decay", "weak"])
def test_blocked_long_step_bf16_plan(L, gate):
    q, k, v, g, beta, h0 = _case(2048, gate, seed=62)
    o, hT = forward(q, k, v, g, beta, h0, L, rb=_bf16, acc=_f32)
    assert np.isfinite(o).all() and np.isfinite(hT).all()
    o_ref, h_ref = _ref(q, k, v, g, beta, h0)
    eo, eh = _rel(o, o_ref), _rel(hT, h_ref)
    assert eo <= 2e-2 and eh <= 1e-2, (eo, eh)
    assert eo <= 6e-3 and eh <= 4e-3, (eo, eh)      # the level of the 32-token step


def test_one_centre_per_long_step_leaves_the_range(monkeypatch):
    """The converse: a 64-token step scaled about a single centre needs
    e^{+-160} at maximal decay, past the bf16 maximum, and turns non-finite;
    the block split above is what keeps longer steps in range."""
    import test_long_step_design as mod

    def one_centre(X, K, b, L, rb, acc, strict):
        m = b[L // 2 - 1]
        with np.errstate(all="ignore"):
            d = acc(rb(X * np.exp(b - m)) @ rb(K * np.exp(m - b)).T)
        mask = np.tril(np.ones((L, L), dtype=bool), -1 if strict else 0)
        return np.where(mask, d, 0.0)

    monkeypatch.setattr(mod, "_pair_products", one_centre)
    q, k, v, g, beta, h0 = _case(256, "max_decay", seed=63)
    with np.errstate(all="ignore"):
        o, hT = mod.forward(q, k, v, g, beta, h0, 64, rb=_bf16, acc=_f32)
    assert not (np.isfinite(o).all() and np.isfinite(hT).all())
