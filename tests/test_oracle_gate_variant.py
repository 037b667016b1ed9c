"""Pins for the oracle's unbounded gate variant, log a = -softplus(g).

Page "Kimi K3 发布核实与 Moonshot AI 主干架构演变", §3 "K3 对 Kimi Linear 的进一步
修改", bullet 1: K3 replaced Kimi Linear's unbounded negative-softplus
log-decay by the -5-bounded scaled sigmoid.  The oracle keeps the older gate
as an option so that a kernel for it (with range-safe sub-tiling) can be
checked; these pins fix it by closed forms, the independent chunked form and
a special case where every token stands alone.
"""
import math

import numpy as np
import pytest

import chunked_form
import oracle


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _inputs(rng, lengths, H, dk, dv, h0_std=None):
    T = sum(lengths)
    q = _unit(rng.standard_normal((T, H, dk)))
    k = _unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    g = rng.standard_normal((T, H, dk))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    h0 = None
    if h0_std is not None:
        h0 = rng.standard_normal((len(lengths), H, dk, dv)) * h0_std
    return q, k, v, g, beta, cu, h0


# closed forms: softplus(0) = ln 2; softplus(ln(e^c - 1)) = c
GATE_CASES = [
    (0.0, -math.log(2.0)),
    (math.log(math.e - 1.0), -1.0),
    (math.log(math.exp(2.0) - 1.0), -2.0),
    (math.log(math.exp(0.25) - 1.0), -0.25),
    (-np.inf, 0.0),
    (np.inf, -np.inf),
    (-745.0, -math.exp(-745.0)),      # log1p keeps the tiny value
    (800.0, -800.0),                  # no overflow for large g
]


def check_scalar_gate(fn):
    for g, want in GATE_CASES:
        got = fn(g)
        if math.isinf(want):
            assert got == want, (g, got)
        else:
            assert got == pytest.approx(want, rel=1e-15, abs=0.0), (g, got, want)


def test_scalar_gate_closed_forms():
    check_scalar_gate(oracle.log_alpha_softplus)


@pytest.mark.parametrize("mutant", [
    lambda g: math.log1p(math.exp(g)) if g < 700 else g,        # sign dropped
    lambda g: -1.0 / (1.0 + math.exp(-g)) if g > -700 else 0.0,  # sigmoid, not softplus
    lambda g: -math.log(math.exp(g)) if abs(g) < 700 else -g,    # log e^g: the 1 dropped
    lambda g: -5.0 * math.log1p(math.exp(g)) if g < 700 else -5.0 * g,  # K3's 5 carried over
])
def test_scalar_gate_pin_rejects_mutants(mutant):
    with pytest.raises(AssertionError):
        check_scalar_gate(mutant)


def test_pure_decay_matches_closed_forms():
    """beta = 0: hT = Diag(a) h0 with a = e^{-softplus(g)} per key channel."""
    gs = np.array([0.0, math.log(math.e - 1.0), -np.inf, np.inf, 3.0])
    a = np.array([0.5, math.exp(-1.0), 1.0, 0.0, 1.0 / (1.0 + math.exp(3.0))])
    dk, dv = 5, 3
    rng = np.random.default_rng(41)
    h0 = rng.standard_normal((1, 1, dk, dv))
    z = np.zeros
    _, hT = oracle.forward(z((1, 1, dk)), z((1, 1, dk)), z((1, 1, dv)),
                           gs.reshape(1, 1, dk), z((1, 1)), [0, 1], h0,
                           gate="softplus")
    np.testing.assert_allclose(hT[0, 0], a[:, None] * h0[0, 0], rtol=1e-14, atol=0)


@pytest.mark.parametrize("shift", [0.0, 6.0, -3.0])
def test_equals_independent_chunked_form(shift):
    """The token recurrence with the softplus gate equals the dense
    within-chunk form for chunks of 1, 7, 16 and the whole sequence, on a
    varlen batch with h0 and dk != dv; shift = 6 makes a 16-token tile decay
    past e^{-88} in most channels (the range the bounded gate avoids)."""
    rng = np.random.default_rng(42)
    lengths = [1, 16, 17, 40]
    q, k, v, g, beta, cu, h0 = _inputs(rng, lengths, 2, 7, 5, 0.3)
    g = g + shift
    o, hT = oracle.forward(q, k, v, g, beta, cu, h0, gate="softplus")
    for C in (1, 7, 16, max(lengths)):
        oc, hc = chunked_form.forward(q, k, v, g, beta, cu, h0, chunk=C,
                                      gate="softplus")
        np.testing.assert_allclose(o, oc, rtol=0, atol=1e-11)
        np.testing.assert_allclose(hT, hc, rtol=0, atol=1e-11)


def test_full_forgetting_makes_tokens_independent():
    """g = +inf in every channel gives a = 0: the state is wiped before each
    write, so S_t = beta_t k_t v_t^T and o_t = beta_t (q_t . k_t) v_t."""
    rng = np.random.default_rng(43)
    q, k, v, g, beta, cu, h0 = _inputs(rng, [6, 3], 2, 4, 3, 1.0)
    g[:] = np.inf
    o, hT = oracle.forward(q, k, v, g, beta, cu, h0, gate="softplus")
    want_o = beta[..., None] * np.sum(q * k, axis=-1)[..., None] * v
    np.testing.assert_allclose(o, want_o, rtol=0, atol=1e-14)
    for n, last in enumerate((5, 8)):
        for h in range(2):
            np.testing.assert_allclose(
                hT[n, h], beta[last, h] * np.outer(k[last, h], v[last, h]),
                rtol=0, atol=1e-14)


def test_default_gate_is_the_bounded_one():
    rng = np.random.default_rng(44)
    q, k, v, g, beta, cu, h0 = _inputs(rng, [9], 1, 4, 4, 0.5)
    a = oracle.forward(q, k, v, g, beta, cu, h0)
    b = oracle.forward(q, k, v, g, beta, cu, h0, gate="sigmoid5")
    c = oracle.forward(q, k, v, g, beta, cu, h0, gate="softplus")
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    assert np.abs(a[0] - c[0]).max() > 1e-3        # the gates differ
