"""Pins for the oracle's prologue (short convolution, L2 norm, beta sigmoid)
and output gate: closed forms, a library convolution, causality and
sequence independence; planted mistakes in the convolution must fail them.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import layer_ops


def _conv_inputs(rng, lengths, H=2, d=3):
    T = sum(lengths)
    x = rng.standard_normal((T, H, d))
    w = rng.standard_normal((H, d, layer_ops.CONV_TAPS))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return x, w, cu


LENGTHS = [5, 0, 1, 9, 3]


def pin_conv_identity_and_lags(conv):
    rng = np.random.default_rng(51)
    x, w, cu = _conv_inputs(rng, LENGTHS)
    for j in range(layer_ops.CONV_TAPS):
        wj = np.zeros_like(w)
        wj[..., j] = 1.0
        y = conv(x, wj, cu)
        want = np.zeros_like(x)
        for n in range(len(LENGTHS)):
            s, e = cu[n], cu[n + 1]
            want[s + j:e] = x[s:e - j] if e - j > s else want[s + j:e]
        np.testing.assert_array_equal(y, want)


def pin_conv_library(conv):
    """Per (head, channel) and sequence: the first L terms of the full
    discrete convolution of the sequence with the filter (numpy.convolve)."""
    rng = np.random.default_rng(52)
    x, w, cu = _conv_inputs(rng, LENGTHS)
    y = conv(x, w, cu)
    for n in range(len(LENGTHS)):
        s, e = cu[n], cu[n + 1]
        if e == s:
            continue
        for h in range(x.shape[1]):
            for c in range(x.shape[2]):
                full = np.convolve(x[s:e, h, c], w[h, c], mode="full")
                np.testing.assert_allclose(y[s:e, h, c], full[:e - s], rtol=0, atol=1e-14)


def pin_conv_causal_and_local(conv):
    """Changing token t of one sequence changes only tokens t .. t+3 of that
    sequence."""
    rng = np.random.default_rng(53)
    x, w, cu = _conv_inputs(rng, LENGTHS)
    y = conv(x, w, cu)
    for t in range(int(cu[-1])):
        x2 = x.copy()
        x2[t] += 1.0
        changed = np.any(conv(x2, w, cu) != y, axis=(1, 2))
        n = int(np.searchsorted(cu, t, side="right") - 1)
        allowed = np.zeros(int(cu[-1]), dtype=bool)
        allowed[t:min(t + layer_ops.CONV_TAPS, int(cu[n + 1]))] = True
        assert not np.any(changed & ~allowed), t


CONV_PINS = [pin_conv_identity_and_lags, pin_conv_library, pin_conv_causal_and_local]


@pytest.mark.parametrize("pin", CONV_PINS, ids=lambda p: p.__name__)
def test_oracle_conv_passes(pin):
    pin(layer_ops.short_conv)


def _mutant_conv(kind):
    def conv(x, w, cu):
        x, w = np.asarray(x, float), np.asarray(w, float)
        cu = [int(c) for c in cu]
        y = np.zeros_like(x)
        for n in range(len(cu) - 1):
            s, e = cu[n], cu[n + 1]
            lo = 0 if kind == "history_leaks" else s
            for t in range(s, e):
                for j in range(4):
                    src = t + j if kind == "anticausal" else t - j
                    tap = 3 - j if kind == "taps_reversed" else j
                    if lo <= src < (e if kind == "anticausal" else t + 1):
                        y[t] += w[:, :, tap] * x[src]
        return y
    return conv


@pytest.mark.parametrize("kind", ["taps_reversed", "history_leaks", "anticausal"])
def test_conv_pins_reject_mutant(kind):
    conv = _mutant_conv(kind)
    failed = []
    for pin in CONV_PINS:
        try:
            pin(conv)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, kind


def test_l2_normalize():
    rng = np.random.default_rng(54)
    x = rng.standard_normal((7, 2, 5))
    x[3, 1] = 0.0
    y = oracle.l2_normalize(x)
    n = np.linalg.norm(y, axis=-1)
    np.testing.assert_allclose(np.delete(n.reshape(-1), 7), 1.0, rtol=0, atol=1e-15)
    np.testing.assert_array_equal(y[3, 1], 0.0)
    np.testing.assert_allclose(y * np.linalg.norm(x, axis=-1, keepdims=True), x,
                               rtol=0, atol=1e-14)


def test_prologue_composition_and_beta():
    rng = np.random.default_rng(55)
    lengths = [4, 6]
    xq, wq, cu = _conv_inputs(rng, lengths, H=2, d=4)
    xk, wk, _ = _conv_inputs(rng, lengths, H=2, d=4)
    xv, wv, _ = _conv_inputs(rng, lengths, H=2, d=3)
    b_raw = np.zeros((10, 2))
    b_raw[0, 0], b_raw[1, 0], b_raw[2, 0], b_raw[3, 0] = math.log(3.0), np.inf, -np.inf, -math.log(3.0)
    q, k, v, beta = oracle.prologue(xq, xk, xv, wq, wk, wv, b_raw, cu)
    np.testing.assert_allclose(beta[:4, 0], [0.75, 1.0, 0.0, 0.25], rtol=1e-15, atol=0)
    np.testing.assert_array_equal(beta[4:, :], 0.5)
    np.testing.assert_allclose(np.linalg.norm(q, axis=-1), 1.0, rtol=0, atol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(k, axis=-1), 1.0, rtol=0, atol=1e-14)
    np.testing.assert_array_equal(v, layer_ops.short_conv(xv, wv, cu))
    # the prologue's outputs drive the operator directly
    g = rng.standard_normal(q.shape)
    o, hT = oracle.forward(q, k, v[..., :3], g, beta, cu)
    assert np.isfinite(o).all() and np.isfinite(hT).all()


def test_output_gate_closed_forms():
    o = np.array([[[2.0, -4.0, 8.0, 1.0, 3.0]]])
    z = np.array([[[0.0, math.log(3.0), -math.log(3.0), np.inf, -np.inf]]])
    np.testing.assert_allclose(oracle.output_gate(o, z),
                               [[[1.0, -3.0, 2.0, 1.0, 0.0]]], rtol=1e-15, atol=0)


def test_output_gate_on_the_one_token_closed_form():
    """T = 1 from S0 = 0: gated o = beta (q.k) v * sigmoid(z)."""
    rng = np.random.default_rng(56)
    q, k = (rng.standard_normal((1, 2, 4)) for _ in range(2))
    v, z = (rng.standard_normal((1, 2, 3)) for _ in range(2))
    g = rng.standard_normal((1, 2, 4))
    beta = np.array([[0.3, 0.9]])
    o, _ = oracle.forward(q, k, v, g, beta, [0, 1])
    want = beta[..., None] * np.sum(q * k, -1)[..., None] * v / (1.0 + np.exp(-z))
    np.testing.assert_allclose(oracle.output_gate(o, z), want, rtol=0, atol=1e-14)
