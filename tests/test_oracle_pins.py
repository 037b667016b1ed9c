"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics.

Each pin is a function of an implementation ``impl(q,k,v,g,beta,cu,h0) ->
(o, hT)``.  The oracle must pass every pin; every planted mistake in
tests/oracle_mutants.py must fail at least one.  None of these re-types the
oracle's loop: they use closed forms, special cases, an independently written
chunked form, algebraic invariants and a hand-derived worked example.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import chunked_form
import oracle_mutants

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _oracle_impl(q, k, v, g, beta, cu, h0=None):
    return oracle.forward(q, k, v, g, beta, cu, h0)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_inputs(rng, lengths, H, dk, dv, h0_std=None):
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


# --------------------------------------------------------------------------
# Pins.  Each returns None on success and raises AssertionError otherwise.
# --------------------------------------------------------------------------

def pin_t1_closed_form(impl):
    """T=1 from S0=0: the decay acts on zero, so S = beta k v^T and
    o = S^T q = beta (q.k) v."""
    rng = np.random.default_rng(1)
    for dk, dv in ((4, 6), (16, 16), (8, 3)):
        q, k, v, g, beta, cu, _ = _rand_inputs(rng, [1], 2, dk, dv)
        o, hT = impl(q, k, v, g, beta, cu, None)
        for h in range(2):
            b = beta[0, h]
            np.testing.assert_allclose(
                o[0, h], b * np.dot(q[0, h], k[0, h]) * v[0, h],
                rtol=0, atol=1e-13)
            np.testing.assert_allclose(
                hT[0, h], b * np.outer(k[0, h], v[0, h]), rtol=0, atol=1e-13)


def pin_exact_retrieval(impl):
    """After a beta=1 write of a unit-norm key, from ANY prior state and any
    gate, the state maps that key exactly to its value: S^T k = v.  With q = k
    the read of the same token returns v."""
    rng = np.random.default_rng(2)
    for dk, dv in ((8, 5), (16, 16)):
        q, k, v, g, beta, cu, h0 = _rand_inputs(rng, [1], 3, dk, dv, 0.7)
        beta[:] = 1.0
        q = k.copy()
        o, hT = impl(q, k, v, g, beta, cu, h0)
        for h in range(3):
            np.testing.assert_allclose(hT[0, h].T @ k[0, h], v[0, h],
                                       rtol=0, atol=1e-12)
            np.testing.assert_allclose(o[0, h], v[0, h], rtol=0, atol=1e-12)


def pin_identity_no_write(impl):
    """alpha == 1 (g = -inf) and beta == 0: the state never changes and every
    read returns S0^T q_t (exact: only multiplications by 1 and adds of 0)."""
    rng = np.random.default_rng(3)
    q, k, v, g, beta, cu, h0 = _rand_inputs(rng, [5, 0, 9], 2, 6, 4, 1.0)
    g[:] = -np.inf
    beta[:] = 0.0
    o, hT = impl(q, k, v, g, beta, cu, h0)
    np.testing.assert_array_equal(hT, h0)
    for n in range(3):
        for t in range(cu[n], cu[n + 1]):
            for h in range(2):
                np.testing.assert_allclose(o[t, h], h0[n, h].T @ q[t, h],
                                           rtol=0, atol=1e-13)


def pin_gate_values(impl):
    """Pure decay (beta = 0) of a known state by a known gate:
    g = 0 -> a = e^-2.5; g = ln 3 -> sigmoid = 3/4, a = e^-3.75;
    g = -ln 3 -> a = e^-1.25; g = +inf -> a = e^-5; g = -inf -> a = 1.
    So hT = Diag(a) h0 with those closed-form factors."""
    gs = np.array([0.0, math.log(3.0), -math.log(3.0), np.inf, -np.inf])
    a = np.array([math.exp(-2.5), math.exp(-3.75), math.exp(-1.25),
                  math.exp(-5.0), 1.0])
    dk, dv = 5, 3
    rng = np.random.default_rng(4)
    h0 = rng.standard_normal((1, 1, dk, dv))
    q = np.zeros((1, 1, dk)); k = np.zeros((1, 1, dk))
    v = np.zeros((1, 1, dv)); beta = np.zeros((1, 1))
    g = gs.reshape(1, 1, dk)
    _, hT = impl(q, k, v, g, beta, np.array([0, 1]), h0)
    np.testing.assert_allclose(hT[0, 0], a[:, None] * h0[0, 0],
                               rtol=1e-14, atol=0)


def pin_chunked_form(impl):
    """Brute force: the token recurrence equals the independently written
    dense-within-chunk form for chunk lengths 1, 7, 16 and whole-sequence,
    on varlen batches with a carried state and dk != dv."""
    rng = np.random.default_rng(5)
    lengths = [1, 15, 16, 17, 40]
    q, k, v, g, beta, cu, h0 = _rand_inputs(rng, lengths, 2, 7, 5, 0.3)
    o, hT = impl(q, k, v, g, beta, cu, h0)
    for C in (1, 7, 16, max(lengths)):
        oc, hc = chunked_form.forward(q, k, v, g, beta, cu, h0, chunk=C)
        np.testing.assert_allclose(o, oc, rtol=0, atol=1e-11)
        np.testing.assert_allclose(hT, hc, rtol=0, atol=1e-11)


def pin_linearity(impl):
    """For fixed q, k, g, beta the map (S0, V) -> (O, S_T) is linear."""
    rng = np.random.default_rng(6)
    q, k, v1, g, beta, cu, h1 = _rand_inputs(rng, [12, 7], 2, 6, 5, 1.0)
    v2 = rng.standard_normal(v1.shape)
    h2 = rng.standard_normal(h1.shape)
    a, b = 0.7, -1.9
    o1, s1 = impl(q, k, v1, g, beta, cu, h1)
    o2, s2 = impl(q, k, v2, g, beta, cu, h2)
    o3, s3 = impl(q, k, a * v1 + b * v2, g, beta, cu, a * h1 + b * h2)
    np.testing.assert_allclose(o3, a * o1 + b * o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s3, a * s1 + b * s2, rtol=0, atol=1e-12)


def pin_orthonormal_keys(impl):
    """Classic delta rule on mutually orthonormal keys (alpha = 1, beta = 1,
    S0 = 0): no interference, so S_T = sum_i k_i v_i^T exactly."""
    rng = np.random.default_rng(7)
    dk, dv, T = 8, 6, 8
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm.T[:T].reshape(T, 1, dk)
    q = _unit(rng.standard_normal((T, 1, dk)))
    v = rng.standard_normal((T, 1, dv))
    g = np.full((T, 1, dk), -np.inf)
    beta = np.ones((T, 1))
    _, hT = impl(q, k, v, g, beta, np.array([0, T]), None)
    np.testing.assert_allclose(hT[0, 0], k[:, 0].T @ v[:, 0], rtol=0,
                               atol=1e-13)


def pin_scalar_gate_householder(impl):
    """A channel-constant gate reduces KDA to the gated delta rule, whose
    textbook form is S_t = a_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
    (a generalised Householder transition)."""
    rng = np.random.default_rng(8)
    dk, dv, T = 6, 4, 11
    q, k, v, g, beta, cu, h0 = _rand_inputs(rng, [T], 1, dk, dv, 0.5)
    g[:] = rng.standard_normal((T, 1, 1))
    o, hT = impl(q, k, v, g, beta, cu, h0)
    S = h0[0, 0].copy()
    for t in range(T):
        a = math.exp(-5.0 / (1.0 + math.exp(-g[t, 0, 0])))
        kt = k[t, 0]
        S = a * (np.eye(dk) - beta[t, 0] * np.outer(kt, kt)) @ S \
            + beta[t, 0] * np.outer(kt, v[t, 0])
        np.testing.assert_allclose(o[t, 0], S.T @ q[t, 0], rtol=0,
                                   atol=1e-12)
    np.testing.assert_allclose(hT[0, 0], S, rtol=0, atol=1e-12)


def pin_norm_bound(impl):
    """With unit keys and beta in [0,1], ||(I - beta k k^T) Diag(a)||_2 <= 1,
    so ||S_T||_2 <= ||S_0||_2 + sum_t beta_t ||v_t|| on a long run."""
    rng = np.random.default_rng(9)
    q, k, v, g, beta, cu, h0 = _rand_inputs(rng, [300], 1, 8, 8, 1.0)
    g = g - 6.0  # mostly slow decay so the state accumulates
    _, hT = impl(q, k, v, g, beta, cu, h0)
    bound = np.linalg.norm(h0[0, 0], 2) + np.sum(
        beta[:, 0] * np.linalg.norm(v[:, 0], axis=-1))
    assert np.linalg.norm(hT[0, 0], 2) <= bound * (1 + 1e-12)


def pin_hand_example(impl):
    """Hand-derived two-token worked example (tests/golden)."""
    with open(os.path.join(GOLDEN, "hand_two_tokens.json")) as f:
        fx = json.load(f)
    inp = {key: np.array(val, dtype=np.float64) if key != "cu_seqlens"
           else np.array(val, dtype=np.int64)
           for key, val in fx["inputs"].items()}
    o, hT = impl(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                 inp["cu_seqlens"], None)
    np.testing.assert_allclose(o, np.array(fx["expected"]["o"]), rtol=0,
                               atol=fx["tolerance_abs"])
    np.testing.assert_allclose(hT, np.array(fx["expected"]["hT"]), rtol=0,
                               atol=fx["tolerance_abs"])


PINS = [pin_t1_closed_form, pin_exact_retrieval, pin_identity_no_write,
        pin_gate_values, pin_chunked_form, pin_linearity,
        pin_orthonormal_keys, pin_scalar_gate_householder, pin_norm_bound,
        pin_hand_example]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_passes(pin):
    pin(_oracle_impl)


@pytest.mark.parametrize("mutation", oracle_mutants.MUTATIONS)
def test_pins_reject_mutant(mutation):
    def impl(q, k, v, g, beta, cu, h0=None):
        return oracle_mutants.forward(q, k, v, g, beta, cu, h0, mutation)
    failed = []
    for pin in PINS:
        if pin is pin_chunked_form:
            continue  # slow in pure numpy; the others suffice
        try:
            pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
        except (ValueError, IndexError):
            failed.append(pin.__name__)   # shape errors count as caught
    assert failed, "mutation %s passed every pin" % mutation


def test_unmutated_python_reference_passes():
    """The mutant harness itself, with no mutation, passes the pins, so a
    rejection above is caused by the planted mistake and nothing else."""
    def impl(q, k, v, g, beta, cu, h0=None):
        return oracle_mutants.forward(q, k, v, g, beta, cu, h0, None)
    for pin in PINS:
        if pin is not pin_chunked_form:
            pin(impl)


def test_decode_equals_one_token_prefill():
    rng = np.random.default_rng(10)
    B, H, dk, dv = 3, 2, 6, 5
    q, k, v, g, beta, _, _ = _rand_inputs(rng, [B], H, dk, dv)
    S = rng.standard_normal((B, H, dk, dv))
    o, S1 = oracle.decode(q.reshape(B, H, dk), k.reshape(B, H, dk),
                          v.reshape(B, H, dv), g.reshape(B, H, dk),
                          beta.reshape(B, H), S)
    cu = np.arange(B + 1)
    o2, S2 = oracle.forward(q, k, v, g, beta, cu, S)
    np.testing.assert_array_equal(o.reshape(B, H, dv), o2)
    np.testing.assert_array_equal(S1, S2)


def test_unit_mask_and_varlen_packing():
    """Packing is only bookkeeping: each sequence run alone gives the same
    result, and a unit mask computes only the selected units."""
    rng = np.random.default_rng(11)
    lengths = [3, 0, 20, 9]
    q, k, v, g, beta, cu, h0 = _rand_inputs(rng, lengths, 3, 4, 4, 0.5)
    o, hT = oracle.forward(q, k, v, g, beta, cu, h0)
    for n, L in enumerate(lengths):
        s, e = cu[n], cu[n + 1]
        o1, h1 = oracle.forward(q[s:e], k[s:e], v[s:e], g[s:e], beta[s:e],
                                [0, L], h0[n:n + 1])
        np.testing.assert_array_equal(o[s:e], o1)
        np.testing.assert_array_equal(hT[n:n + 1], h1)
    mask = np.zeros((4, 3), dtype=bool)
    mask[2, 1] = True
    om, hm = oracle.forward(q, k, v, g, beta, cu, h0, unit_mask=mask)
    np.testing.assert_array_equal(hm[2, 1], hT[2, 1])
    np.testing.assert_array_equal(om[cu[2]:cu[3], 1], o[cu[2]:cu[3], 1])
    assert np.isnan(hm[0, 0]).all()


def test_malformed_cu_seqlens_rejected():
    rng = np.random.default_rng(12)
    q, k, v, g, beta, cu, _ = _rand_inputs(rng, [4, 4], 1, 2, 2)
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, g, beta, [0, 5, 4], None)
