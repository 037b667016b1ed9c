"""Pins for the fp64 backward pass of the oracle (the gradient of the prefill).

The pages name training as the use of the chunked form ("Kimi K3 发布核实与
Moonshot AI 主干架构演变", §3 "KDA 为什么不同于 MLA", item 3); the backward is
fixed by the forward through calculus.  Each pin is a function of an
implementation impl(q, k, v, g, beta, cu, h0, d_o, d_hT) -> dict and uses
something other than the chain rule it checks: central differences of the
(separately pinned) forward oracle, the adjoint identity of the linear map
(h0, V) -> (O, hT), and closed forms for one token and for a frozen state.
Every planted mistake in tests/oracle_backward_mutants.py must fail a pin.
"""
import numpy as np
import pytest

import oracle
import oracle_backward_mutants as bm


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _inputs(rng, lengths, H, dk, dv, h0_std=0.5):
    T = sum(lengths)
    q = _unit(rng.standard_normal((T, H, dk)))
    k = _unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    g = rng.standard_normal((T, H, dk))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    h0 = rng.standard_normal((len(lengths), H, dk, dv)) * h0_std
    return q, k, v, g, beta, cu, h0


def _oracle_bwd(q, k, v, g, beta, cu, h0, d_o, d_hT):
    return oracle.backward(q, k, v, g, beta, cu, h0, d_o, d_hT)


def _loss(q, k, v, g, beta, cu, h0, d_o, d_hT):
    o, hT = oracle.forward(q, k, v, g, beta, cu, h0)
    return float(np.sum(o * d_o) + np.sum(hT * d_hT))


# --------------------------------------------------------------------------
# Pins
# --------------------------------------------------------------------------

def pin_finite_differences(impl):
    """Central differences of the forward oracle, for every entry of every
    input, on a varlen batch with an empty sequence and a 70-token one."""
    rng = np.random.default_rng(21)
    lengths = [3, 0, 70]
    q, k, v, g, beta, cu, h0 = _inputs(rng, lengths, 2, 3, 2)
    d_o = rng.standard_normal(v.shape)
    d_hT = rng.standard_normal(h0.shape)
    got = impl(q, k, v, g, beta, cu, h0, d_o, d_hT)
    args = dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0)
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "beta": "dbeta", "h0": "dh0"}
    eps = 1e-6
    for name, grad in names.items():
        x = args[name]
        num = np.zeros_like(x)
        flat = x.reshape(-1)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + eps
            lp = _loss(cu=cu, d_o=d_o, d_hT=d_hT, **args)
            flat[i] = keep - eps
            lm = _loss(cu=cu, d_o=d_o, d_hT=d_hT, **args)
            flat[i] = keep
            num.reshape(-1)[i] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(got[grad], num, rtol=0, atol=2e-8,
                                   err_msg=grad)


def pin_adjoint_identity(impl):
    """For fixed q, k, g, beta the map (h0, V) -> (O, hT) is linear, so its
    adjoint satisfies <dO, O> + <dhT, hT> = <dh0, h0> + <dV, V>."""
    rng = np.random.default_rng(22)
    q, k, v, g, beta, cu, h0 = _inputs(rng, [40, 17], 2, 8, 6)
    d_o = rng.standard_normal(v.shape)
    d_hT = rng.standard_normal(h0.shape)
    o, hT = oracle.forward(q, k, v, g, beta, cu, h0)
    got = impl(q, k, v, g, beta, cu, h0, d_o, d_hT)
    lhs = np.sum(d_o * o) + np.sum(d_hT * hT)
    rhs = np.sum(got["dh0"] * h0) + np.sum(got["dv"] * v)
    assert abs(lhs - rhs) <= 1e-11 * (abs(lhs) + 1.0), (lhs, rhs)


def pin_one_token_closed_form(impl):
    """T = 1 from S0: with S' = Diag(a) S0, r = S'^T k, u = beta (v - r),
    S_1 = S' + k u^T, o = S_1^T q and L = <do, o> + <D, S_1>, the gradient is
    written out by hand (G = D + q do^T is dL/dS_1, du = G^T k):
      dq = S_1 do,  dv = beta du,  dbeta = du.(v - r),
      dk = G u - beta S' du,  dS0 = Diag(a) (G - beta k du^T),
      dg_i = a_i (-5 s_i (1 - s_i)) sum_j (G - beta k du^T)_ij S0_ij."""
    rng = np.random.default_rng(23)
    dk_, dv_ = 5, 4
    q, k, v, g, beta, cu, h0 = _inputs(rng, [1], 1, dk_, dv_)
    d_o = rng.standard_normal(v.shape)
    D = rng.standard_normal(h0.shape)
    got = impl(q, k, v, g, beta, cu, h0, d_o, D)
    s = 1.0 / (1.0 + np.exp(-g[0, 0]))
    a = np.exp(-5.0 * s)
    S0 = h0[0, 0]
    Sp = a[:, None] * S0
    kk, vv, qq, b = k[0, 0], v[0, 0], q[0, 0], beta[0, 0]
    r = Sp.T @ kk
    u = b * (vv - r)
    S1 = Sp + np.outer(kk, u)
    G = D[0, 0] + np.outer(qq, d_o[0, 0])
    du = G.T @ kk
    Gp = G - b * np.outer(kk, du)
    want = {
        "dq": S1 @ d_o[0, 0],
        "dv": b * du,
        "dbeta": du @ (vv - r),
        "dk": G @ u - b * (Sp @ du),
        "dh0": a[:, None] * Gp,
        "dg": a * (-5.0 * s * (1.0 - s)) * np.sum(Gp * S0, axis=1),
    }
    for name, w in want.items():
        np.testing.assert_allclose(np.reshape(got[name], -1), np.reshape(w, -1),
                                   rtol=0, atol=1e-13, err_msg=name)


def pin_frozen_state(impl):
    """alpha = 1 (g = -inf) and beta = 0 freeze the state at S0, so
    o_t = S0^T q_t and, with G_t = dhT + sum_{s >= t} q_s do_s^T:
    dq_t = S0 do_t, dk = dv = dg = 0, dbeta_t = (G_t^T k_t).(v_t - S0^T k_t),
    dh0 = G_first."""
    rng = np.random.default_rng(24)
    T, dk_, dv_ = 9, 4, 3
    q, k, v, g, beta, cu, h0 = _inputs(rng, [T], 1, dk_, dv_)
    g[:] = -np.inf
    beta[:] = 0.0
    d_o = rng.standard_normal(v.shape)
    D = rng.standard_normal(h0.shape)
    got = impl(q, k, v, g, beta, cu, h0, d_o, D)
    S0 = h0[0, 0]
    G = D[0, 0].copy()
    for t in range(T - 1, -1, -1):
        G = G + np.outer(q[t, 0], d_o[t, 0])
        np.testing.assert_allclose(got["dq"][t, 0], S0 @ d_o[t, 0], rtol=0, atol=1e-13)
        want_b = (G.T @ k[t, 0]) @ (v[t, 0] - S0.T @ k[t, 0])
        np.testing.assert_allclose(got["dbeta"][t, 0], want_b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["dh0"][0, 0], G, rtol=0, atol=1e-12)
    for name in ("dk", "dv", "dg"):
        np.testing.assert_array_equal(got[name], 0.0, err_msg=name)


PINS = [pin_finite_differences, pin_adjoint_identity, pin_one_token_closed_form,
        pin_frozen_state]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_backward_passes(pin):
    pin(_oracle_bwd)


def _mutant_impl(mutation):
    def impl(q, k, v, g, beta, cu, h0, d_o, d_hT):
        return bm.backward(q, k, v, g, beta, cu, h0, d_o, d_hT, mutation)
    return impl


@pytest.mark.parametrize("mutation", bm.MUTATIONS)
def test_backward_pins_reject_mutant(mutation):
    impl = _mutant_impl(mutation)
    failed = []
    for pin in PINS:
        if pin is pin_finite_differences:
            continue   # slow through the numpy harness; the others suffice
        try:
            pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, "mutation %s passed every backward pin" % mutation


def test_unmutated_backward_harness_passes():
    impl = _mutant_impl(None)
    for pin in PINS:
        if pin is not pin_finite_differences:
            pin(impl)


def test_backward_without_upstream_terms():
    """No d_o and no d_hT: every gradient is zero; d_o alone and d_hT alone
    add up to the gradient of their sum (the backward is linear in them)."""
    rng = np.random.default_rng(25)
    q, k, v, g, beta, cu, h0 = _inputs(rng, [6, 11], 2, 4, 4)
    zero = oracle.backward(q, k, v, g, beta, cu, h0)
    for val in zero.values():
        np.testing.assert_array_equal(val, 0.0)
    d_o = rng.standard_normal(v.shape)
    d_hT = rng.standard_normal(h0.shape)
    a = oracle.backward(q, k, v, g, beta, cu, h0, d_o=d_o)
    b = oracle.backward(q, k, v, g, beta, cu, h0, d_hT=d_hT)
    c = oracle.backward(q, k, v, g, beta, cu, h0, d_o, d_hT)
    for name in c:
        np.testing.assert_allclose(a[name] + b[name], c[name], rtol=0, atol=1e-12)


def test_backward_checkpoint_boundaries():
    """Sequences of 63, 64, 65 and 129 tokens (around the 64-token
    checkpoints of the reverse sweep) agree with the numpy restatement."""
    rng = np.random.default_rng(26)
    q, k, v, g, beta, cu, h0 = _inputs(rng, [63, 64, 65, 129], 1, 4, 3)
    d_o = rng.standard_normal(v.shape)
    d_hT = rng.standard_normal(h0.shape)
    got = oracle.backward(q, k, v, g, beta, cu, h0, d_o, d_hT)
    ref = bm.backward(q, k, v, g, beta, cu, h0, d_o, d_hT, None)
    for name in got:
        np.testing.assert_allclose(got[name], ref[name], rtol=0, atol=1e-12,
                                   err_msg=name)
