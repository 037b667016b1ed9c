"""Property-based pins of the fp64 oracle (CPU; hypothesis draws the cases).

Random packed batches (any lengths, 0 included), head counts, key and value
sizes (dk != dv allowed), gate values from the whole real line with the
infinities, write strengths in [0, 1] and carried states.  For each draw:

  * the oracle equals the independently written chunked form
    (tests/chunked_form.py: dense within a chunk, every decay ratio formed
    directly) at a random chunk length, for the K3 gate and for the
    unbounded softplus gate;
  * the map (S0, V) -> (O, S_T) is linear: the result for a S0 + b V equals
    a times the result for (S0, 0) plus b times the result for (0, V);
  * packing is invisible: a batch gives, sequence by sequence, exactly what
    separate one-sequence calls give.

The draws are derandomised, so a run is repeatable.
"""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import chunked_form
import oracle

SETTINGS = settings(max_examples=60, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow])


@st.composite
def batches(draw):
    N = draw(st.integers(1, 4))
    lengths = draw(st.lists(st.integers(0, 37), min_size=N, max_size=N))
    H = draw(st.integers(1, 3))
    dk = draw(st.integers(1, 9))
    dv = draw(st.integers(1, 9))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    T = sum(lengths)

    def unit(x):
        n = np.linalg.norm(x, axis=-1, keepdims=True)
        return x / np.where(n > 0, n, 1.0)

    q = unit(rng.standard_normal((T, H, dk)))
    k = unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    # gates: mostly N(0, 3^2), some entries at the extremes
    g = 3.0 * rng.standard_normal((T, H, dk))
    if T:
        extreme = rng.random((T, H, dk)) < draw(st.sampled_from([0.0, 0.1, 0.5]))
        g[extreme] = rng.choice([np.inf, -np.inf, 40.0, -40.0], size=int(extreme.sum()))
    beta = rng.random((T, H))
    if T:
        beta[rng.random((T, H)) < 0.1] = draw(st.sampled_from([0.0, 1.0]))
    h0 = draw(st.sampled_from([None, 0.1, 1.0]))
    if h0 is not None:
        h0 = h0 * rng.standard_normal((N, H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    chunk = draw(st.sampled_from([1, 3, 5, 16, 40]))
    return q, k, v, g, beta, cu, h0, chunk


def _close(x, ref, tol):
    scale = max(np.max(np.abs(ref)) if ref.size else 0.0, 1.0)
    assert np.all(np.isfinite(x)) and np.all(np.isfinite(ref))
    assert np.max(np.abs(x - ref)) <= tol * scale if ref.size else True


@SETTINGS
@given(batches(), st.sampled_from(["sigmoid5", "softplus"]))
def test_oracle_equals_the_chunked_form(batch, gate):
    q, k, v, g, beta, cu, h0, chunk = batch
    if gate == "softplus":
        # the chunked form subtracts cumulative log-decays, and -inf - (-inf)
        # is undefined; a decay of e^-1000 per token is as complete in fp64
        # (full forgetting at g = +inf is pinned by its closed form elsewhere)
        g = np.where(g == np.inf, 1000.0, g)
    o, hT = oracle.forward(q, k, v, g, beta, cu, h0, gate=gate)
    o_c, hT_c = chunked_form.forward(q, k, v, g, beta, cu, h0, chunk=chunk, gate=gate)
    _close(o, o_c, 1e-10)
    _close(hT, hT_c, 1e-10)


@SETTINGS
@given(batches(), st.floats(-3, 3), st.floats(-3, 3))
def test_linear_in_state_and_values(batch, a, b):
    q, k, v, g, beta, cu, h0, _ = batch
    N, H, dk, dv = len(cu) - 1, q.shape[1], q.shape[2], v.shape[2]
    S0 = np.ones((N, H, dk, dv)) if h0 is None else h0
    o_s, h_s = oracle.forward(q, k, np.zeros_like(v), g, beta, cu, S0)
    o_v, h_v = oracle.forward(q, k, v, g, beta, cu, None)
    o, hT = oracle.forward(q, k, b * v, g, beta, cu, a * S0)
    _close(o, a * o_s + b * o_v, 1e-11)
    _close(hT, a * h_s + b * h_v, 1e-11)


@SETTINGS
@given(batches())
def test_packing_is_invisible(batch):
    q, k, v, g, beta, cu, h0, _ = batch
    o, hT = oracle.forward(q, k, v, g, beta, cu, h0)
    for n in range(len(cu) - 1):
        s, e = int(cu[n]), int(cu[n + 1])
        o1, h1 = oracle.forward(q[s:e], k[s:e], v[s:e], g[s:e], beta[s:e],
                                np.array([0, e - s]), None if h0 is None else h0[n:n + 1])
        assert np.array_equal(o[s:e], o1)
        assert np.array_equal(hT[n:n + 1], h1)


@SETTINGS
@given(batches())
def test_backward_adjoint_identity(batch):
    """(h0, V) -> (O, hT) is linear, so its gradient is its adjoint:
    <dO, O> + <dhT, hT> = <dh0, h0> + <dV, V> for any dO, dhT."""
    q, k, v, g, beta, cu, h0, _ = batch
    N, H, dk, dv = len(cu) - 1, q.shape[1], q.shape[2], v.shape[2]
    rng = np.random.default_rng(int(cu[-1]) + 7 * N + dk)
    h0 = rng.standard_normal((N, H, dk, dv)) if h0 is None else h0
    d_o = rng.standard_normal(v.shape)
    d_hT = rng.standard_normal((N, H, dk, dv))
    o, hT = oracle.forward(q, k, v, g, beta, cu, h0)
    gr = oracle.backward(q, k, v, g, beta, cu, h0=h0, d_o=d_o, d_hT=d_hT)
    lhs = np.sum(d_o * o) + np.sum(d_hT * hT)
    rhs = np.sum(gr["dh0"] * h0) + np.sum(gr["dv"] * v)
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs))


@SETTINGS
@given(batches())
def test_backward_directional_derivative(batch):
    """Along a random direction in every input at once, the central
    difference of L = <dO, O> + <dhT, hT> matches the gradient's inner
    product with the direction (finite gates, beta inside (0, 1))."""
    q, k, v, g, beta, cu, h0, _ = batch
    N, H, dk, dv = len(cu) - 1, q.shape[1], q.shape[2], v.shape[2]
    g = np.clip(np.nan_to_num(g, posinf=6.0, neginf=-6.0), -6.0, 6.0)
    beta = np.clip(beta, 0.05, 0.95)
    rng = np.random.default_rng(int(cu[-1]) + 11 * H + dv)
    h0 = 0.3 * rng.standard_normal((N, H, dk, dv)) if h0 is None else h0
    d_o = rng.standard_normal(v.shape)
    d_hT = rng.standard_normal((N, H, dk, dv))
    x = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "h0": h0}
    dx = {n: rng.standard_normal(a.shape) for n, a in x.items()}

    def loss(eps):
        y = {n: x[n] + eps * dx[n] for n in x}
        o, hT = oracle.forward(y["q"], y["k"], y["v"], y["g"], y["beta"], cu, y["h0"])
        return np.sum(d_o * o) + np.sum(d_hT * hT)

    gr = oracle.backward(q, k, v, g, beta, cu, h0=h0, d_o=d_o, d_hT=d_hT)
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "beta": "dbeta", "h0": "dh0"}
    analytic = sum(np.sum(gr[names[n]] * dx[n]) for n in x)
    eps = 1e-5
    numeric = (loss(eps) - loss(-eps)) / (2 * eps)
    scale = max(1.0, abs(analytic), sum(np.sum(np.abs(gr[names[n]] * dx[n])) for n in x))
    assert abs(numeric - analytic) <= 1e-6 * scale, (numeric, analytic)
