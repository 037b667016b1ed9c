"""The range claim behind reciprocal decay scaling (page "Kimi K3 发布核实与
Moonshot AI 主干架构演变", "K3 对 Kimi Linear 的进一步修改", bullet 1).

log a = -5 sigmoid(g) lies in [-5, 0], so the cumulative log-decay b over a
16-token tile lies in [-80, 0].  e^{+-80} is inside the bf16 normal range
(2^-126 .. 3.39e38), so a tile's keys and queries scaled by e^{b} or e^{-b}
stay finite in bf16; over 32 tokens the same scaling would overflow.

The tensor-core prefill advances the state in 32-token steps and centres the
exponents on the end of the first tile, m = b_15 (0-based row 15): every
scaled exponent b_r - m then stays within one tile's range, |b_r - m| <= 80.
These tests check those facts in fp64 and through torch's bf16 rounding; they
use no code of the library.
"""
import math

import numpy as np
import pytest
import torch

BF16_MAX = 3.3895313892515355e38      # (2 - 2^-7) * 2^127
BF16_MIN_NORMAL = 2.0 ** -126


def log_decay(g):
    return -5.0 / (1.0 + np.exp(-g))


def to_bf16(x):
    with np.errstate(over="ignore"):            # fp32 overflow to inf is checked
        x32 = np.ascontiguousarray(x, dtype=np.float32)
    return torch.from_numpy(x32).to(torch.bfloat16)


def gates(kind, rng, rows, d):
    if kind == "normal":
        return rng.standard_normal((rows, d))
    if kind == "max_decay":
        return np.full((rows, d), np.inf)
    if kind == "no_decay":
        return np.full((rows, d), -np.inf)
    if kind == "mixed_extremes":
        return rng.choice([np.inf, -np.inf, 0.0, 30.0, -30.0], size=(rows, d))
    raise ValueError(kind)


KINDS = ["normal", "max_decay", "no_decay", "mixed_extremes"]


def test_gate_bounds_closed_form():
    g = np.array([-np.inf, -50.0, -1.0, 0.0, 1.0, 50.0, np.inf])
    la = log_decay(g)
    assert la[0] == 0.0 and la[-1] == -5.0 and la[3] == -2.5
    assert np.all(la <= 0.0) and np.all(la >= -5.0)
    assert np.all(np.diff(la) <= 0.0)          # monotone in g
    # one full tile at the strongest decay reaches the bound exactly
    assert np.sum(np.full(16, -5.0)) == -80.0
    # and that bound is inside the bf16 normal range on both sides
    assert BF16_MIN_NORMAL < math.exp(-80.0) and math.exp(80.0) < BF16_MAX
    assert math.exp(90.0) > BF16_MAX           # 18 tokens at -5 would not fit


@pytest.mark.parametrize("kind", KINDS)
def test_step_centering_keeps_one_tile_range(kind):
    """Per key channel over a 32-token step: b_r - b_15 lies in [-80, 80]
    (rows 16..31 add at most one tile of decay, rows 0..14 undo at most 15
    tokens of it), and the scaled unit-norm keys / queries are finite in bf16."""
    rng = np.random.default_rng(31)
    d = 128
    for _ in range(8):
        b = np.cumsum(log_decay(gates(kind, rng, 32, d)), axis=0)
        e = b - b[15]
        assert e.max() <= 75.0 + 1e-9 and e.min() >= -80.0 - 1e-9
        k = rng.standard_normal((32, d))
        k /= np.linalg.norm(k, axis=1, keepdims=True)
        for x in (k * np.exp(e), k * np.exp(-e)):
            xb = to_bf16(x)
            assert torch.isfinite(xb).all()
        # the step decays themselves: eps = e^{b_15}, delta = e^{b_31 - b_15}
        for f in (np.exp(b[15]), np.exp(b[31] - b[15])):
            fb = to_bf16(f).float().numpy()
            assert np.all(fb >= BF16_MIN_NORMAL) and np.all(fb <= 1.0)


def test_uncentred_step_overflows():
    """The converse: without centring, a 32-token step at the strongest decay
    needs e^{160} for the reciprocal scaling, which bf16 cannot hold; a
    16-token tile without centring (e^{80}) still fits."""
    b32 = np.cumsum(np.full(32, -5.0))
    b16 = b32[:16]
    assert not torch.isfinite(to_bf16(np.exp(-b32))).all()
    assert torch.isfinite(to_bf16(np.exp(-b16))).all()
    # and the forward scaling underflows to zero past one tile
    assert (to_bf16(np.exp(b32)).float() == 0).any()
    assert (to_bf16(np.exp(b16)).float() > 0).all()


def lost(x):
    """Entries that are non-zero in fp64 but below the bf16 normal range
    after rounding (flushed to zero or left subnormal)."""
    a = to_bf16(x).float().abs().numpy()
    return int(((a < BF16_MIN_NORMAL) & (x != 0)).sum())


def test_lost_precision_centred_vs_absolute():
    """Strongest decay over a 32-token step, unit-norm queries (d = 128):
    absolute scaling q e^{b} pushes almost every component past the first
    tile below the bf16 normal range, while scaling relative to m = b_15
    loses only components smaller than e^{80} 2^-126 (about 6.5e-4 of the row
    norm) in the last row, the same as one uncentred tile."""
    rng = np.random.default_rng(32)
    d = 128
    q = rng.standard_normal((32, d))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    b = np.cumsum(np.full((32, d), -5.0), axis=0)
    absolute = q * np.exp(b)
    centred = q * np.exp(b - b[15])
    assert lost(absolute[16:]) >= 0.9 * 16 * d
    assert lost(absolute[:16]) <= 0.02 * 16 * d
    expect = int((np.abs(centred) < BF16_MIN_NORMAL).sum())
    assert lost(centred) <= 0.01 * 32 * d
    assert abs(lost(centred) - expect) <= 2
    assert lost(centred[:31]) == 0


def test_unbounded_gate_breaks_the_tile_range():
    """The gate K3 replaced, log a = -softplus(g), has no lower bound: from
    g of about 5.6 upwards one 16-token tile decays past e^{-88.7}, so the
    reciprocal factor e^{-b} of that tile no longer fits bf16, while the
    bounded gate stays at e^{80} for any g."""
    softplus = lambda x: np.log1p(np.exp(x))
    g = np.array([0.0, 3.0, 5.6, 8.0, 30.0])
    tile = 16 * softplus(g)                       # -b over one tile
    assert np.all(tile[2:] > math.log(BF16_MAX)) and np.all(tile[:2] < 80.0)
    assert not torch.isfinite(to_bf16(np.exp(tile[2:]))).any()
    bounded = -16 * log_decay(np.array([0.0, 5.6, 30.0, np.inf]))
    assert np.all(bounded <= 80.0)
    assert torch.isfinite(to_bf16(np.exp(bounded))).all()
