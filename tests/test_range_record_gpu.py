"""The bf16 range claim of the bounded gate, recorded on the tensor-core
kernel itself (page "Kimi K3 发布核实与 Moonshot AI 主干架构演变", §3 "K3 对
Kimi Linear 的进一步修改", bullet 1: reciprocal decay scaling inside a
16-token tile stays within the BF16 range).

kda_debug_range_prefill makes the first chain of the next prefill record one
step's scaled operands as the gate pass writes them (Kr, Qr, Kh in bf16) and
Z = Kh^T T before the delta rescale (fp32).  For normal, maximal, mixed and
slow decay the record must hold no non-finite value, stay below the bf16 and
fp32 maxima, and its maxima of Kr, Qr, Kh must equal the same quantities
computed in fp64 from the inputs (the step's cumulative log-decay b and its
centre m = b_15) within bf16 rounding.  The record is printed; the
measured figures are quoted in the design notes."""
import numpy as np
import pytest
import torch

from gated_delta_rule_60_b200 import binding, inputs

pytestmark = pytest.mark.gpu

T, H, STEP = 512, 2, 3
BF16_MAX = 3.3895313892515355e38


def _gate(kind, g):
    if kind == "normal":
        return g
    if kind == "max_decay":
        return torch.full_like(g, 30.0)
    if kind == "mixed":
        vals = torch.tensor([-float("inf"), -30.0, 0.0, 30.0, float("inf")])
        idx = torch.randint(0, 5, g.shape, generator=torch.Generator().manual_seed(9))
        return vals[idx].to(g.dtype)
    if kind == "slow":
        return g - 12.0
    raise ValueError(kind)


def _expected_max(inp, g):
    """max |Kr|, |Qr|, |Kh| of head 0, step STEP, in fp64."""
    sl = slice(32 * STEP, 32 * STEP + 32)
    k = inp.k[sl, 0].double().numpy()
    q = inp.q[sl, 0].double().numpy()
    gg = g[sl, 0].double().numpy()
    la = -5.0 / (1.0 + np.exp(-gg))                     # log decay, natural log
    b = np.cumsum(la, axis=0)
    m = b[15]
    er = np.exp(b - m)
    return {"Kr": np.abs(k * er).max(), "Qr": np.abs(q * er).max(), "Kh": np.abs(k / er).max()}


@pytest.mark.parametrize("kind", ["normal", "max_decay", "mixed", "slow"])
def test_range_record(kind):
    inp = inputs.make_prefill([T], H, 128, 128, torch.bfloat16, seed=410)
    g = _gate(kind, inp.g)
    c = lambda t: t.cuda()
    binding.kda_debug_range_prefill(STEP)
    o, hT = binding.kda_chunk_fwd(c(inp.q), c(inp.k), c(inp.v), c(g), c(inp.beta), None,
                                  c(inp.cu_seqlens))
    assert binding.kda_stream_status() == binding.KDA_OK
    rec = binding.kda_debug_range_read()
    print("range record", kind, {r: {k: "%.4g" % v for k, v in d.items()} for r, d in rec.items()})
    for row in ("Kr", "Qr", "Kh", "Z"):
        assert rec[row]["count"] == 4096, (row, rec[row])
        assert rec[row]["nonfinite"] == 0, (row, rec[row])
        assert np.isfinite(rec[row]["max_abs"]), (row, rec[row])
    for row in ("Kr", "Qr", "Kh"):
        assert rec[row]["max_abs"] < BF16_MAX
    assert rec["Z"]["max_abs"] < 3.4e38
    exp = _expected_max(inp, g)
    for row in ("Kr", "Qr", "Kh"):
        assert rec[row]["max_abs"] == pytest.approx(exp[row], rel=1e-2), (row, rec[row], exp[row])
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
