"""No kernel writes outside its outputs: o, hT and the decode state live in
the middle of larger buffers whose margins hold a sentinel, and after each
call the margins are unchanged while the outputs still match the oracle.
The cases are chosen around the places where a store could run over: partial
32-token steps, empty sequences, the segment-parallel path with a ragged last
segment, and ragged head counts in the decode."""
import pytest
import torch

from gated_delta_rule_60_b200 import binding, inputs
from guard_bands import guarded, margins_intact
from kda_testutil import oracle_forward, rel_err, to_device, tolerances
import oracle

SENTINEL = 12352.0        # exact in bf16 and fp32


def test_margin_check_catches_an_overrun():
    """The check itself, on the CPU: writes inside the view leave the margins
    intact; one element past either end is caught."""
    for dtype in (torch.bfloat16, torch.float32):
        buf, view = guarded((10, 3, 4), dtype, SENTINEL, "cpu")
        assert view.is_contiguous() and view.data_ptr() % 16 == 0
        view.fill_(1.0)
        assert margins_intact(buf, SENTINEL)
        flat = buf.view(-1)
        first = view.storage_offset()
        last = first + view.numel() - 1
        for idx in (first - 1, last + 1):
            keep = flat[idx].clone()
            flat[idx] = 0.0
            assert not margins_intact(buf, SENTINEL)
            flat[idx] = keep
        assert margins_intact(buf, SENTINEL)


def _prefill_guarded(inp):
    d = to_device(inp)
    T, H, dv = inp.v.shape
    N = inp.cu_seqlens.numel() - 1
    dk = inp.k.shape[-1]
    obuf, o = guarded((T, H, dv), inp.v.dtype, SENTINEL, "cuda")
    hbuf, hT = guarded((N, H, dk, dv), torch.float32, SENTINEL, "cuda")
    binding.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"],
                          d["cu_seqlens"], o=o, hT=hT)
    assert binding.kda_stream_status() == binding.KDA_OK
    return obuf, o, hbuf, hT


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,dim", [(torch.bfloat16, 128), (torch.float32, 16)])
def test_prefill_stays_inside_its_outputs(dtype, dim):
    lengths = [1, 15, 31, 0, 32, 33, 47, 64, 100]
    inp = inputs.make_prefill(lengths, 3, dim, dim, dtype, seed=80, h0_std=0.02)
    obuf, o, hbuf, hT = _prefill_guarded(inp)
    assert margins_intact(obuf, SENTINEL) and margins_intact(hbuf, SENTINEL)
    o_ref, h_ref = oracle_forward(inp)
    tol_o, tol_s = tolerances(dtype)
    assert rel_err(o, o_ref) <= tol_o and rel_err(hT, h_ref) <= tol_s


@pytest.mark.gpu
def test_segmented_prefill_stays_inside_its_outputs():
    """One 16,401-token sequence on 2 heads takes the segment-parallel path
    (local pass, combine, final pass) with a ragged last segment."""
    T, H = 16384 + 17, 2
    assert binding.kda_chunk_fwd_workspace_size(1, T, H, 128, 128, torch.bfloat16) > 0
    inp = inputs.make_prefill([T], H, 128, 128, torch.bfloat16, seed=81)
    obuf, o, hbuf, hT = _prefill_guarded(inp)
    assert margins_intact(obuf, SENTINEL) and margins_intact(hbuf, SENTINEL)
    o_ref, h_ref = oracle_forward(inp)
    tol_o, tol_s = tolerances(torch.bfloat16)
    assert rel_err(o, o_ref) <= tol_o and rel_err(hT, h_ref) <= tol_s


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,dim", [(torch.bfloat16, 128), (torch.float32, 16)])
def test_decode_stays_inside_its_outputs(dtype, dim):
    B, H = 5, 3
    x = inputs.make_decode_step(B, H, dim, dim, dtype, seed=82)
    S = inputs.make_state(B, H, dim, dim, std=0.5, seed=83)
    sbuf, Sd = guarded((B, H, dim, dim), torch.float32, SENTINEL, "cuda")
    Sd.copy_(S.cuda())
    obuf, o = guarded((B, H, dim), dtype, SENTINEL, "cuda")
    binding.kda_decode_step(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.g.cuda(),
                            x.beta.cuda(), Sd, o=o)
    assert binding.kda_stream_status() == binding.KDA_OK
    assert margins_intact(sbuf, SENTINEL) and margins_intact(obuf, SENTINEL)
    o_ref, S_ref = oracle.decode(x.q, x.k, x.v, x.g, x.beta, S)
    tol_o, tol_s = tolerances(dtype)
    assert rel_err(o, o_ref) <= tol_o and rel_err(Sd, S_ref) <= tol_s
