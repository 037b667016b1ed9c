"""Failure detection without a fault: a bounded wait that runs out is
reported through the status word, the word is cleared once read, and the
context stays usable for the next call."""
import pytest
import torch

from gated_delta_rule_60_b200 import binding, inputs
from kda_testutil import oracle_forward, rel_err, to_device, tolerances

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_is_reported_and_cleared():
    assert binding.kda_stream_status() == binding.KDA_OK
    binding.kda_selftest_wait_timeout(2_000_000)          # about a millisecond
    assert binding.kda_stream_status() == binding.KDA_ERR_TIMEOUT
    assert binding.kda_stream_status() == binding.KDA_OK  # read and cleared
    # the context still runs the operator correctly
    inp = inputs.make_prefill([45, 70], 2, 128, 128, torch.bfloat16, seed=95, h0_std=0.02)
    d = to_device(inp)
    o, hT = binding.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"],
                                  d["cu_seqlens"])
    assert binding.kda_stream_status() == binding.KDA_OK
    o_ref, h_ref = oracle_forward(inp)
    tol_o, tol_s = tolerances(torch.bfloat16)
    assert rel_err(o, o_ref) <= tol_o and rel_err(hT, h_ref) <= tol_s


@pytest.mark.parametrize("stall_step", [0, 3])
def test_prefill_pipeline_wait_that_runs_out_drains_and_reports(stall_step):
    """The prefill's own failure path, with no fault: the scan of every CTA
    waits at a chosen step on a barrier nothing arrives on, with a short
    bound.  The wait gives up; the kernel reports KDA_ERR_TIMEOUT once, every
    role leaves its loop, the CTA drains its copies, stores and tensor-core
    products and frees its tensor memory.  Nothing is written outside o and
    hT, and the next call on the same context matches the oracle."""
    from guard_bands import guarded, margins_intact
    sentinel = 12352.0
    inp = inputs.make_prefill([300, 45, 200], 2, 128, 128, torch.bfloat16, seed=96,
                              h0_std=0.02)
    d = to_device(inp)
    T, H = inp.v.shape[0], inp.v.shape[1]
    obuf, o = guarded((T, H, 128), torch.bfloat16, sentinel, "cuda")
    hbuf, hT = guarded((3, H, 128, 128), torch.float32, sentinel, "cuda")
    assert binding.kda_stream_status() == binding.KDA_OK
    binding.kda_debug_stall_prefill(stall_step, 4_000_000)   # about 2 ms of SM clock
    binding.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"],
                          d["cu_seqlens"], o=o, hT=hT)
    assert binding.kda_stream_status() == binding.KDA_ERR_TIMEOUT
    assert binding.kda_stream_status() == binding.KDA_OK     # read and cleared
    assert margins_intact(obuf, sentinel) and margins_intact(hbuf, sentinel)
    # the setting was consumed by that call: this one runs normally
    binding.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"],
                          d["cu_seqlens"], o=o, hT=hT)
    assert binding.kda_stream_status() == binding.KDA_OK
    assert margins_intact(obuf, sentinel) and margins_intact(hbuf, sentinel)
    o_ref, h_ref = oracle_forward(inp)
    tol_o, tol_s = tolerances(torch.bfloat16)
    assert rel_err(o, o_ref) <= tol_o and rel_err(hT, h_ref) <= tol_s
