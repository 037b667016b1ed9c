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
