"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device
memory (for example a serving engine that has reserved nearly all GPU memory
for its caches, or code that must not call cudaMalloc because it can
synchronise the device).  The long-sequence scratch comes from the library's
static device array instead of a caller workspace.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import pytest
import torch

import oracle
from gated_delta_rule_60_b200 import binding, inputs
from kda_testutil import TOL_BF16_O, TOL_BF16_S, rel_err

pytestmark = pytest.mark.gpu


def _segmented_inputs():
    # one long sequence, two heads: the segment-parallel path, which needs scratch
    T, H = 16384 + 77, 2
    need = binding.kda_chunk_fwd_workspace_size(1, T, H, 128, 128, torch.bfloat16)
    assert 0 < need <= 16 << 20
    return inputs.make_prefill([T], H, 128, 128, torch.bfloat16, seed=97, h0_std=0.02)


def test_noalloc_matches_workspace_entry_point_twice():
    inp = _segmented_inputs()
    d = {n: getattr(inp, n).cuda() for n in ("q", "k", "v", "g", "beta", "h0",
                                             "cu_seqlens")}
    o_ref, h_ref = binding.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                         d["h0"], d["cu_seqlens"])
    assert binding.kda_stream_status() == binding.KDA_OK
    # the same kernels on the same inputs: results must be bitwise equal
    for _ in range(2):   # two calls in a row share the static scratch
        o = torch.empty_like(o_ref)
        hT = torch.empty_like(h_ref)
        binding.kda_chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                      d["h0"], d["cu_seqlens"], o=o, hT=hT)
        assert binding.kda_stream_status() == binding.KDA_OK
        assert torch.equal(o, o_ref) and torch.equal(hT, h_ref)
    # and both match the fp64 oracle at the bf16 tolerance
    o_or, h_or = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens,
                                inp.h0)
    assert rel_err(o, o_or) <= TOL_BF16_O
    assert rel_err(hT, h_or) <= TOL_BF16_S


def test_noalloc_rejects_problems_beyond_the_static_scratch():
    """A problem whose scratch exceeds the 16 MiB array (here the 1M-token,
    16-head shape) is refused before any launch: the pointers below are
    never dereferenced."""
    lib = binding.load_library()
    T, H = 1 << 20, 16
    assert binding.kda_chunk_fwd_workspace_size(1, T, H, 128, 128, torch.bfloat16) > 16 << 20
    P = ctypes.c_void_p
    st = lib.kda_chunk_fwd_noalloc(P(256), P(256), P(256), P(256), P(256), None, None,
                                   1, T, H, 128, 128, binding.KDA_BF16, P(256), None, None)
    assert st == binding.KDA_ERR_WORKSPACE
