"""hT may alias h0 exactly (the header's in-place carry): a call whose final
states overwrite its initial states gives bitwise the same o and hT as a call
with separate buffers, on the chain path and on the segment-parallel path."""
import pytest
import torch

from gated_delta_rule_60_b200 import binding, inputs
from kda_testutil import to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,dim,lengths", [
    (torch.bfloat16, 128, [5, 40, 0, 77]),
    (torch.float32, 16, [5, 40, 0, 77]),
    (torch.bfloat16, 128, [16384 + 17]),        # segment-parallel path
])
def test_hT_may_alias_h0(dtype, dim, lengths):
    H = 2
    inp = inputs.make_prefill(lengths, H, dim, dim, dtype, seed=90, h0_std=0.02)
    d = to_device(inp)
    o1, h1 = binding.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                   d["h0"], d["cu_seqlens"])
    assert binding.kda_stream_status() == binding.KDA_OK
    state = d["h0"].clone()
    o2, h2 = binding.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                   state, d["cu_seqlens"], hT=state)
    assert binding.kda_stream_status() == binding.KDA_OK
    assert h2.data_ptr() == state.data_ptr()
    assert torch.equal(o1, o2)
    assert torch.equal(h1, state)
