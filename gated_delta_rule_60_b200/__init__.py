"""libkda: the Kimi Delta Attention (KDA) operator on NVIDIA B200 (sm_100a).

The operator lives in a C-ABI CUDA library (include/kda.h, built in-tree as
gated_delta_rule_60_b200/libkda.so).  This package holds its ctypes binding
(names identical to the C entry points), the in-tree build script, and the
seeded synthetic input generator.  Importing the package does not load the
library; the first call of a binding function does, and raises if the library
is missing.
"""
from .binding import (KdaError, kda_chunk_bwd, kda_chunk_bwd_workspace_size,  # noqa: F401
                      kda_chunk_fwd, kda_chunk_fwd_gated, kda_chunk_fwd_noalloc,
                      kda_chunk_fwd_softplus, kda_chunk_fwd_workspace_size,
                      kda_debug_range_prefill, kda_debug_range_read,
                      kda_debug_stall_prefill, kda_decode_step, kda_decode_step_softplus,
                      kda_prologue, kda_selftest_wait_timeout, kda_status_string,
                      kda_stream_status, kda_version, load_library)
