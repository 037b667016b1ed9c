"""libkda: the Kimi Delta Attention (KDA) operator on NVIDIA B200 (sm_100a).

The operator lives in a C-ABI CUDA library (include/kda.h, built in-tree as
gated_delta_rule_60_b200/libkda.so).  This package holds its ctypes binding
(names identical to the C entry points), the in-tree build script, and the
seeded synthetic input generator.  Importing the package does not load the
library; the first call of a binding function does, and raises if the library
is missing.
"""
from .binding import (KdaError, kda_chunk_fwd, kda_chunk_fwd_workspace_size,  # noqa: F401
                      kda_decode_step, kda_status_string, kda_stream_status,
                      kda_version, load_library)
