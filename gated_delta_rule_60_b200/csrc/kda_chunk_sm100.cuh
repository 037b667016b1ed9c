// kda_chunk_sm100.cuh -- tcgen05 chunked prefill (bf16, d = 128).  In progress.
#pragma once
#include "kda_common.cuh"
#include "../../include/kda.h"

namespace kda {
inline size_t sm100_workspace_bytes(int, int64_t, int) { return 0; }
template <typename F>
inline kda_status sm100_chunk_fwd_or(F fallback) { return fallback(); }
}  // namespace kda
