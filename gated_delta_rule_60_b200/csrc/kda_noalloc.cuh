// kda_noalloc.cuh -- kda_chunk_fwd for callers that cannot allocate device
// memory.  Included by kda_api.cu so that the static scratch array, the
// kernels that use it and the address lookup live in one translation unit.
//
// Who needs this: a serving engine that reserves almost all device memory
// for its own caches at start-up and has no pool left for a library's
// scratch; a plugin whose host owns the allocator and does not expose it;
// latency-sensitive code that must not call cudaMalloc because it can
// synchronise the device.  Such callers still pass every input and output;
// only the scratch the long-sequence path needs comes from the library.
#pragma once

#include <atomic>

namespace kda {
namespace noalloc {

// Library-owned scratch.  Every GPU that loads libkda holds this array until
// the process exits; all calls on a device share it.
constexpr size_t kScratchBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
static std::atomic<void *> g_scratch_addr[kMaxDevices];

// Device address of g_scratch on the current device, looked up once per
// device (the first call on a device does it; that first call should be
// made before any stream capture).  In host code `g_scratch` only names a
// host-side stand-in; kernels must be given this address instead.
inline void *scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void *ptr = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (ptr == nullptr) {
        if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess) return nullptr;
        g_scratch_addr[dev].store(ptr, std::memory_order_release);
    }
    return ptr;
}

}  // namespace noalloc
}  // namespace kda

extern "C" KDA_API kda_status kda_chunk_fwd_noalloc(
    const void *q, const void *k, const void *v, const void *g, const void *beta,
    const float *h0, const int32_t *cu_seqlens, int32_t N, int64_t T_tot, int32_t H,
    int32_t dk, int32_t dv, kda_dtype dt, void *o, float *hT, void *stream) {
    // Same argument rules as kda_chunk_fwd; the scratch the long-sequence
    // path needs must fit the static array.
    const size_t need = kda_chunk_fwd_workspace_size(N, T_tot, H, dk, dv, dt);
    if (need > kda::noalloc::kScratchBytes) {
        // validate the arguments first so a malformed call reports that instead
        const kda_status st = kda_chunk_fwd(q, k, v, g, beta, h0, cu_seqlens, N, T_tot, H, dk,
                                            dv, dt, o, hT, nullptr, 0, nullptr);
        return st == KDA_ERR_WORKSPACE ? KDA_ERR_WORKSPACE : st;
    }
    void *scratch = nullptr;
    if (need > 0) {
        scratch = kda::noalloc::scratch_address();
        if (scratch == nullptr) return KDA_ERR_CUDA;
    }
    return kda_chunk_fwd(q, k, v, g, beta, h0, cu_seqlens, N, T_tot, H, dk, dv, dt, o, hT,
                         scratch, need, stream);
}
