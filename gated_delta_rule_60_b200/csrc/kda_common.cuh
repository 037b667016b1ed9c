// kda_common.cuh -- small device helpers shared by the libkda kernels.
//
// The KDA gate: log a = -5 * sigmoid(g), the bounded scaled sigmoid of the
// page "Kimi K3 发布核实与 Moonshot AI 主干架构演变", §3 "K3 对 Kimi Linear
// 的进一步修改", bullet 1.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Per-device status word.  Kernels OR error bits into it; the host reads and
// clears it in kda_stream_status().
enum : unsigned { kErrSeqlens = 1u, kErrTimeout = 2u };
__device__ unsigned int g_status_word;

// kda_stream_status() takes the word with one atomic exchange on the device,
// so a bit set by a kernel on another stream is never lost between a read
// and a clear.  Each call gets its own slot for the value it took.
constexpr int kStatusSlots = 64;
__device__ unsigned int g_status_taken[kStatusSlots];

__global__ void status_take_kernel(int slot) {
    g_status_taken[slot] = atomicExch(&g_status_word, 0u);
}

__device__ __forceinline__ void raise_error(unsigned bit) {
    atomicOr(&g_status_word, bit);
}

constexpr float kLog2e = 1.4426950408889634f;

// Natural-log decay of one gate value, fp32, accurate to a few ulp.
// g = -inf gives 0 (no decay), g = +inf gives -5.
__device__ __forceinline__ float log_decay(float g) {
    float e = exp2f(-g * kLog2e);
    return -5.0f / (1.0f + e);
}

// Output gate o * sigmoid(z) (page "Kimi K3 发布核实与 Moonshot AI 主干架构演变",
// §3 "K3 对 Kimi Linear 的进一步修改", bullet 2: a full-rank, input-dependent
// channel gate on the output).  z = -inf gives 0, z = +inf gives 1.
__device__ __forceinline__ float out_gate(float z) {
    return 1.0f / (1.0f + __expf(-z));
}

// The unbounded gate of Kimi Linear that K3 replaced (same page, same bullet):
// log a = -softplus(g), in fp32, stable for every g (g = +inf gives -inf,
// g = -inf gives 0).
__device__ __forceinline__ float log_decay_softplus(float g) {
    return -(fmaxf(g, 0.f) + log1pf(expf(-fabsf(g))));
}

template <typename T>
struct IO;

template <>
struct IO<float> {
    static __device__ __forceinline__ float ld(const float *p) { return *p; }
    static __device__ __forceinline__ void st(float *p, float x) { *p = x; }
};

template <>
struct IO<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16 *p) {
        return __bfloat162float(*p);
    }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, float x) {
        *p = __float2bfloat16_rn(x);
    }
};

// Reads the bounds of sequence n.  Returns false (and raises the status bit)
// when they are malformed; the caller then skips the sequence.
__device__ __forceinline__ bool seq_bounds(const int32_t *cu, int n, int N,
                                           int64_t T_tot, int64_t &start,
                                           int64_t &end) {
    if (cu == nullptr) {
        int64_t L = T_tot / N;
        start = (int64_t)n * L;
        end = start + L;
        return true;
    }
    start = cu[n];
    end = cu[n + 1];
    bool ok = start >= 0 && end >= start && end <= T_tot;
    if (n == 0) ok = ok && start == 0;
    if (n == N - 1) ok = ok && end == T_tot;
    if (!ok) raise_error(kErrSeqlens);
    return ok;
}

}  // namespace kda
