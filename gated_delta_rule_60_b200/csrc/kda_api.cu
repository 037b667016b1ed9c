// kda_api.cu -- the C ABI of libkda: argument checks, dispatch, launches.
//
// One translation unit holds every kernel so that the per-device status word
// (kda_common.cuh) is a single symbol.  See include/kda.h for the contract of
// each entry point.
#include <cstring>
#include "../../include/kda.h"

#include "kda_common.cuh"
#include "kda_decode.cuh"
#include "kda_chunk_simt.cuh"
#include "kda_chunk_sm100.cuh"
#include "kda_prologue.cuh"
#include "kda_backward.cuh"

#include <cuda_runtime.h>

#include <atomic>

namespace {

inline bool aligned16(const void *p) {
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// Largest T_tot of the bf16 d = 128 path: the last 32-token box must start
// below 2^31.
constexpr int64_t kMaxTokensSm100 = 0x7fffffc0;

inline bool supported_simt_d(int d) {
    return d == 16 || d == 32 || d == 64 || d == 128;
}

template <typename T, int D, bool kSoftplus = false>
kda_status launch_simt(const void *q, const void *k, const void *v,
                       const void *g, const void *beta, const float *h0,
                       const int32_t *cu, int N, int64_t T_tot, int H,
                       const void *z, void *o, float *hT, cudaStream_t s) {
    const size_t smem = sizeof(kda::SimtSmem<D>);
    auto kern = kda::chunk_fwd_simt_kernel<T, D, kSoftplus>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return KDA_ERR_CUDA;
    kern<<<(unsigned)(N * H), 256, smem, s>>>(
        (const T *)q, (const T *)k, (const T *)v, (const T *)g,
        (const T *)beta, h0, cu, N, (long)T_tot, H, (const T *)z, (T *)o, hT);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

template <typename T, bool kSoftplus = false>
kda_status dispatch_simt(int d, const void *q, const void *k, const void *v,
                         const void *g, const void *beta, const float *h0,
                         const int32_t *cu, int N, int64_t T_tot, int H,
                         const void *z, void *o, float *hT, cudaStream_t s) {
    switch (d) {
    case 16: return launch_simt<T, 16, kSoftplus>(q, k, v, g, beta, h0, cu, N, T_tot, H, z, o, hT, s);
    case 32: return launch_simt<T, 32, kSoftplus>(q, k, v, g, beta, h0, cu, N, T_tot, H, z, o, hT, s);
    case 64: return launch_simt<T, 64, kSoftplus>(q, k, v, g, beta, h0, cu, N, T_tot, H, z, o, hT, s);
    case 128: return launch_simt<T, 128, kSoftplus>(q, k, v, g, beta, h0, cu, N, T_tot, H, z, o, hT, s);
    default: return KDA_ERR_UNSUPPORTED;
    }
}

template <typename T, int D>
kda_status launch_prologue(const void *xq, const void *xk, const void *xv, const float *wq,
                           const float *wk, const float *wv, const void *braw, const int32_t *cu,
                           int N, int64_t T_tot, int H, void *q, void *k, void *v, void *beta,
                           cudaStream_t s) {
    using Sh = kda::pro::Shape<D>;
    const int64_t blocks = (T_tot + Sh::kTokPerBlock - 1) / Sh::kTokPerBlock;
    const dim3 grid((unsigned)blocks, (unsigned)H, 3);
    kda::pro::prologue_kernel<T, D><<<grid, kda::pro::kThreads, 0, s>>>(
        (const T *)xq, (const T *)xk, (const T *)xv, wq, wk, wv, (const T *)braw, cu, N, T_tot, H,
        (T *)q, (T *)k, (T *)v, (T *)beta);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

template <typename T>
kda_status dispatch_prologue(int d, const void *xq, const void *xk, const void *xv,
                             const float *wq, const float *wk, const float *wv, const void *braw,
                             const int32_t *cu, int N, int64_t T_tot, int H, void *q, void *k,
                             void *v, void *beta, cudaStream_t s) {
    switch (d) {
    case 16: return launch_prologue<T, 16>(xq, xk, xv, wq, wk, wv, braw, cu, N, T_tot, H, q, k, v, beta, s);
    case 32: return launch_prologue<T, 32>(xq, xk, xv, wq, wk, wv, braw, cu, N, T_tot, H, q, k, v, beta, s);
    case 64: return launch_prologue<T, 64>(xq, xk, xv, wq, wk, wv, braw, cu, N, T_tot, H, q, k, v, beta, s);
    case 128: return launch_prologue<T, 128>(xq, xk, xv, wq, wk, wv, braw, cu, N, T_tot, H, q, k, v, beta, s);
    default: return KDA_ERR_UNSUPPORTED;
    }
}

template <typename T, int D>
kda_status launch_bwd(const void *q, const void *k, const void *v, const void *g,
                      const void *beta, const float *h0, const int32_t *cu, int N, int64_t T_tot,
                      int H, const void *dO, const float *dhT, void *dq, void *dk, void *dv,
                      void *dg, void *dbeta, float *dh0, void *ws, cudaStream_t s) {
    const size_t smem = sizeof(kda::bwd::Smem<D>);
    auto kern = kda::bwd::chunk_bwd_kernel<T, D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return KDA_ERR_CUDA;
    const size_t DD = (size_t)D * D;
    float *ckpt = static_cast<float *>(ws);
    float *tok = ckpt + (size_t)H * ((T_tot + kda::bwd::kChunk - 1) / kda::bwd::kChunk + N) * DD;
    kern<<<(unsigned)(N * H), kda::bwd::threads_of<D>(), smem, s>>>(
        (const T *)q, (const T *)k, (const T *)v, (const T *)g, (const T *)beta, h0, cu, N, T_tot,
        H, (const T *)dO, dhT, (T *)dq, (T *)dk, (T *)dv, (T *)dg, (T *)dbeta, dh0, ckpt, tok);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

template <typename T>
kda_status dispatch_bwd(int d, const void *q, const void *k, const void *v, const void *g,
                        const void *beta, const float *h0, const int32_t *cu, int N,
                        int64_t T_tot, int H, const void *dO, const float *dhT, void *dq,
                        void *dk, void *dv, void *dg, void *dbeta, float *dh0, void *ws,
                        cudaStream_t s) {
    switch (d) {
    case 16: return launch_bwd<T, 16>(q, k, v, g, beta, h0, cu, N, T_tot, H, dO, dhT, dq, dk, dv, dg, dbeta, dh0, ws, s);
    case 32: return launch_bwd<T, 32>(q, k, v, g, beta, h0, cu, N, T_tot, H, dO, dhT, dq, dk, dv, dg, dbeta, dh0, ws, s);
    case 64: return launch_bwd<T, 64>(q, k, v, g, beta, h0, cu, N, T_tot, H, dO, dhT, dq, dk, dv, dg, dbeta, dh0, ws, s);
    case 128: return launch_bwd<T, 128>(q, k, v, g, beta, h0, cu, N, T_tot, H, dO, dhT, dq, dk, dv, dg, dbeta, dh0, ws, s);
    default: return KDA_ERR_UNSUPPORTED;
    }
}

template <typename T, int D, int SPLIT, bool kSoftplus = false>
kda_status launch_decode(const void *q, const void *k, const void *v,
                         const void *g, const void *beta, float *S, void *o,
                         long units, cudaStream_t s) {
    using Sh = kda::DecodeShape<D, SPLIT>;
    const long blocks = (units + Sh::kHeadsPerBlock - 1) / Sh::kHeadsPerBlock;
    kda::decode_step_kernel<T, D, SPLIT, kSoftplus><<<(unsigned)blocks, Sh::kThreads, 0, s>>>(
        (const T *)q, (const T *)k, (const T *)v, (const T *)g,
        (const T *)beta, S, (T *)o, units);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

template <typename T, bool kSoftplus = false>
kda_status dispatch_decode(int d, const void *q, const void *k, const void *v,
                           const void *g, const void *beta, float *S, void *o,
                           long units, cudaStream_t s) {
    switch (d) {
    case 16: return launch_decode<T, 16, 1, kSoftplus>(q, k, v, g, beta, S, o, units, s);
    case 32: return launch_decode<T, 32, 1, kSoftplus>(q, k, v, g, beta, S, o, units, s);
    case 64: return launch_decode<T, 64, 1, kSoftplus>(q, k, v, g, beta, S, o, units, s);
    case 128:
        kda::decode_step_d128_kernel<T, kSoftplus><<<(unsigned)units, kda::kDecode128Threads, 0, s>>>(
            (const T *)q, (const T *)k, (const T *)v, (const T *)g, (const T *)beta, S, (T *)o);
        return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    default: return KDA_ERR_UNSUPPORTED;
    }
}

}  // namespace

extern "C" {

int32_t kda_version(void) { return 10100; }

const char *kda_status_string(kda_status s) {
    switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case KDA_ERR_UNSUPPORTED: return "unsupported dtype, head size or length";
    case KDA_ERR_WORKSPACE: return "workspace missing or too small";
    case KDA_ERR_CUDA: return "CUDA runtime error";
    case KDA_ERR_TIMEOUT: return "a kernel's bounded wait ran out";
    case KDA_ERR_BAD_SEQLENS: return "malformed cu_seqlens";
    }
    return "unknown status";
}

size_t kda_chunk_fwd_workspace_size(int32_t N, int64_t T_tot, int32_t H,
                                    int32_t dk, int32_t dv, kda_dtype dt) {
    if (N <= 0 || T_tot < 0 || H <= 0 || dk != dv) return 0;
    if (dt == KDA_BF16 && dk == 128)
        return kda::sm100_workspace_bytes(N, T_tot, H);
    return 0;
}

static kda_status chunk_fwd_impl(const void *q, const void *k, const void *v,
                                 const void *g, const void *beta, const float *h0,
                                 const int32_t *cu_seqlens, int32_t N, int64_t T_tot,
                                 int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                                 const void *z, void *o, float *hT, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    if (N < 0 || T_tot < 0 || H <= 0) return KDA_ERR_INVALID_ARGUMENT;
    if (dt != KDA_BF16 && dt != KDA_FP32) return KDA_ERR_UNSUPPORTED;
    if (dk != dv || !supported_simt_d(dk)) return KDA_ERR_UNSUPPORTED;
    // The tensor-core path addresses tokens with signed 32-bit TMA coordinates.
    if (dt == KDA_BF16 && dk == 128 && T_tot > kMaxTokensSm100) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return T_tot == 0 ? KDA_OK : KDA_ERR_INVALID_ARGUMENT;
    if (cu_seqlens == nullptr && (T_tot % N) != 0) return KDA_ERR_INVALID_ARGUMENT;
    if ((int64_t)N * H > 0x7fffffff) return KDA_ERR_INVALID_ARGUMENT;
    if (T_tot > 0) {
        const void *req[] = {q, k, v, g, beta, o};
        for (const void *p : req)
            if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
        if (z && !aligned16(z)) return KDA_ERR_INVALID_ARGUMENT;
    }
    if ((h0 && !aligned16(h0)) || (hT && !aligned16(hT)) ||
        (cu_seqlens && !aligned16(cu_seqlens)))
        return KDA_ERR_INVALID_ARGUMENT;
    const size_t ws_need = kda_chunk_fwd_workspace_size(N, T_tot, H, dk, dv, dt);
    if (ws_need > 0 && (workspace == nullptr || workspace_bytes < ws_need ||
                        (reinterpret_cast<uintptr_t>(workspace) & 255u)))
        return KDA_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    if (dt == KDA_BF16 && dk == 128)
        return T_tot == 0 && hT == nullptr
                   ? KDA_OK
                   : kda::sm100_chunk_fwd(q, k, v, g, beta, h0, cu_seqlens, N, T_tot, H,
                                          z, o, hT, workspace, s);
    if (dt == KDA_BF16)
        return dispatch_simt<__nv_bfloat16>(dk, q, k, v, g, beta, h0, cu_seqlens,
                                            N, T_tot, H, z, o, hT, s);
    return dispatch_simt<float>(dk, q, k, v, g, beta, h0, cu_seqlens, N, T_tot,
                                H, z, o, hT, s);
}

kda_status kda_chunk_fwd(const void *q, const void *k, const void *v,
                         const void *g, const void *beta, const float *h0,
                         const int32_t *cu_seqlens, int32_t N, int64_t T_tot,
                         int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                         void *o, float *hT, void *workspace,
                         size_t workspace_bytes, void *stream) {
    return chunk_fwd_impl(q, k, v, g, beta, h0, cu_seqlens, N, T_tot, H, dk, dv, dt, nullptr,
                          o, hT, workspace, workspace_bytes, stream);
}

kda_status kda_chunk_fwd_gated(const void *q, const void *k, const void *v,
                               const void *g, const void *beta, const float *h0,
                               const int32_t *cu_seqlens, int32_t N, int64_t T_tot,
                               int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                               const void *z, void *o, float *hT, void *workspace,
                               size_t workspace_bytes, void *stream) {
    if (T_tot > 0 && z == nullptr) return KDA_ERR_INVALID_ARGUMENT;
    return chunk_fwd_impl(q, k, v, g, beta, h0, cu_seqlens, N, T_tot, H, dk, dv, dt, z, o, hT,
                          workspace, workspace_bytes, stream);
}

kda_status kda_chunk_fwd_softplus(const void *q, const void *k, const void *v,
                                  const void *g, const void *beta, const float *h0,
                                  const int32_t *cu_seqlens, int32_t N, int64_t T_tot,
                                  int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                                  void *o, float *hT, void *stream) {
    if (N < 0 || T_tot < 0 || H <= 0) return KDA_ERR_INVALID_ARGUMENT;
    if (dt != KDA_BF16 && dt != KDA_FP32) return KDA_ERR_UNSUPPORTED;
    if (dk != dv || !supported_simt_d(dk)) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return T_tot == 0 ? KDA_OK : KDA_ERR_INVALID_ARGUMENT;
    if (cu_seqlens == nullptr && (T_tot % N) != 0) return KDA_ERR_INVALID_ARGUMENT;
    if ((int64_t)N * H > 0x7fffffff) return KDA_ERR_INVALID_ARGUMENT;
    if (T_tot > 0) {
        const void *req[] = {q, k, v, g, beta, o};
        for (const void *p : req)
            if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
    }
    if ((h0 && !aligned16(h0)) || (hT && !aligned16(hT)) ||
        (cu_seqlens && !aligned16(cu_seqlens)))
        return KDA_ERR_INVALID_ARGUMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (dt == KDA_BF16)
        return dispatch_simt<__nv_bfloat16, true>(dk, q, k, v, g, beta, h0, cu_seqlens, N, T_tot,
                                                  H, nullptr, o, hT, s);
    return dispatch_simt<float, true>(dk, q, k, v, g, beta, h0, cu_seqlens, N, T_tot, H,
                                      nullptr, o, hT, s);
}

static kda_status decode_impl(const void *q, const void *k, const void *v, const void *g,
                              const void *beta, float *S, void *o, int32_t B, int32_t H,
                              int32_t dk, int32_t dv, kda_dtype dt, bool softplus,
                              void *stream) {
    if (B < 0 || H <= 0) return KDA_ERR_INVALID_ARGUMENT;
    if (dt != KDA_BF16 && dt != KDA_FP32) return KDA_ERR_UNSUPPORTED;
    if (dk != dv || !supported_simt_d(dk)) return KDA_ERR_UNSUPPORTED;
    if (B == 0) return KDA_OK;
    if ((int64_t)B * H > 0x7fffffff) return KDA_ERR_INVALID_ARGUMENT;
    const void *req[] = {q, k, v, g, beta, S, o};
    for (const void *p : req)
        if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const long units = (long)B * H;
    if (softplus)
        return dt == KDA_BF16
                   ? dispatch_decode<__nv_bfloat16, true>(dk, q, k, v, g, beta, S, o, units, s)
                   : dispatch_decode<float, true>(dk, q, k, v, g, beta, S, o, units, s);
    if (dt == KDA_BF16)
        return dispatch_decode<__nv_bfloat16>(dk, q, k, v, g, beta, S, o, units, s);
    return dispatch_decode<float>(dk, q, k, v, g, beta, S, o, units, s);
}

kda_status kda_decode_step(const void *q, const void *k, const void *v,
                           const void *g, const void *beta, float *S, void *o,
                           int32_t B, int32_t H, int32_t dk, int32_t dv,
                           kda_dtype dt, void *stream) {
    return decode_impl(q, k, v, g, beta, S, o, B, H, dk, dv, dt, false, stream);
}

kda_status kda_decode_step_softplus(const void *q, const void *k, const void *v,
                                    const void *g, const void *beta, float *S, void *o,
                                    int32_t B, int32_t H, int32_t dk, int32_t dv,
                                    kda_dtype dt, void *stream) {
    return decode_impl(q, k, v, g, beta, S, o, B, H, dk, dv, dt, true, stream);
}

size_t kda_chunk_bwd_workspace_size(int32_t N, int64_t T_tot, int32_t H, int32_t dk,
                                    int32_t dv, kda_dtype dt) {
    if (N <= 0 || T_tot < 0 || H <= 0 || dk != dv || !supported_simt_d(dk)) return 0;
    if (dt != KDA_BF16 && dt != KDA_FP32) return 0;
    const size_t DD = (size_t)dk * dk;
    const size_t ck = (size_t)H * ((size_t)(T_tot + kda::bwd::kChunk - 1) / kda::bwd::kChunk + N);
    const size_t tok = (size_t)N * H * kda::bwd::kChunk;
    return (ck + tok) * DD * sizeof(float);
}

kda_status kda_chunk_bwd(const void *q, const void *k, const void *v, const void *g,
                         const void *beta, const float *h0, const int32_t *cu_seqlens,
                         int32_t N, int64_t T_tot, int32_t H, int32_t dk, int32_t dv,
                         kda_dtype dt, const void *dO, const float *dhT, void *dq, void *dk_,
                         void *dv_, void *dg, void *dbeta, float *dh0, void *workspace,
                         size_t workspace_bytes, void *stream) {
    if (N < 0 || T_tot < 0 || H <= 0) return KDA_ERR_INVALID_ARGUMENT;
    if (dt != KDA_BF16 && dt != KDA_FP32) return KDA_ERR_UNSUPPORTED;
    if (dk != dv || !supported_simt_d(dk)) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return T_tot == 0 ? KDA_OK : KDA_ERR_INVALID_ARGUMENT;
    if (cu_seqlens == nullptr && (T_tot % N) != 0) return KDA_ERR_INVALID_ARGUMENT;
    if ((int64_t)N * H > 0x7fffffff) return KDA_ERR_INVALID_ARGUMENT;
    if (T_tot > 0) {
        const void *req[] = {q, k, v, g, beta, dO, dq, dk_, dv_, dg, dbeta};
        for (const void *p : req)
            if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
    }
    if ((h0 && !aligned16(h0)) || (dhT && !aligned16(dhT)) || (dh0 && !aligned16(dh0)) ||
        (cu_seqlens && !aligned16(cu_seqlens)))
        return KDA_ERR_INVALID_ARGUMENT;
    const size_t need = kda_chunk_bwd_workspace_size(N, T_tot, H, dk, dv, dt);
    if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return KDA_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (dt == KDA_BF16)
        return dispatch_bwd<__nv_bfloat16>(dk, q, k, v, g, beta, h0, cu_seqlens, N, T_tot, H, dO,
                                           dhT, dq, dk_, dv_, dg, dbeta, dh0, workspace, s);
    return dispatch_bwd<float>(dk, q, k, v, g, beta, h0, cu_seqlens, N, T_tot, H, dO, dhT, dq,
                               dk_, dv_, dg, dbeta, dh0, workspace, s);
}

kda_status kda_prologue(const void *xq, const void *xk, const void *xv, const float *wq,
                        const float *wk, const float *wv, const void *beta_raw,
                        const int32_t *cu_seqlens, int32_t N, int64_t T_tot, int32_t H, int32_t d,
                        kda_dtype dt, void *q, void *k, void *v, void *beta, void *stream) {
    if (N < 0 || T_tot < 0 || H <= 0 || H > 65535) return KDA_ERR_INVALID_ARGUMENT;
    if (dt != KDA_BF16 && dt != KDA_FP32) return KDA_ERR_UNSUPPORTED;
    if (!supported_simt_d(d)) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return T_tot == 0 ? KDA_OK : KDA_ERR_INVALID_ARGUMENT;
    if (cu_seqlens == nullptr && (T_tot % N) != 0) return KDA_ERR_INVALID_ARGUMENT;
    if (T_tot == 0) return KDA_OK;
    const void *req[] = {xq, xk, xv, wq, wk, wv, beta_raw, q, k, v, beta};
    for (const void *p : req)
        if (p == nullptr || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
    if (cu_seqlens && !aligned16(cu_seqlens)) return KDA_ERR_INVALID_ARGUMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (dt == KDA_BF16)
        return dispatch_prologue<__nv_bfloat16>(d, xq, xk, xv, wq, wk, wv, beta_raw, cu_seqlens, N,
                                                T_tot, H, q, k, v, beta, s);
    return dispatch_prologue<float>(d, xq, xk, xv, wq, wk, wv, beta_raw, cu_seqlens, N, T_tot, H,
                                    q, k, v, beta, s);
}

#ifdef KDA_TRACE
// Profiling builds only: copy the stage timestamps of the traced chain out.
KDA_API int kda_debug_trace_read(unsigned long long *dst, size_t n) {
    const size_t bytes = sizeof(kda::prefill::g_trace);
    if (n * sizeof(unsigned long long) < bytes) return -1;
    return cudaMemcpyFromSymbol(dst, kda::prefill::g_trace, bytes) == cudaSuccess ? 0 : -1;
}
KDA_API int kda_debug_cta_times(unsigned long long *dst, size_t n) {
    const size_t bytes = sizeof(kda::prefill::g_cta_time);
    if (n * sizeof(unsigned long long) < bytes) return -1;
    return cudaMemcpyFromSymbol(dst, kda::prefill::g_cta_time, bytes) == cudaSuccess ? 0 : -1;
}
#endif

kda_status kda_debug_stall_prefill(int32_t step, uint64_t limit_cycles) {
    if (step < 0 || limit_cycles == 0 || limit_cycles > (1ull << 32))
        return KDA_ERR_INVALID_ARGUMENT;
    kda::DebugStall &d = kda::debug_stall();
    d.limit.store((unsigned long long)limit_cycles);
    d.step.store(step);
    return KDA_OK;
}

kda_status kda_debug_range_prefill(int32_t step) {
    if (step < 0) return KDA_ERR_INVALID_ARGUMENT;
    static const unsigned int init[4][kda::prefill::kRangeCols] = {
        {0u, 0x7f800000u, 0u, 0u, 0u, 0u}, {0u, 0x7f800000u, 0u, 0u, 0u, 0u},
        {0u, 0x7f800000u, 0u, 0u, 0u, 0u}, {0u, 0x7f800000u, 0u, 0u, 0u, 0u}};
    if (cudaMemcpyToSymbol(kda::prefill::g_range, init, sizeof(init)) != cudaSuccess)
        return KDA_ERR_CUDA;
    kda::debug_range().step.store(step);
    return KDA_OK;
}

kda_status kda_debug_range_read(float *out, size_t n) {
    unsigned int r[4][kda::prefill::kRangeCols];
    if (out == nullptr || n < 4 * (size_t)kda::prefill::kRangeCols) return KDA_ERR_INVALID_ARGUMENT;
    if (cudaMemcpyFromSymbol(r, kda::prefill::g_range, sizeof(r)) != cudaSuccess) return KDA_ERR_CUDA;
    for (int i = 0; i < 4; ++i)
        for (int j = 0; j < kda::prefill::kRangeCols; ++j) {
            uint32_t b = r[i][j];
            float f;
            if (j <= kda::prefill::kRangeMinNz) std::memcpy(&f, &b, 4);
            else f = (float)b;
            out[i * kda::prefill::kRangeCols + j] = f;
        }
    return KDA_OK;
}

kda_status kda_stream_status(void *stream) {
    static std::atomic<unsigned> next_slot{0};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
    // read and clear the word in one atomic exchange, on this stream
    const int slot = (int)(next_slot.fetch_add(1u, std::memory_order_relaxed) % kda::kStatusSlots);
    kda::status_take_kernel<<<1, 1, 0, s>>>(slot);
    if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbolAsync(&word, kda::g_status_taken, sizeof(word),
                                  sizeof(word) * (size_t)slot, cudaMemcpyDeviceToHost,
                                  s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (word & kda::kErrTimeout) return KDA_ERR_TIMEOUT;
    if (word & kda::kErrSeqlens) return KDA_ERR_BAD_SEQLENS;
    return KDA_OK;
}

}  // extern "C"

#include "kda_noalloc.cuh"
#include "kda_selftest.cuh"
