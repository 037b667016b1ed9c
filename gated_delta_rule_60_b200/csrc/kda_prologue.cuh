// kda_prologue.cuh -- the step just before the operator, fused into one
// memory-bound pass: the operator's q, k, v and beta from the raw projections.
//
// Page "Kimi K3 模型架构解析：KDA、AttnRes 与 Stable LatentMoE", §二.3: KDA
// mixes neighbouring tokens with a length-4 short convolution.  Readings where
// the pages are silent: the convolution is causal and depthwise (one 4-tap
// filter per head and channel, tap j multiplies the token j steps back), it is
// applied to the q, k and v projections, it restarts at every sequence start
// (zero history) and no activation follows it; q and k are then L2-normalised
// per (token, head), and beta is the sigmoid of its raw projection.  The gate
// g stays raw: the operator applies log a = -5 sigmoid(g) itself.
//
//   q_t = l2(sum_j wq_j * xq_{t-j}),  k_t = l2(sum_j wk_j * xk_{t-j}),
//   v_t = sum_j wv_j * xv_{t-j},      beta_t = sigmoid(braw_t)
//
// Layout: grid (token chunk, head, tensor q / k / v).  A thread owns 8
// consecutive channels of one head and walks kTokPerLane consecutive tokens,
// keeping the filter taps and the last three input rows in
// registers, so every input row is read once (plus a three-row halo per lane).
// The d / 8 threads of one token row sit in adjacent lanes of a warp and
// reduce the squared norm with shuffles.  All arithmetic is fp32; outputs are
// rounded to the storage type (RNE).
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace pro {

constexpr int kThreads = 128;
constexpr int kTokPerLane = 16;

template <int D>
struct Shape {
    static constexpr int kGroups = D / 8;                  // threads per token row
    static constexpr int kLanes = kThreads / kGroups;      // token rows per block at a time
    static constexpr int kTokPerBlock = kLanes * kTokPerLane;
};

template <typename T>
struct Vec8;

template <>
struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void ld(const __nv_bfloat16 *p, float (&v)[8]) {
        const uint4 r = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, const float (&v)[8]) {
        uint4 r;
        uint32_t *w = reinterpret_cast<uint32_t *>(&r);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&b);
        }
        *reinterpret_cast<uint4 *>(p) = r;
    }
};

template <>
struct Vec8<float> {
    static __device__ __forceinline__ void ld(const float *p, float (&v)[8]) {
        const float4 a = reinterpret_cast<const float4 *>(p)[0];
        const float4 b = reinterpret_cast<const float4 *>(p)[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    static __device__ __forceinline__ void st(float *p, const float (&v)[8]) {
        reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
};

// Sequence n with cu[n] <= t < cu[n + 1] (the last such n, so that empty
// sequences are skipped); equal lengths T_tot / N when cu is NULL.
__device__ __forceinline__ int seq_of(const int32_t *cu, int N, int64_t T_tot, int64_t t) {
    if (cu == nullptr) return (int)(t / (T_tot / N));
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)cu[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ int64_t seq_start(const int32_t *cu, int N, int64_t T_tot, int n) {
    return cu == nullptr ? (int64_t)n * (T_tot / N) : (int64_t)cu[n];
}

__device__ __forceinline__ float sigmoid_f(float x) {
    return 1.f / (1.f + expf(-x));
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
prologue_kernel(const T *__restrict__ xq, const T *__restrict__ xk, const T *__restrict__ xv,
                const float *__restrict__ wq, const float *__restrict__ wk,
                const float *__restrict__ wv, const T *__restrict__ braw,
                const int32_t *__restrict__ cu, int N, int64_t T_tot, int H,
                T *__restrict__ q, T *__restrict__ k, T *__restrict__ v, T *__restrict__ beta) {
    using Sh = Shape<D>;
    const int tensor = blockIdx.z;                    // 0: q, 1: k, 2: v
    const int h = blockIdx.y;
    const int cg = threadIdx.x % Sh::kGroups, lane_row = threadIdx.x / Sh::kGroups;
    const int64_t t0 = (int64_t)blockIdx.x * Sh::kTokPerBlock + (int64_t)lane_row * kTokPerLane;
    const T *x = tensor == 0 ? xq : (tensor == 1 ? xk : xv);
    const float *w = tensor == 0 ? wq : (tensor == 1 ? wk : wv);
    T *y = tensor == 0 ? q : (tensor == 1 ? k : v);
    const bool norm = tensor < 2;
    const size_t row = (size_t)H * D;                 // elements between consecutive tokens
    const size_t col = (size_t)h * D + 8 * cg;

    // one thread checks cu_seqlens (reported, not faulted: every read below
    // stays inside cu[0 .. N] whatever its contents are)
    if (cu != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) {
        bool ok = cu[0] == 0 && (int64_t)cu[N] == T_tot;
        for (int i = 0; i < N && ok; ++i) ok = cu[i] <= cu[i + 1];
        if (!ok) raise_error(kErrSeqlens);
    }
    // filter taps of this thread's 8 channels: w[h][c][j]
    float wr[8][4];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float4 t4 = reinterpret_cast<const float4 *>(w + ((size_t)h * D + 8 * cg + c) * 4)[0];
        wr[c][0] = t4.x; wr[c][1] = t4.y; wr[c][2] = t4.z; wr[c][3] = t4.w;
    }

    // the sequence of the first token and its history (zero before its start)
    int n = 0;
    int64_t s_begin = 0, s_end = 0;
    float hist[3][8];                                 // x_{t-1}, x_{t-2}, x_{t-3}
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int c = 0; c < 8; ++c) hist[i][c] = 0.f;
    if (t0 < T_tot) {
        n = seq_of(cu, N, T_tot, t0);
        s_begin = seq_start(cu, N, T_tot, n);
        s_end = seq_start(cu, N, T_tot, n + 1);
        // (tp >= 0 as well: a malformed cu_seqlens may give a negative start)
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const int64_t tp = t0 - 1 - i;
            if (tp >= s_begin && tp >= 0) Vec8<T>::ld(x + (size_t)tp * row + col, hist[i]);
        }
    }

#pragma unroll 1
    for (int it = 0; it < kTokPerLane; ++it) {
        const int64_t t = t0 + it;
        const bool live = t < T_tot;                  // every lane keeps shuffling
        float yv[8];
        if (live) {
            // crossing into the next non-empty sequence: zero history
            if (t >= s_end) {
                while (n + 1 < N && seq_start(cu, N, T_tot, n + 1) <= t) ++n;
                s_begin = seq_start(cu, N, T_tot, n);
                s_end = seq_start(cu, N, T_tot, n + 1);
#pragma unroll
                for (int i = 0; i < 3; ++i)
#pragma unroll
                    for (int c = 0; c < 8; ++c) hist[i][c] = 0.f;
            }
            float xv8[8];
            Vec8<T>::ld(x + (size_t)t * row + col, xv8);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float a = wr[c][0] * xv8[c];
                a = fmaf(wr[c][1], hist[0][c], a);
                a = fmaf(wr[c][2], hist[1][c], a);
                a = fmaf(wr[c][3], hist[2][c], a);
                yv[c] = a;
                hist[2][c] = hist[1][c];
                hist[1][c] = hist[0][c];
                hist[0][c] = xv8[c];
            }
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) yv[c] = 0.f;
        }
        if (norm) {
            float ss = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) ss = fmaf(yv[c], yv[c], ss);
#pragma unroll
            for (int o = 1; o < Sh::kGroups; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;   // an all-zero row stays zero
#pragma unroll
            for (int c = 0; c < 8; ++c) yv[c] *= inv;
        }
        if (live) {
            Vec8<T>::st(y + (size_t)t * row + col, yv);
            if (tensor == 0 && cg == 0) {
                const size_t e = (size_t)t * H + h;
                IO<T>::st(beta + e, sigmoid_f(IO<T>::ld(braw + e)));
            }
        }
    }
}

}  // namespace pro
}  // namespace kda
