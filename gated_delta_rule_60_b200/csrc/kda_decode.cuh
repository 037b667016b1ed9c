// kda_decode.cuh -- single-token KDA decode step (memory-bound).
//
// For each (sequence b, head h) one token updates the fp32 state in place:
//   a = exp(-5 sigmoid(g));  S' = Diag(a) S;  u = beta (v - S'^T k)
//   S = S' + k u^T;          o = S^T q = S'^T q + u (k . q)
// (page "Kimi K3 发布核实与 Moonshot AI 主干架构演变", §3 "KDA 为什么不同于
// MLA": decay first, correct with beta, k and v, read from the updated state).
//
// Layout: thread (part, j) of a head owns column j of the state rows
// [part * D/SPLIT, (part+1) * D/SPLIT).  Per row, a warp touches 32
// consecutive floats (one 128-byte segment), so every access is coalesced.
// The column slice stays in registers; the partial reductions
// r_j = sum_i S'_ij k_i and p_j = sum_i S'_ij q_i are combined across the
// SPLIT row parts through shared memory, then every part writes its rows back.
// Each state element is read once and written once, with the streaming
// (evict-first) cache hint: the state is far larger than L2 and is not
// re-read within a step.  d = 128 has its own kernel below with 128-bit
// accesses.
#pragma once

#include "kda_common.cuh"

namespace kda {

template <int D, int SPLIT>
struct DecodeShape {
    static constexpr int kRows = D / SPLIT;                // rows per thread
    static constexpr int kThreadsPerHead = D * SPLIT;
    static constexpr int kHeadsPerBlock =
        kThreadsPerHead >= 128 ? 1 : 128 / kThreadsPerHead;
    static constexpr int kThreads = kHeadsPerBlock * kThreadsPerHead;
};

// kSoftplus: the unbounded gate log a = -softplus(g) instead of -5 sigmoid(g).
template <typename T, int D, int SPLIT, bool kSoftplus = false>
__global__ void __launch_bounds__(DecodeShape<D, SPLIT>::kThreads)
decode_step_kernel(const T *__restrict__ q, const T *__restrict__ k,
                   const T *__restrict__ v, const T *__restrict__ g,
                   const T *__restrict__ beta, float *__restrict__ S,
                   T *__restrict__ o, long units) {
    using Sh = DecodeShape<D, SPLIT>;
    constexpr int HPB = Sh::kHeadsPerBlock;
    constexpr int R = Sh::kRows;
    __shared__ float sa[HPB][D], sk[HPB][D], sq[HPB][D];
    __shared__ float sr[HPB][SPLIT][D], sp[HPB][SPLIT][D], su[HPB][D];

    const int hl = threadIdx.x / Sh::kThreadsPerHead;
    const int t = threadIdx.x % Sh::kThreadsPerHead;
    const int part = t / D, j = t % D;
    const long u = (long)blockIdx.x * HPB + hl;
    const bool active = u < units;

    float *Su = S + (size_t)(active ? u : 0) * D * D + (size_t)part * R * D + j;
    float s[R];
    if (active) {
#pragma unroll
        for (int i = 0; i < R; ++i) s[i] = __ldcs(Su + (size_t)i * D);
        if (part == 0) {
            const size_t e = (size_t)u * D + j;
            sq[hl][j] = IO<T>::ld(q + e);
            sk[hl][j] = IO<T>::ld(k + e);
            const float gv = IO<T>::ld(g + e);
            sa[hl][j] = expf(kSoftplus ? log_decay_softplus(gv) : log_decay(gv));
        }
    }
    __syncthreads();
    if (active) {
        float r = 0.f, p = 0.f;
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int row = part * R + i;
            s[i] *= sa[hl][row];
            r = fmaf(s[i], sk[hl][row], r);
            p = fmaf(s[i], sq[hl][row], p);
        }
        sr[hl][part][j] = r;
        sp[hl][part][j] = p;
    }
    __syncthreads();
    if (active && part == 0) {
        // k . q, computed by every owner thread from shared memory (no
        // cross-lane shuffles: a warp may hold several heads, some inactive)
        float kq = 0.f;
#pragma unroll 8
        for (int i = 0; i < D; ++i) kq = fmaf(sk[hl][i], sq[hl][i], kq);
        float r = 0.f, p = 0.f;
#pragma unroll
        for (int x = 0; x < SPLIT; ++x) { r += sr[hl][x][j]; p += sp[hl][x][j]; }
        const float uj = IO<T>::ld(beta + u) * (IO<T>::ld(v + (size_t)u * D + j) - r);
        su[hl][j] = uj;
        IO<T>::st(o + (size_t)u * D + j, fmaf(uj, kq, p));
    }
    __syncthreads();
    if (active) {
        const float uj = su[hl][j];
#pragma unroll
        for (int i = 0; i < R; ++i)
            __stcs(Su + (size_t)i * D, fmaf(sk[hl][part * R + i], uj, s[i]));
    }
}

// d = 128: the state of one (b, h) is 128 rows of 512 bytes.  Warp w of the
// 256-thread block owns rows 16 w .. 16 w + 15; lane l owns columns
// 4 l .. 4 l + 3 of each, so every access is one 128-bit streaming load or
// store and a warp covers a whole row in one instruction.  A thread issues its
// 16 row loads back to back (64 KB in flight per block) before it needs any
// of them.  The column sums r = S'^T k and p = S'^T q are partial per warp and
// meet in shared memory.
__device__ __forceinline__ float4 ld_stream_f4(const float *p) {
    float4 r;
    asm volatile("ld.global.cs.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_stream_f4(float *p, float4 v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w)
                 : "memory");
}

constexpr int kDecode128Threads = 256;

template <typename T, bool kSoftplus = false>
__global__ void __launch_bounds__(kDecode128Threads)
decode_step_d128_kernel(const T *__restrict__ q, const T *__restrict__ k,
                        const T *__restrict__ v, const T *__restrict__ g,
                        const T *__restrict__ beta, float *__restrict__ S,
                        T *__restrict__ o) {
    constexpr int D = 128, W = kDecode128Threads / 32, R = D / W;
    __shared__ float sa[D], sk[D], sq[D], su[D];
    __shared__ float4 sr[W][D / 4], sp[W][D / 4];
    __shared__ float skq[W];
    const long u = blockIdx.x;
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    float *Su = S + (size_t)u * D * D + (size_t)(R * w) * D + 4 * l;
    float4 s[R];
#pragma unroll
    for (int i = 0; i < R; ++i) s[i] = ld_stream_f4(Su + (size_t)i * D);
    if (tid < D) {
        const size_t e = (size_t)u * D + tid;
        sq[tid] = IO<T>::ld(q + e);
        sk[tid] = IO<T>::ld(k + e);
        const float gv = IO<T>::ld(g + e);
        sa[tid] = expf(kSoftplus ? log_decay_softplus(gv) : log_decay(gv));
    }
    __syncthreads();
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f), p = r;
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int row = R * w + i;
        const float a = sa[row], kr = sk[row], qr = sq[row];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        r.x = fmaf(s[i].x, kr, r.x); r.y = fmaf(s[i].y, kr, r.y);
        r.z = fmaf(s[i].z, kr, r.z); r.w = fmaf(s[i].w, kr, r.w);
        p.x = fmaf(s[i].x, qr, p.x); p.y = fmaf(s[i].y, qr, p.y);
        p.z = fmaf(s[i].z, qr, p.z); p.w = fmaf(s[i].w, qr, p.w);
    }
    sr[w][l] = r;
    sp[w][l] = p;
    if (l == 0) {                                   // k . q over this warp's rows
        float kq = 0.f;
#pragma unroll
        for (int i = 0; i < R; ++i) kq = fmaf(sk[R * w + i], sq[R * w + i], kq);
        skq[w] = kq;
    }
    __syncthreads();
    if (tid < D) {
        const int j = tid;
        float kq = 0.f;
#pragma unroll
        for (int x = 0; x < W; ++x) kq += skq[x];
        const float *srf = reinterpret_cast<const float *>(sr);
        const float *spf = reinterpret_cast<const float *>(sp);
        float rj = 0.f, pj = 0.f;
#pragma unroll
        for (int x = 0; x < W; ++x) { rj += srf[x * D + j]; pj += spf[x * D + j]; }
        const float uj = IO<T>::ld(beta + u) * (IO<T>::ld(v + (size_t)u * D + j) - rj);
        su[j] = uj;
        IO<T>::st(o + (size_t)u * D + j, fmaf(uj, kq, pj));
    }
    __syncthreads();
    const float4 uu = reinterpret_cast<const float4 *>(su)[l];
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const float kr = sk[R * w + i];
        float4 y = s[i];
        y.x = fmaf(kr, uu.x, y.x); y.y = fmaf(kr, uu.y, y.y);
        y.z = fmaf(kr, uu.z, y.z); y.w = fmaf(kr, uu.w, y.w);
        st_stream_f4(Su + (size_t)i * D, y);
    }
}

}  // namespace kda
