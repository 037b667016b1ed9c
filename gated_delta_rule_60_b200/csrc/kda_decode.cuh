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
// re-read within a step.
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

template <typename T, int D, int SPLIT>
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
            sa[hl][j] = expf(log_decay(IO<T>::ld(g + e)));
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

}  // namespace kda
