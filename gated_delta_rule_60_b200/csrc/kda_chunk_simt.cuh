// kda_chunk_simt.cuh -- chunked KDA prefill on CUDA cores, all in fp32.
//
// This is the fp32 test mode (and the path for head sizes below 128).  It
// runs the same 16-token chunk algorithm as the tensor-core kernel, with
// every product in fp32 FFMA, so it can be held to 1e-5 against the oracle.
//
// Chunk algorithm (derived from the recurrence of the page "Kimi K3 发布核实
// 与 Moonshot AI 主干架构演变", §3: recurrent across chunks, parallel within
// a chunk).  For rows r = 0..15 of one chunk with start state S0:
//   l_r = -5 sigmoid(g_r),  b_r = l_0 + .. + l_r  (per key channel)
//   m   = b_7 (centring reference: every exponent below is within +-40)
//   A_ri = beta_r sum_c (k_rc e^{b_rc - m_c}) (k_ic e^{m_c - b_ic})   i < r
//   M_ri =        sum_c (q_rc e^{b_rc - m_c}) (k_ic e^{m_c - b_ic})   i <= r
//   T = (I + A)^-1 Diag(beta)            (forward substitution)
//   W = T (K * e^b),  U = T V - W S0
//   O = (Q * e^b) S0 + M U
//   S = Diag(e^{b_15}) S0 + (K * e^{b_15 - b})^T U
// Rows past the end of a sequence are padded with exact no-op tokens
// (k = q = v = 0, beta = 0, log-decay 0).
//
// kSoftplus: the unbounded gate log a = -softplus(g).  A chunk's cumulative
// log-decay is then unbounded, so the centred split e^{b-m} e^{m-b} can leave
// the fp32 range; every decay factor is formed instead as the exponential of
// a direct sum over the tokens it spans (prefix sums from the chunk start,
// suffix sums from its end, and for A and M the sum over tokens i+1 .. r of
// each pair), all <= 0, so each factor lies in [0, 1] and a token that forgets
// everything (g = +inf) gives exact zeros rather than -inf - (-inf).
//
// One CTA runs one (sequence, head) chain over all of its chunks; the state
// lives in shared memory in fp32.  With z given, every output row is
// multiplied by sigmoid(z) before it is stored (the fused output gate).
#pragma once

#include "kda_common.cuh"

namespace kda {

constexpr int kChunk = 16;

template <int D>
struct SimtSmem {
    float S[D][D];
    float q[kChunk][D], k[kChunk][D], v[kChunk][D], l[kChunk][D];
    float Qr[kChunk][D], Kr[kChunk][D], Kh[kChunk][D];
    float Qa[kChunk][D], Ka[kChunk][D], Ke[kChunk][D];
    float W[kChunk][D], U[kChunk][D];
    float A[kChunk][kChunk], M[kChunk][kChunk], T[kChunk][kChunk];
    float gam[D];
    float beta[kChunk];
};

template <typename T, int D, bool kSoftplus = false>
__global__ void __launch_bounds__(256)
chunk_fwd_simt_kernel(const T *__restrict__ q, const T *__restrict__ k,
                      const T *__restrict__ v, const T *__restrict__ g,
                      const T *__restrict__ beta, const float *__restrict__ h0,
                      const int32_t *__restrict__ cu, int N, long T_tot, int H,
                      const T *__restrict__ z, T *__restrict__ o, float *__restrict__ hT) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SimtSmem<D> &sm = *reinterpret_cast<SimtSmem<D> *>(smem_raw);
    const int tid = threadIdx.x;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    int64_t start, end;
    if (!seq_bounds(cu, n, N, T_tot, start, end)) return;
    const size_t unit = (size_t)n * H + h;

    for (int e = tid; e < D * D; e += 256)
        (&sm.S[0][0])[e] = h0 ? h0[unit * D * D + e] : 0.f;

    for (int64_t c0 = start; c0 < end; c0 += kChunk) {
        const int L = (int)((end - c0) < kChunk ? (end - c0) : kChunk);
        __syncthreads();
        // 1. load the chunk (pad rows >= L with no-op tokens)
        for (int e = tid; e < kChunk * D; e += 256) {
            int r = e / D, c = e % D;
            float qv = 0.f, kv = 0.f, vv = 0.f, lv = 0.f;
            if (r < L) {
                size_t x = ((size_t)(c0 + r) * H + h) * D + c;
                qv = IO<T>::ld(q + x);
                kv = IO<T>::ld(k + x);
                vv = IO<T>::ld(v + x);
                lv = kSoftplus ? log_decay_softplus(IO<T>::ld(g + x)) : log_decay(IO<T>::ld(g + x));
            }
            sm.q[r][c] = qv; sm.k[r][c] = kv; sm.v[r][c] = vv; sm.l[r][c] = lv;
        }
        if (tid < kChunk)
            sm.beta[tid] = tid < L ? IO<T>::ld(beta + (size_t)(c0 + tid) * H + h) : 0.f;
        __syncthreads();
        // 2. per channel: cumulative log-decay and the scaled operands
        for (int c = tid; c < D && kSoftplus; c += 256) {
            // prefix sums b_r from the chunk start, suffix sums from its end
            float b[kChunk], sfx[kChunk];
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < kChunk; ++r) { acc += sm.l[r][c]; b[r] = acc; }
            acc = 0.f;
#pragma unroll
            for (int r = kChunk - 1; r >= 0; --r) { sfx[r] = acc; acc += sm.l[r][c]; }
            sm.gam[c] = expf(b[kChunk - 1]);
#pragma unroll
            for (int r = 0; r < kChunk; ++r) {
                const float kr = sm.k[r][c], qr = sm.q[r][c];
                sm.Qa[r][c] = qr * expf(b[r]);
                sm.Ka[r][c] = kr * expf(b[r]);
                sm.Ke[r][c] = kr * expf(sfx[r]);
            }
        }
        for (int c = tid; c < D && !kSoftplus; c += 256) {
            float b[kChunk];
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < kChunk; ++r) { acc += sm.l[r][c]; b[r] = acc; }
            const float m = b[7], bC = b[kChunk - 1];
            sm.gam[c] = expf(bC);
#pragma unroll
            for (int r = 0; r < kChunk; ++r) {
                const float kr = sm.k[r][c], qr = sm.q[r][c];
                sm.Qr[r][c] = qr * expf(b[r] - m);
                sm.Kr[r][c] = kr * expf(b[r] - m);
                sm.Kh[r][c] = kr * expf(m - b[r]);
                sm.Qa[r][c] = qr * expf(b[r]);
                sm.Ka[r][c] = kr * expf(b[r]);
                sm.Ke[r][c] = kr * expf(bC - b[r]);
            }
        }
        __syncthreads();
        // 3. intra-chunk products A (strict lower, beta-scaled) and M (causal)
        {
            const int r = tid / kChunk, i = tid % kChunk;
            float akk = 0.f, aqk = 0.f;
            if (kSoftplus) {
                // decay between token i and token r: e^{l_{i+1} + .. + l_r}
                if (i <= r)
                    for (int c = 0; c < D; ++c) {
                        float sp = 0.f;
                        for (int t = i + 1; t <= r; ++t) sp += sm.l[t][c];
                        const float w = expf(sp) * sm.k[i][c];
                        akk = fmaf(sm.k[r][c], w, akk);
                        aqk = fmaf(sm.q[r][c], w, aqk);
                    }
            } else {
                for (int c = 0; c < D; ++c) {
                    akk = fmaf(sm.Kr[r][c], sm.Kh[i][c], akk);
                    aqk = fmaf(sm.Qr[r][c], sm.Kh[i][c], aqk);
                }
            }
            sm.A[r][i] = i < r ? sm.beta[r] * akk : 0.f;
            sm.M[r][i] = i <= r ? aqk : 0.f;
        }
        __syncthreads();
        // 4. T = (I + A)^-1 Diag(beta): column i of T depends only on column i
        if (tid < kChunk) {
            const int i = tid;
            float col[kChunk];
#pragma unroll
            for (int r = 0; r < kChunk; ++r) {
                float x = (r == i) ? sm.beta[r] : 0.f;
#pragma unroll
                for (int j = 0; j < r; ++j) x = fmaf(-sm.A[r][j], col[j], x);
                col[r] = x;
            }
#pragma unroll
            for (int r = 0; r < kChunk; ++r) sm.T[r][i] = col[r];
        }
        __syncthreads();
        // 5. W = T (K * e^b);  U = T V  (U gets "- W S0" in step 6)
        for (int e = tid; e < kChunk * D; e += 256) {
            const int r = e / D, c = e % D;
            float w = 0.f, uv = 0.f;
#pragma unroll
            for (int i = 0; i < kChunk; ++i) {
                w = fmaf(sm.T[r][i], sm.Ka[i][c], w);
                uv = fmaf(sm.T[r][i], sm.v[i][c], uv);
            }
            sm.W[r][c] = w;
            sm.U[r][c] = uv;
        }
        __syncthreads();
        // 6. U -= W S0
        for (int e = tid; e < kChunk * D; e += 256) {
            const int r = e / D, j = e % D;
            float acc = sm.U[r][j];
            for (int c = 0; c < D; ++c) acc = fmaf(-sm.W[r][c], sm.S[c][j], acc);
            sm.U[r][j] = acc;
        }
        __syncthreads();
        // 7. O = (Q * e^b) S0 + M U  -> store the valid rows
        for (int e = tid; e < kChunk * D; e += 256) {
            const int r = e / D, j = e % D;
            if (r >= L) continue;
            float acc = 0.f;
            for (int c = 0; c < D; ++c) acc = fmaf(sm.Qa[r][c], sm.S[c][j], acc);
#pragma unroll
            for (int i = 0; i < kChunk; ++i) acc = fmaf(sm.M[r][i], sm.U[i][j], acc);
            const size_t oe = ((size_t)(c0 + r) * H + h) * D + j;
            if (z) acc *= out_gate(IO<T>::ld(z + oe));       // fused output gate
            IO<T>::st(o + oe, acc);
        }
        __syncthreads();
        // 8. S = Diag(gamma) S0 + (K * e^{b_C - b})^T U
        for (int e = tid; e < D * D; e += 256) {
            const int c = e / D, j = e % D;
            float acc = sm.gam[c] * sm.S[c][j];
#pragma unroll
            for (int i = 0; i < kChunk; ++i) acc = fmaf(sm.Ke[i][c], sm.U[i][j], acc);
            sm.S[c][j] = acc;
        }
    }
    __syncthreads();
    if (hT)
        for (int e = tid; e < D * D; e += 256) hT[unit * D * D + e] = (&sm.S[0][0])[e];
}

}  // namespace kda
