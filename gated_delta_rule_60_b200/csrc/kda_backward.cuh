// kda_backward.cuh -- gradient of the prefill (dq, dk, dv, dg, dbeta, dh0) for
// L = <dO, O> + <dhT, hT>, on CUDA cores in fp32.
//
// The operator (page "Kimi K3 发布核实与 Moonshot AI 主干架构演变", §3 "KDA 为什
// 么不同于 MLA"; item 3 there: the chunked form serves training), one token:
//   a = exp(l(g)), l(g) = -5 sigmoid(g);  S' = Diag(a) S;  w = v - S'^T k;
//   u = beta w;  S_t = S' + k u^T;  o = S_t^T q.
// Its derivative, token by token in reverse (dS = dL/dS_t on entry):
//   dq   = S_t dO                       dS  += q dO^T
//   du   = dS^T k                       dk   = dS u - beta S' du
//   dv   = beta du                      dbeta = du . w
//   dS'  = dS - beta k du^T             da_i = sum_j dS'_ij S_ij   (S = S_{t-1})
//   dg_i = da_i a_i l'(g_i)             dS_{t-1} = Diag(a) dS'
// with l'(g) = -5 sigmoid(g) (1 - sigmoid(g)).
//
// One CTA runs one (sequence, head): a forward sweep keeps the state at every
// 16-token chunk boundary in the workspace; the reverse sweep then takes the
// chunks last to first, recomputes the chunk's 16 token states from its
// checkpoint into a per-CTA scratch, and runs the token derivative above in
// reverse.  Thread i < D owns row i (d_k) or column i (d_v) of the current
// pass, so every sum over a row or a column is one thread's loop: no
// cross-thread reduction except dbeta.  State rows are padded by one float in
// shared memory so that the row passes are free of bank conflicts.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace bwd {

constexpr int kThreads = 128;
constexpr int kChunk = 16;

template <int D>
struct Smem {
    static constexpr int kRow = D + 1;               // padded row stride
    float S[D * kRow];
    float dS[D * kRow];
    float q[D], k[D], v[D], a[D], lg[D], dO[D], u[D], w[D], du[D];
    float red[kThreads / 32];
};

// Column j of Diag(a) S times k: four independent partial sums, so the FMA
// latency does not serialise the loop.
template <int D>
__device__ __forceinline__ float col_dot_ak(const Smem<D> &sm, int j) {
    constexpr int R = Smem<D>::kRow;
    float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
#pragma unroll 4
    for (int i = 0; i < D; i += 4) {
        r0 = fmaf(sm.a[i] * sm.S[i * R + j], sm.k[i], r0);
        r1 = fmaf(sm.a[i + 1] * sm.S[(i + 1) * R + j], sm.k[i + 1], r1);
        r2 = fmaf(sm.a[i + 2] * sm.S[(i + 2) * R + j], sm.k[i + 2], r2);
        r3 = fmaf(sm.a[i + 3] * sm.S[(i + 3) * R + j], sm.k[i + 3], r3);
    }
    return (r0 + r1) + (r2 + r3);
}

// Copies between a padded shared-memory matrix (rows of D + 1 floats) and a
// dense D x D global array, 16 bytes per global access, eight accesses in
// flight per thread (the reverse sweep moves one 64 KB state per token).
template <int D>
__device__ __forceinline__ void mat_from_global(float *sdst, const float *__restrict__ src, int tid) {
    constexpr int R = D + 1, N4 = D * D / 4, B = 8;
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
#pragma unroll 1
    for (int base = tid; base < N4; base += B * kThreads) {
        float4 v[B];
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int e4 = base + u * kThreads;
            v[u] = e4 < N4 ? s4[e4] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int e4 = base + u * kThreads;
            if (e4 < N4) {
                const int e = 4 * e4, i = e / D, j = e % D;
                float *d = sdst + i * R + j;
                d[0] = v[u].x;
                d[1] = v[u].y;
                d[2] = v[u].z;
                d[3] = v[u].w;
            }
        }
    }
}

template <int D>
__device__ __forceinline__ void mat_to_global(float *__restrict__ dst, const float *ssrc, int tid) {
    constexpr int R = D + 1, N4 = D * D / 4;
    float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll 4
    for (int e4 = tid; e4 < N4; e4 += kThreads) {
        const int e = 4 * e4, i = e / D, j = e % D;
        const float *sp = ssrc + i * R + j;
        d4[e4] = make_float4(sp[0], sp[1], sp[2], sp[3]);
    }
}

__device__ __forceinline__ float sigmoid_acc(float x) {
    return 1.f / (1.f + expf(-x));
}

// Number of 16-token chunks of sequence n, and the checkpoints before it.
__device__ __forceinline__ int64_t n_chunks(int64_t L) { return (L + kChunk - 1) / kChunk; }

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
chunk_bwd_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                 const T *__restrict__ g, const T *__restrict__ beta,
                 const float *__restrict__ h0, const int32_t *__restrict__ cu, int N,
                 int64_t T_tot, int H, const T *__restrict__ dO, const float *__restrict__ dhT,
                 T *__restrict__ dq, T *__restrict__ dk, T *__restrict__ dv,
                 T *__restrict__ dg, T *__restrict__ dbeta, float *__restrict__ dh0,
                 float *__restrict__ ckpt, float *__restrict__ tok) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem<D> &sm = *reinterpret_cast<Smem<D> *>(smem_raw);
    constexpr int R = Smem<D>::kRow;
    constexpr size_t DD = (size_t)D * D;
    const int tid = threadIdx.x;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    int64_t s0, s1;
    if (!seq_bounds(cu, n, N, T_tot, s0, s1)) return;
    const int64_t L = s1 - s0;
    const size_t unit = (size_t)n * H + h;
    // checkpoints of this unit: after those of sequences 0 .. n-1 (all heads)
    int64_t base = 0;
    if (cu == nullptr) {
        base = (int64_t)n * n_chunks(T_tot / N);
    } else {
        for (int m = 0; m < n; ++m) {
            const int64_t lm = (int64_t)cu[m + 1] - cu[m];
            base += n_chunks(lm < 0 ? 0 : (lm > T_tot ? T_tot : lm));
        }
    }
    // the workspace holds n_chunks(T_tot) + N checkpoints per head; a
    // malformed cu_seqlens elsewhere in the batch cannot push this unit past it
    if (base + n_chunks(L) > n_chunks(T_tot) + N) {
        if (tid == 0) raise_error(kErrSeqlens);
        return;
    }
    float *ck = ckpt + ((size_t)base * H + (size_t)h * n_chunks(L)) * DD;
    float *tk = tok + unit * kChunk * DD;

    auto load_vec = [&](float *dst, const T *src) {
        for (int i = tid; i < D; i += kThreads) dst[i] = IO<T>::ld(src + i);
    };
    // token t's inputs into shared memory (a = decay, lg = dl/dg)
    auto load_token = [&](int64_t t, bool grads) {
        const size_t x = ((size_t)t * H + h) * D;
        load_vec(sm.q, q + x);
        load_vec(sm.k, k + x);
        load_vec(sm.v, v + x);
        for (int i = tid; i < D; i += kThreads) {
            const float gi = IO<T>::ld(g + x + i);
            const float s = sigmoid_acc(gi);
            sm.a[i] = expf(-5.f * s);
            sm.lg[i] = -5.f * s * (1.f - s);
        }
        if (grads) load_vec(sm.dO, dO + x);
    };
    // one forward token on the state in shared memory: w, u, then S <- S_t
    auto forward_token = [&](float bt) {
        __syncthreads();
        for (int j = tid; j < D; j += kThreads) {      // column j
            const float r = col_dot_ak<D>(sm, j);
            sm.w[j] = sm.v[j] - r;
            sm.u[j] = bt * sm.w[j];
        }
        __syncthreads();
        for (int j = tid; j < D; j += kThreads) {
            const float uj = sm.u[j];
            for (int i = 0; i < D; ++i) sm.S[i * R + j] = fmaf(sm.a[i], sm.S[i * R + j], sm.k[i] * uj);
        }
    };
    auto beta_of = [&](int64_t t) { return IO<T>::ld(beta + (size_t)t * H + h); };

    // ---- forward sweep: checkpoints before every 16th token
    if (h0) {
        mat_from_global<D>(sm.S, h0 + unit * DD, tid);
    } else {
        for (int e = tid; e < D * D; e += kThreads) sm.S[(e / D) * R + e % D] = 0.f;
    }
    for (int64_t t = s0; t < s1; ++t) {
        if ((t - s0) % kChunk == 0) {
            __syncthreads();
            float *dst = ck + (size_t)((t - s0) / kChunk) * DD;
            mat_to_global<D>(dst, sm.S, tid);
        }
        __syncthreads();
        load_token(t, false);
        forward_token(beta_of(t));
    }

    // ---- reverse sweep
    __syncthreads();
    if (dhT) {
        mat_from_global<D>(sm.dS, dhT + unit * DD, tid);
    } else {
        for (int e = tid; e < D * D; e += kThreads) sm.dS[(e / D) * R + e % D] = 0.f;
    }
    for (int64_t c = n_chunks(L) - 1; c >= 0; --c) {
        const int64_t a0 = s0 + c * kChunk;
        const int64_t a1 = a0 + kChunk < s1 ? a0 + kChunk : s1;
        // the chunk's token states S_{t-1}, recomputed from its checkpoint
        __syncthreads();
        mat_from_global<D>(sm.S, ck + (size_t)c * DD, tid);
        for (int64_t t = a0; t < a1; ++t) {
            __syncthreads();
            float *dst = tk + (size_t)(t - a0) * DD;
            mat_to_global<D>(dst, sm.S, tid);
            load_token(t, false);
            forward_token(beta_of(t));
        }
        for (int64_t t = a1 - 1; t >= a0; --t) {
            __syncthreads();
            const float *src = tk + (size_t)(t - a0) * DD;
            mat_from_global<D>(sm.S, src, tid);
            load_token(t, true);
            const float bt = beta_of(t);
            __syncthreads();
            // w = v - S'^T k, u = beta w (S = S_{t-1}, S' = Diag(a) S)
            for (int j = tid; j < D; j += kThreads) {
                const float r = col_dot_ak<D>(sm, j);
                sm.w[j] = sm.v[j] - r;
                sm.u[j] = bt * sm.w[j];
            }
            __syncthreads();
            const size_t x = ((size_t)t * H + h) * D;
            // rows: dq = S_t dO = Diag(a) S dO + k (u . dO);  dS += q dO^T;  dk = dS u
            float udo0 = 0.f, udo1 = 0.f;
#pragma unroll 4
            for (int j = 0; j < D; j += 2) {
                udo0 = fmaf(sm.u[j], sm.dO[j], udo0);
                udo1 = fmaf(sm.u[j + 1], sm.dO[j + 1], udo1);
            }
            const float udo = udo0 + udo1;
            float dk_part[(D + kThreads - 1) / kThreads];
#pragma unroll
            for (int s = 0; s < (D + kThreads - 1) / kThreads; ++s) dk_part[s] = 0.f;
#pragma unroll
            for (int s = 0; s < (D + kThreads - 1) / kThreads; ++s) {
                const int i = tid + s * kThreads;
                if (i >= D) break;
                float sd0 = 0.f, sd1 = 0.f, dsu0 = 0.f, dsu1 = 0.f;
                const float qi = sm.q[i];
#pragma unroll 4
                for (int j = 0; j < D; j += 2) {
                    sd0 = fmaf(sm.S[i * R + j], sm.dO[j], sd0);
                    sd1 = fmaf(sm.S[i * R + j + 1], sm.dO[j + 1], sd1);
                    const float ds0 = fmaf(qi, sm.dO[j], sm.dS[i * R + j]);
                    const float ds1 = fmaf(qi, sm.dO[j + 1], sm.dS[i * R + j + 1]);
                    sm.dS[i * R + j] = ds0;
                    sm.dS[i * R + j + 1] = ds1;
                    dsu0 = fmaf(ds0, sm.u[j], dsu0);
                    dsu1 = fmaf(ds1, sm.u[j + 1], dsu1);
                }
                IO<T>::st(dq + x + i, fmaf(sm.a[i], sd0 + sd1, sm.k[i] * udo));
                dk_part[s] = dsu0 + dsu1;
            }
            __syncthreads();
            // columns: du = dS^T k;  dv = beta du
            float dbp = 0.f;
            for (int j = tid; j < D; j += kThreads) {
                float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll 4
                for (int i = 0; i < D; i += 4) {
                    d0 = fmaf(sm.dS[i * R + j], sm.k[i], d0);
                    d1 = fmaf(sm.dS[(i + 1) * R + j], sm.k[i + 1], d1);
                    d2 = fmaf(sm.dS[(i + 2) * R + j], sm.k[i + 2], d2);
                    d3 = fmaf(sm.dS[(i + 3) * R + j], sm.k[i + 3], d3);
                }
                const float d = (d0 + d1) + (d2 + d3);
                sm.du[j] = d;
                IO<T>::st(dv + x + j, bt * d);
                dbp = fmaf(d, sm.w[j], dbp);
            }
            __syncthreads();
            // rows: dk -= beta S' du;  dS' = dS - beta k du^T;  da = sum_j dS' S;
            // dg = da a l';  dS <- Diag(a) dS'
#pragma unroll
            for (int s = 0; s < (D + kThreads - 1) / kThreads; ++s) {
                const int i = tid + s * kThreads;
                if (i >= D) break;
                const float ai = sm.a[i], bki = bt * sm.k[i];
                float sdu0 = 0.f, sdu1 = 0.f, da0 = 0.f, da1 = 0.f;
#pragma unroll 4
                for (int j = 0; j < D; j += 2) {
                    const float s0 = sm.S[i * R + j], s1 = sm.S[i * R + j + 1];
                    sdu0 = fmaf(s0, sm.du[j], sdu0);
                    sdu1 = fmaf(s1, sm.du[j + 1], sdu1);
                    const float p0 = fmaf(-bki, sm.du[j], sm.dS[i * R + j]);
                    const float p1 = fmaf(-bki, sm.du[j + 1], sm.dS[i * R + j + 1]);
                    da0 = fmaf(p0, s0, da0);
                    da1 = fmaf(p1, s1, da1);
                    sm.dS[i * R + j] = ai * p0;
                    sm.dS[i * R + j + 1] = ai * p1;
                }
                IO<T>::st(dk + x + i, dk_part[s] - bt * ai * (sdu0 + sdu1));
                IO<T>::st(dg + x + i, (da0 + da1) * ai * sm.lg[i]);
            }
            // dbeta = du . w (block reduction)
            for (int o = 16; o > 0; o >>= 1) dbp += __shfl_xor_sync(0xffffffffu, dbp, o);
            if ((tid & 31) == 0) sm.red[tid >> 5] = dbp;
            __syncthreads();
            if (tid == 0) {
                float s = 0.f;
                for (int w = 0; w < kThreads / 32; ++w) s += sm.red[w];
                IO<T>::st(dbeta + (size_t)t * H + h, s);
            }
        }
    }
    __syncthreads();
    if (dh0)
        mat_to_global<D>(dh0 + unit * DD, sm.dS, tid);
}

}  // namespace bwd
}  // namespace kda
