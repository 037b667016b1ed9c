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
// reverse.  Four threads (adjacent lanes) own each row (d_k) or column (d_v)
// of the current pass, each a quarter of it (every fourth element), and meet
// in two shuffles; the CTA has 4 d threads.  State rows are padded to d + 8
// floats in shared memory, so that a column pass reads 32 distinct banks per
// warp; in a row pass, rows 4-7 of a warp's eight walk their columns in a
// permuted order, which makes it conflict-free too.  Shared memory is the
// limit of this kernel: every warp-wide access costs a wavefront, even a
// broadcast of a few vector elements, so vectors read together are packed.
// A reverse token takes two passes: one over columns, for S'^T k and du,
// using du = (dS + q dO^T)^T k = dS^T k + dO (q . k) on dS as it enters, and
// one over rows for everything else.  A forward token (checkpoint and
// recompute sweeps) is one pass over columns: the four threads of a column
// keep their quarter of it in registers between the read and the update.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace bwd {

constexpr int kChunk = 16;
constexpr int kParts = 4;                         // threads per row or column

template <int D>
__host__ __device__ constexpr int threads_of() { return kParts * D; }

template <int D>
struct Smem {
    static constexpr int kRow = D + 8;               // padded row stride
    float S[D * kRow];
    float dS[D * kRow];
    static constexpr int kQkParts = D >= 32 ? D / 32 : 1;   // warps holding q and k
    // vectors read together are packed, one shared-memory access each:
    // ak[i] = (a_i, k_i) in the column passes, vec[j] = (dO_j, du_j, u_j, -)
    // in the row pass
    float4 vec[D];
    float2 ak[D];
    float q[D], v[D], lg[D];
    float red[threads_of<D>() / 32];
    float qkp[kQkParts];                             // per-warp partial sums of q . k
};

// Sum over the four lanes of a row or column.
__device__ __forceinline__ float quad_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    return x;
}

// Copies between a padded shared-memory matrix and a dense D x D global
// array, 16 bytes per access, up to eight global loads in flight per thread
// (h0, dhT, the checkpoints and the recomputed token states; the reverse
// pass fetches its token states one token ahead instead).
template <int D>
__device__ __forceinline__ void mat_from_global(float *sdst, const float *__restrict__ src, int tid) {
    constexpr int R = Smem<D>::kRow, N4 = D * D / 4, NT = threads_of<D>(), B = 8;
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
#pragma unroll 1
    for (int base = tid; base < N4; base += B * NT) {
        float4 v[B];
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int e4 = base + u * NT;
            v[u] = e4 < N4 ? s4[e4] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int e4 = base + u * NT;
            if (e4 < N4) {
                const int e = 4 * e4;
                *reinterpret_cast<float4 *>(sdst + (e / D) * R + e % D) = v[u];
            }
        }
    }
}

template <int D>
__device__ __forceinline__ void mat_to_global(float *__restrict__ dst, const float *ssrc, int tid) {
    constexpr int R = Smem<D>::kRow, N4 = D * D / 4, NT = threads_of<D>();
    float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll 4
    for (int e4 = tid; e4 < N4; e4 += NT) {
        const int e = 4 * e4;
        d4[e4] = *reinterpret_cast<const float4 *>(ssrc + (e / D) * R + e % D);
    }
}

template <int D>
__device__ __forceinline__ void mat_zero(float *sdst, int tid) {
    constexpr int R = Smem<D>::kRow;
    for (int e = tid; e < D * D; e += threads_of<D>()) sdst[(e / D) * R + e % D] = 0.f;
}

__device__ __forceinline__ float sigmoid_acc(float x) {
    return 1.f / (1.f + expf(-x));
}

// Number of 16-token chunks of sequence n, and the checkpoints before it.
__device__ __forceinline__ int64_t n_chunks(int64_t L) { return (L + kChunk - 1) / kChunk; }

template <typename T, int D>
__global__ void __launch_bounds__(threads_of<D>())
chunk_bwd_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                 const T *__restrict__ g, const T *__restrict__ beta,
                 const float *__restrict__ h0, const int32_t *__restrict__ cu, int N,
                 int64_t T_tot, int H, const T *__restrict__ dO, const float *__restrict__ dhT,
                 T *__restrict__ dq, T *__restrict__ dk, T *__restrict__ dv,
                 T *__restrict__ dg, T *__restrict__ dbeta, float *__restrict__ dh0,
                 float *__restrict__ ckpt, float *__restrict__ tok) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem<D> &sm = *reinterpret_cast<Smem<D> *>(smem_raw);
    constexpr int R = Smem<D>::kRow, NT = threads_of<D>(), Q = D / kParts;
    constexpr size_t DD = (size_t)D * D;
    const int tid = threadIdx.x;
    const int idx = tid >> 2, part = tid & 3;         // row or column idx, quarter `part`
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

    // token t's inputs: fetched into registers (thread i < D holds element i
    // of each vector, every thread holds beta) and written to shared memory
    // one token later, so that the loads fly while the previous token runs
    struct TokIn { float q, k, v, g, dO, beta; };
    auto fetch_token = [&](int64_t t, bool grads) {
        TokIn r{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const size_t x = ((size_t)t * H + h) * D + tid;
        if (tid < D) {
            r.q = IO<T>::ld(q + x);
            r.k = IO<T>::ld(k + x);
            r.v = IO<T>::ld(v + x);
            r.g = IO<T>::ld(g + x);
            if (grads) r.dO = IO<T>::ld(dO + x);
        }
        r.beta = IO<T>::ld(beta + (size_t)t * H + h);
        return r;
    };
    // a = decay, lg = dl/dg; with grads, also the partial sums of q . k
    auto put_token = [&](const TokIn &r, bool grads) {
        if (grads && tid < 32 * Smem<D>::kQkParts) {
            float p = tid < D ? r.q * r.k : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
            if ((tid & 31) == 0) sm.qkp[tid >> 5] = p;
        }
        if (tid < D) {
            const float s = sigmoid_acc(r.g);
            sm.q[tid] = r.q;
            sm.v[tid] = r.v;
            sm.ak[tid] = make_float2(expf(-5.f * s), r.k);
            sm.lg[tid] = -5.f * s * (1.f - s);
            sm.vec[tid].x = r.dO;
        }
    };
    // one token state (D x D fp32) through registers, 16 bytes per access
    constexpr int kPf = D / 16;                      // float4 per thread
    auto fetch_state = [&](float4 (&pf)[kPf], const float *src) {
        const float4 *s4 = reinterpret_cast<const float4 *>(src);
#pragma unroll
        for (int u = 0; u < kPf; ++u) pf[u] = s4[tid + u * NT];
    };
    auto put_state = [&](const float4 (&pf)[kPf]) {
#pragma unroll
        for (int u = 0; u < kPf; ++u) {
            const int e = 4 * (tid + u * NT);
            *reinterpret_cast<float4 *>(sm.S + (e / D) * R + e % D) = pf[u];
        }
    };
    // one forward token on the state in shared memory, S <- S_t: the four
    // threads of column j keep their quarter of it in registers, meet in
    // shuffles for u_j = beta (v_j - ((Diag(a) S)^T k)_j) and update their own
    // elements, so the token reads and writes S once, with no barrier between
    auto forward_token = [&](float bt) {
        __syncthreads();
        const int j = idx;
        float col[Q];
        float2 akr[Q];
        float r0 = 0.f, r1 = 0.f;
#pragma unroll
        for (int s = 0; s < Q; s += 2) {
            const int i0 = kParts * s + part, i1 = i0 + kParts;
            col[s] = sm.S[i0 * R + j];
            col[s + 1] = sm.S[i1 * R + j];
            akr[s] = sm.ak[i0];
            akr[s + 1] = sm.ak[i1];
            r0 = fmaf(akr[s].x * col[s], akr[s].y, r0);
            r1 = fmaf(akr[s + 1].x * col[s + 1], akr[s + 1].y, r1);
        }
        const float uj = bt * (sm.v[j] - quad_sum(r0 + r1));
#pragma unroll
        for (int s = 0; s < Q; ++s) {
            const int i = kParts * s + part;
            sm.S[i * R + j] = fmaf(akr[s].x, col[s], akr[s].y * uj);
        }
    };

    // ---- forward sweep: checkpoints before every 16th token
    if (h0) mat_from_global<D>(sm.S, h0 + unit * DD, tid);
    else mat_zero<D>(sm.S, tid);
    TokIn ti{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (s0 < s1) ti = fetch_token(s0, false);
    for (int64_t t = s0; t < s1; ++t) {
        if ((t - s0) % kChunk == 0) {
            __syncthreads();
            mat_to_global<D>(ck + (size_t)((t - s0) / kChunk) * DD, sm.S, tid);
        }
        __syncthreads();
        put_token(ti, false);
        const float bt = ti.beta;
        if (t + 1 < s1) ti = fetch_token(t + 1, false);
        forward_token(bt);
    }

    // ---- reverse sweep
    __syncthreads();
    if (dhT) mat_from_global<D>(sm.dS, dhT + unit * DD, tid);
    else mat_zero<D>(sm.dS, tid);
    for (int64_t c = n_chunks(L) - 1; c >= 0; --c) {
        const int64_t a0 = s0 + c * kChunk;
        const int64_t a1 = a0 + kChunk < s1 ? a0 + kChunk : s1;
        // the chunk's token states S_{t-1}, recomputed from its checkpoint
        __syncthreads();
        mat_from_global<D>(sm.S, ck + (size_t)c * DD, tid);
        ti = fetch_token(a0, false);
        for (int64_t t = a0; t < a1; ++t) {
            __syncthreads();
            mat_to_global<D>(tk + (size_t)(t - a0) * DD, sm.S, tid);
            put_token(ti, false);
            const float bt = ti.beta;
            if (t + 1 < a1) ti = fetch_token(t + 1, false);
            forward_token(bt);
        }
        // the reverse pass over the chunk: token t - 1's state and inputs load
        // while token t is differentiated
        __syncthreads();
        float4 pf[kPf];
        fetch_state(pf, tk + (size_t)(a1 - 1 - a0) * DD);
        ti = fetch_token(a1 - 1, true);
        for (int64_t t = a1 - 1; t >= a0; --t) {
            __syncthreads();
            put_state(pf);
            put_token(ti, true);
            const float bt = ti.beta;
            if (t > a0) {
                fetch_state(pf, tk + (size_t)(t - 1 - a0) * DD);
                ti = fetch_token(t - 1, true);
            }
            __syncthreads();
            const size_t x = ((size_t)t * H + h) * D;
            // columns: w = v - S'^T k, u = beta w (S = S_{t-1}, S' = Diag(a) S);
            // du = (dS + q dO^T)^T k = dS^T k + dO (q . k);  dv = beta du
            float dbp = 0.f;
            {
                const int j = idx;
                float r0 = 0.f, r1 = 0.f, d0 = 0.f, d1 = 0.f;
#pragma unroll 4
                for (int s = 0; s < Q; s += 2) {
                    const int i0 = kParts * s + part, i1 = i0 + kParts;
                    const float2 ak0 = sm.ak[i0], ak1 = sm.ak[i1];
                    r0 = fmaf(ak0.x * sm.S[i0 * R + j], ak0.y, r0);
                    r1 = fmaf(ak1.x * sm.S[i1 * R + j], ak1.y, r1);
                    d0 = fmaf(sm.dS[i0 * R + j], ak0.y, d0);
                    d1 = fmaf(sm.dS[i1 * R + j], ak1.y, d1);
                }
                const float r = quad_sum(r0 + r1), dsk = quad_sum(d0 + d1);
                if (part == 0) {
                    float qk = 0.f;
#pragma unroll
                    for (int p = 0; p < Smem<D>::kQkParts; ++p) qk += sm.qkp[p];
                    const float wj = sm.v[j] - r, du = fmaf(sm.vec[j].x, qk, dsk);
                    sm.vec[j].y = du;
                    sm.vec[j].z = bt * wj;
                    IO<T>::st(dv + x + j, bt * du);
                    dbp = du * wj;
                }
            }
            __syncthreads();
            // rows, one pass: dq = S_t dO = Diag(a) S dO + k (u . dO);
            // dS1 = dS + q dO^T;  dk = dS1 u - beta a (S du);
            // dS' = dS1 - beta k du^T;  da = sum_j dS' S;  dg = da a l';  dS <- Diag(a) dS'
            {
                // rows 4-7 of each group of eight (one warp) walk their columns
                // in the order s ^ 1, so that a warp's 32 lanes hit 32 banks
                const int i = idx, flip = (idx >> 2) & 1;
                const float qi = sm.q[i];
                const float2 aki = sm.ak[i];
                const float ai = aki.x, bki = bt * aki.y;
                float sd = 0.f, dsu = 0.f, sdu = 0.f, da = 0.f, udo = 0.f;
#pragma unroll 4
                for (int s = 0; s < Q; ++s) {
                    const int j = kParts * (s ^ flip) + part;
                    const float4 vj = sm.vec[j];             // dO_j, du_j, u_j
                    const float sij = sm.S[i * R + j];
                    udo = fmaf(vj.z, vj.x, udo);
                    sd = fmaf(sij, vj.x, sd);
                    const float ds = fmaf(qi, vj.x, sm.dS[i * R + j]);
                    dsu = fmaf(ds, vj.z, dsu);
                    sdu = fmaf(sij, vj.y, sdu);
                    const float dsp = fmaf(-bki, vj.y, ds);
                    da = fmaf(dsp, sij, da);
                    sm.dS[i * R + j] = ai * dsp;
                }
                sd = quad_sum(sd);
                dsu = quad_sum(dsu);
                sdu = quad_sum(sdu);
                da = quad_sum(da);
                udo = quad_sum(udo);
                if (part == 0) {
                    IO<T>::st(dq + x + i, fmaf(ai, sd, aki.y * udo));
                    IO<T>::st(dk + x + i, dsu - bt * ai * sdu);
                    IO<T>::st(dg + x + i, da * ai * sm.lg[i]);
                }
            }
            // dbeta = du . w (block reduction)
            for (int o = 16; o > 0; o >>= 1) dbp += __shfl_xor_sync(0xffffffffu, dbp, o);
            if ((tid & 31) == 0) sm.red[tid >> 5] = dbp;
            __syncthreads();
            if (tid == 0) {
                float sum = 0.f;
                for (int w = 0; w < NT / 32; ++w) sum += sm.red[w];
                IO<T>::st(dbeta + (size_t)t * H + h, sum);
            }
        }
    }
    __syncthreads();
    if (dh0) mat_to_global<D>(dh0 + unit * DD, sm.dS, tid);
}

}  // namespace bwd
}  // namespace kda
