/*
 * kda_oracle.c -- fp64 CPU oracle for the Kimi Delta Attention (KDA) recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * definition that the CUDA path of libkda is checked against.  Only tests/,
 * __graft_entry__.smoke() and bench.py's CPU-baseline leg may load it.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (one head of one sequence, token by token, in fp64):
 *
 *   log a_t = -5 * sigmoid(g_t)                      per key channel
 *   S       = Diag(a_t) S                            decay the old state first
 *   u_t     = beta_t * (v_t - S^T k_t)               delta-rule error, read with
 *                                                    the *decayed* state
 *   S       = S + k_t u_t^T                          write only the difference
 *   o_t     = S^T q_t                                read from the *updated* state
 *
 * Sources (web pages on Kimi K3):
 *   - "Kimi K3 发布核实与 Moonshot AI 主干架构演变" (dllmharness report), §3,
 *     paragraph "KDA 为什么不同于 MLA": per-head state matrix; per-channel
 *     retention alpha decays the old state first, then the write strength beta
 *     with the current key and value corrects it, and the query reads the
 *     updated state.
 *   - same page, §3, "K3 对 Kimi Linear 的进一步修改", bullet 1: the
 *     log-decay is a scaled sigmoid bounded below by -5.
 *   - "Kimi K3 模型架构解析：KDA、AttnRes 与 Stable LatentMoE", §二.2
 *     (S_t = Update(S_{t-1}, k_t, v_t), o_t = Read(S_t, q_t)) and §二.3
 *     (delta rule: read the old mapping with the key, take the error
 *     against the value, write back only the difference).
 *
 * Readings where the pages are silent: beta arrives already in (0,1); no
 * query scale; q and k are used as given (their normalisation belongs to the
 * input); sequences restart from h0 (or zero) at each cu_seqlens boundary.
 *
 * kda_oracle_backward (at the end of the file) is the gradient of the same
 * prefill by the chain rule, token by token in reverse.
 *
 * Layouts (row-major, last index contiguous), all fp64:
 *   q, k, g  [T_tot, H, dk]      v, o  [T_tot, H, dv]      beta [T_tot, H]
 *   h0, hT   [N, H, dk, dv]      cu_seqlens int64 [N+1]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* log a = -5 * sigmoid(g), written so that g = +/-inf give exact limits. */
static double log_alpha(double g)
{
    double s;
    if (g >= 0.0) {
        s = 1.0 / (1.0 + exp(-g));
    } else {
        double e = exp(g);
        s = e / (1.0 + e);
    }
    return -5.0 * s;
}

/* The unbounded gate that K3 replaced (same page, same bullet: Kimi
 * Linear's negative-softplus log-decay): log a = -softplus(g) = -log(1 + e^g),
 * written so that g = -inf gives 0 and g = +inf gives -inf (a = 0). */
static double log_alpha_softplus(double g)
{
    if (g > 0.0) return -(g + log1p(exp(-g)));
    return -log1p(exp(g));
}

enum { GATE_SIGMOID5 = 0, GATE_SOFTPLUS = 1 };

static double log_alpha_mode(double g, int gate)
{
    return gate == GATE_SOFTPLUS ? log_alpha_softplus(g) : log_alpha(g);
}

/* One token of the recurrence on one head's state S [dk][dv] (in place).
 * o may be NULL.  r is scratch of length dv.  gate selects the log-decay. */
static void kda_token_gate(double *S, int dk, int dv,
                           const double *q, const double *k, const double *v,
                           const double *g, double beta, double *o, double *r,
                           int gate)
{
    /* decay first */
    for (int i = 0; i < dk; ++i) {
        double a = exp(log_alpha_mode(g[i], gate));
        double *row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) row[j] *= a;
    }
    /* r = S^T k with the decayed state */
    for (int j = 0; j < dv; ++j) r[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double *row = S + (size_t)i * dv;
        double ki = k[i];
        for (int j = 0; j < dv; ++j) r[j] += row[j] * ki;
    }
    /* u = beta (v - r);  S += k u^T */
    for (int j = 0; j < dv; ++j) r[j] = beta * (v[j] - r[j]);
    for (int i = 0; i < dk; ++i) {
        double *row = S + (size_t)i * dv;
        double ki = k[i];
        for (int j = 0; j < dv; ++j) row[j] += ki * r[j];
    }
    /* o = S^T q with the updated state */
    if (o) {
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double *row = S + (size_t)i * dv;
            double qi = q[i];
            for (int j = 0; j < dv; ++j) o[j] += row[j] * qi;
        }
    }
}

/* The token step with the K3 gate, log a = -5 sigmoid(g). */
static void kda_token(double *S, int dk, int dv,
                      const double *q, const double *k, const double *v,
                      const double *g, double beta, double *o, double *r)
{
    kda_token_gate(S, dk, dv, q, k, v, g, beta, o, r, GATE_SIGMOID5);
}

/*
 * Prefill: every token of every (sequence n, head h) unit whose mask byte is
 * nonzero (mask may be NULL = all units).  Units are independent; OpenMP runs
 * them in parallel, the tokens of a unit run in order.  gate: 0 = the K3
 * gate -5 sigmoid(g), 1 = the unbounded -softplus(g).
 * Returns 0, or -1 on a malformed cu_seqlens, an unknown gate or allocation
 * failure.
 */
int kda_oracle_forward_gate(const double *q, const double *k, const double *v,
                            const double *g, const double *beta, const double *h0,
                            const int64_t *cu_seqlens, int N, int64_t T_tot,
                            int H, int dk, int dv, const uint8_t *unit_mask,
                            double *o, double *hT, int gate)
{
    if (gate != GATE_SIGMOID5 && gate != GATE_SOFTPLUS) return -1;
    if (cu_seqlens[0] != 0 || cu_seqlens[N] != T_tot) return -1;
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    int err = 0;
    long units = (long)N * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        if (unit_mask && !unit_mask[u]) continue;
        int n = (int)(u / H), h = (int)(u % H);
        double *S = (double *)malloc(sizeof(double) * ((size_t)dk * dv + dv));
        if (!S) {
#pragma omp atomic write
            err = 1;
            continue;
        }
        double *r = S + (size_t)dk * dv;
        const size_t sz = (size_t)dk * dv;
        if (h0) memcpy(S, h0 + (size_t)u * sz, sizeof(double) * sz);
        else memset(S, 0, sizeof(double) * sz);
        for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
            size_t th = (size_t)t * H + h;
            kda_token_gate(S, dk, dv, q + th * dk, k + th * dk, v + th * dv,
                           g + th * dk, beta[th], o ? o + th * dv : NULL, r, gate);
        }
        if (hT) memcpy(hT + (size_t)u * sz, S, sizeof(double) * sz);
        free(S);
    }
    return err ? -1 : 0;
}

/* Prefill with the K3 gate. */
int kda_oracle_forward(const double *q, const double *k, const double *v,
                       const double *g, const double *beta, const double *h0,
                       const int64_t *cu_seqlens, int N, int64_t T_tot,
                       int H, int dk, int dv, const uint8_t *unit_mask,
                       double *o, double *hT)
{
    return kda_oracle_forward_gate(q, k, v, g, beta, h0, cu_seqlens, N, T_tot, H,
                                   dk, dv, unit_mask, o, hT, GATE_SIGMOID5);
}

/*
 * Decode: one token per (b, h); S [B, H, dk, dv] is updated in place and
 * o [B, H, dv] receives the read from the updated state.  The body is the
 * same token step as the prefill.
 */
int kda_oracle_decode(const double *q, const double *k, const double *v,
                      const double *g, const double *beta, double *S,
                      int B, int H, int dk, int dv, double *o)
{
    int err = 0;
    long units = (long)B * H;
#pragma omp parallel for schedule(static)
    for (long u = 0; u < units; ++u) {
        double *r = (double *)malloc(sizeof(double) * dv);
        if (!r) {
#pragma omp atomic write
            err = 1;
            continue;
        }
        kda_token(S + (size_t)u * dk * dv, dk, dv, q + (size_t)u * dk,
                  k + (size_t)u * dk, v + (size_t)u * dv, g + (size_t)u * dk,
                  beta[u], o ? o + (size_t)u * dv : NULL, r);
        free(r);
    }
    return err ? -1 : 0;
}

/* The gates on their own, so tests can pin them against closed forms. */
double kda_oracle_log_alpha(double g) { return log_alpha(g); }
double kda_oracle_log_alpha_softplus(double g) { return log_alpha_softplus(g); }

/* ------------------------------------------------------------------------
 * Backward pass: the gradient of the prefill by the chain rule, token by
 * token in reverse (the pages name training as the use of the chunked form:
 * "Kimi K3 发布核实与 Moonshot AI 主干架构演变", §3 "KDA 为什么不同于 MLA",
 * item 3).  Given dL/do_t and dL/dhT it returns dL/dq, dk, dv, dg, dbeta,
 * dh0 for L = <dO, O> + <dhT, hT>.
 * ---------------------------------------------------------------------- */

/* d(log a)/dg = -5 sigmoid(g) (1 - sigmoid(g)); 0 at g = +/-inf. */
static double dlog_alpha(double g)
{
    double s, c;   /* s = sigmoid(g), c = 1 - s = sigmoid(-g) */
    if (g >= 0.0) {
        double e = exp(-g);
        s = 1.0 / (1.0 + e);
        c = e / (1.0 + e);
    } else {
        double e = exp(g);
        s = e / (1.0 + e);
        c = 1.0 / (1.0 + e);
    }
    return -5.0 * s * c;
}

/*
 * Adjoint of one token step.  P is the state before the token (S_{t-1}).
 * On entry dS holds dL/dS_t from the later tokens (and hT); on exit it holds
 * dL/dS_{t-1}.  dout may be NULL (no gradient on o_t).  work has room for
 * 2 dk dv + 4 dv + dk doubles.  Forward quantities are recomputed from P:
 *   S' = Diag(a) P,  r = S'^T k,  u = beta (v - r),  S_t = S' + k u^T,
 *   o = S_t^T q.
 */
static void kda_token_backward(const double *P, int dk, int dv,
                               const double *q, const double *k,
                               const double *v, const double *g, double beta,
                               const double *dout, double *dS, double *dq,
                               double *dk_, double *dv_, double *dg,
                               double *dbeta, double *work)
{
    double *Sp = work;                       /* S'   [dk][dv] */
    double *St = Sp + (size_t)dk * dv;       /* S_t  [dk][dv] */
    double *r = St + (size_t)dk * dv;        /* dv */
    double *u = r + dv, *du = u + dv, *dr = du + dv;
    double *a = dr + dv;                     /* dk */

    /* recompute the forward step */
    for (int i = 0; i < dk; ++i) {
        a[i] = exp(log_alpha(g[i]));
        for (int j = 0; j < dv; ++j)
            Sp[(size_t)i * dv + j] = a[i] * P[(size_t)i * dv + j];
    }
    for (int j = 0; j < dv; ++j) r[j] = 0.0;
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) r[j] += Sp[(size_t)i * dv + j] * k[i];
    for (int j = 0; j < dv; ++j) u[j] = beta * (v[j] - r[j]);
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            St[(size_t)i * dv + j] = Sp[(size_t)i * dv + j] + k[i] * u[j];

    /* o = S_t^T q:  dq = S_t do,  dS_t += q do^T */
    for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        if (dout)
            for (int j = 0; j < dv; ++j) acc += St[(size_t)i * dv + j] * dout[j];
        dq[i] = acc;
    }
    if (dout)
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] += q[i] * dout[j];

    /* S_t = S' + k u^T:  du = dS_t^T k,  dk = dS_t u,  dS' = dS_t (+ below) */
    for (int j = 0; j < dv; ++j) du[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) {
            du[j] += dS[(size_t)i * dv + j] * k[i];
            acc += dS[(size_t)i * dv + j] * u[j];
        }
        dk_[i] = acc;
    }

    /* u = beta (v - r) */
    double db = 0.0;
    for (int j = 0; j < dv; ++j) {
        db += du[j] * (v[j] - r[j]);
        dv_[j] = beta * du[j];
        dr[j] = -beta * du[j];
    }
    *dbeta = db;

    /* r = S'^T k:  dk += S' dr,  dS' += k dr^T */
    for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) {
            acc += Sp[(size_t)i * dv + j] * dr[j];
            dS[(size_t)i * dv + j] += k[i] * dr[j];
        }
        dk_[i] += acc;
    }

    /* S' = Diag(a) P:  da_i = sum_j dS'_ij P_ij,  dg_i = da_i a_i dlog_alpha(g_i),
     * dP = Diag(a) dS' */
    for (int i = 0; i < dk; ++i) {
        double da = 0.0;
        for (int j = 0; j < dv; ++j) {
            da += dS[(size_t)i * dv + j] * P[(size_t)i * dv + j];
            dS[(size_t)i * dv + j] *= a[i];
        }
        dg[i] = da * a[i] * dlog_alpha(g[i]);
    }
}

/*
 * Backward of kda_oracle_forward.  dO [T_tot,H,dv] and dhT [N,H,dk,dv] may
 * be NULL (zero).  Outputs (all required except dh0, which may be NULL):
 * dq, dk, dg [T_tot,H,dk], dv [T_tot,H,dv], dbeta [T_tot,H], dh0 [N,H,dk,dv].
 * The states before each token are recomputed by the forward step from
 * checkpoints kept every kCkpt tokens, so memory per unit stays small; the
 * arithmetic is the same forward step.  Returns 0, or -1 on a malformed
 * cu_seqlens or allocation failure.
 */
int kda_oracle_backward(const double *q, const double *k, const double *v,
                        const double *g, const double *beta, const double *h0,
                        const int64_t *cu_seqlens, int N, int64_t T_tot,
                        int H, int dk, int dv, const double *dO,
                        const double *dhT, double *dq, double *dk_,
                        double *dv_, double *dg, double *dbeta, double *dh0)
{
    enum { kCkpt = 64 };
    if (cu_seqlens[0] != 0 || cu_seqlens[N] != T_tot) return -1;
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    int err = 0;
    long units = (long)N * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        int n = (int)(u / H), h = (int)(u % H);
        const int64_t t0 = cu_seqlens[n], t1 = cu_seqlens[n + 1];
        const int64_t L = t1 - t0;
        const int64_t nseg = (L + kCkpt - 1) / kCkpt;
        const size_t sz = (size_t)dk * dv;
        double *S = (double *)malloc(sizeof(double) * (2 * sz + dv));
        double *ckpt = (double *)malloc(sizeof(double) * sz * (size_t)(nseg > 0 ? nseg : 1));
        double *buf = (double *)malloc(sizeof(double) * sz * kCkpt);
        double *work = (double *)malloc(sizeof(double) * (2 * sz + 4 * (size_t)dv + dk));
        if (!S || !ckpt || !buf || !work) {
            free(S); free(ckpt); free(buf); free(work);
#pragma omp atomic write
            err = 1;
            continue;
        }
        double *dS = S + sz, *r = dS + sz;
        /* forward, keeping the state before every kCkpt-th token */
        if (h0) memcpy(S, h0 + (size_t)u * sz, sizeof(double) * sz);
        else memset(S, 0, sizeof(double) * sz);
        for (int64_t t = t0; t < t1; ++t) {
            if ((t - t0) % kCkpt == 0)
                memcpy(ckpt + (size_t)((t - t0) / kCkpt) * sz, S, sizeof(double) * sz);
            size_t th = (size_t)t * H + h;
            kda_token(S, dk, dv, q + th * dk, k + th * dk, v + th * dv,
                      g + th * dk, beta[th], NULL, r);
        }
        /* reverse sweep */
        if (dhT) memcpy(dS, dhT + (size_t)u * sz, sizeof(double) * sz);
        else memset(dS, 0, sizeof(double) * sz);
        for (int64_t sg = nseg - 1; sg >= 0; --sg) {
            const int64_t a0 = t0 + sg * kCkpt;
            const int64_t a1 = a0 + kCkpt < t1 ? a0 + kCkpt : t1;
            memcpy(S, ckpt + (size_t)sg * sz, sizeof(double) * sz);
            for (int64_t t = a0; t < a1; ++t) {
                memcpy(buf + (size_t)(t - a0) * sz, S, sizeof(double) * sz);
                size_t th = (size_t)t * H + h;
                kda_token(S, dk, dv, q + th * dk, k + th * dk, v + th * dv,
                          g + th * dk, beta[th], NULL, r);
            }
            for (int64_t t = a1 - 1; t >= a0; --t) {
                size_t th = (size_t)t * H + h;
                kda_token_backward(buf + (size_t)(t - a0) * sz, dk, dv,
                                   q + th * dk, k + th * dk, v + th * dv,
                                   g + th * dk, beta[th],
                                   dO ? dO + th * dv : NULL, dS,
                                   dq + th * dk, dk_ + th * dk, dv_ + th * dv,
                                   dg + th * dk, dbeta + th, work);
            }
        }
        if (dh0) memcpy(dh0 + (size_t)u * sz, dS, sizeof(double) * sz);
        free(S); free(ckpt); free(buf); free(work);
    }
    return err ? -1 : 0;
}
