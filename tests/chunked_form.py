"""Independent fp64 chunked (dense-within-chunk) form of the KDA recurrence.

Used only to pin the token-by-token oracle: it is written from the chunk
equations, not from the oracle's loop, and it forms every decay ratio
exp(b_r - b_i) directly (no reciprocal scaling), so it cannot share a mistake
with either the oracle or the CUDA path.

For one head and a chunk of rows r = 1..C with start state S0 (dk x dv):
  l_r   = -5 * sigmoid(g_r)                      (log-decay per key channel;
                                                  -softplus(g_r) for the
                                                  unbounded gate variant)
  b_r   = l_1 + ... + l_r                        (inclusive prefix sum)
  A_ri  = beta_r * sum_c k_rc k_ic exp(b_rc - b_ic)      for i < r, else 0
  T     = (I + A)^-1 Diag(beta)
  U     = T (V - (K * e^b) S0)
  M_ri  = sum_c q_rc k_ic exp(b_rc - b_ic)               for i <= r, else 0
  O     = (Q * e^b) S0 + M U
  S_C   = Diag(e^{b_C}) S0 + (K * e^{b_C - b})^T U
(The unrolled recurrence: every write k_i u_i^T made at row i has decayed by
exp(b_r - b_i) when row r reads it.)
"""
import numpy as np


def _log_decay(g, gate="sigmoid5"):
    with np.errstate(over="ignore"):
        if gate == "softplus":          # -log(1 + e^g), stable for large |g|
            return -(np.maximum(g, 0.0) + np.log1p(np.exp(-np.abs(g))))
        return -5.0 / (1.0 + np.exp(-g))


def chunk_step(q, k, v, g, beta, S0, gate="sigmoid5"):
    """One chunk.  q,k,g [C,dk]; v [C,dv]; beta [C]; S0 [dk,dv]."""
    C = q.shape[0]
    b = np.cumsum(_log_decay(g, gate), axis=0)               # [C, dk]
    # decay ratios for i <= r only (the others would be growth factors that
    # the causal masks drop; forming them could overflow for an unbounded gate)
    lower = np.tril(np.ones((C, C), dtype=bool))[:, :, None]
    ratio = np.exp(np.where(lower, b[:, None, :] - b[None, :, :], -np.inf))
    kk = np.einsum("rc,ic,ric->ri", k, k, ratio)
    qk = np.einsum("rc,ic,ric->ri", q, k, ratio)
    strict = np.tril(np.ones((C, C)), -1)
    causal = np.tril(np.ones((C, C)), 0)
    A = beta[:, None] * kk * strict
    T = np.linalg.solve(np.eye(C) + A, np.diag(beta))
    U = T @ (v - (k * np.exp(b)) @ S0)
    O = (q * np.exp(b)) @ S0 + (qk * causal) @ U
    S = np.exp(b[-1])[:, None] * S0 + (k * np.exp(b[-1][None, :] - b)).T @ U
    return O, S


def forward(q, k, v, g, beta, cu_seqlens, h0=None, chunk=16, gate="sigmoid5"):
    """Whole packed batch, chunk by chunk.  Same layouts as the oracle."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64)
                        for x in (q, k, v, g, beta))
    cu = [int(x) for x in cu_seqlens]
    T, H, dk = q.shape
    dv = v.shape[2]
    N = len(cu) - 1
    o = np.zeros((T, H, dv))
    hT = np.zeros((N, H, dk, dv))
    for n in range(N):
        for h in range(H):
            S = np.zeros((dk, dv)) if h0 is None else np.array(
                h0[n, h], dtype=np.float64)
            for s in range(cu[n], cu[n + 1], chunk):
                e = min(s + chunk, cu[n + 1])
                O, S = chunk_step(q[s:e, h], k[s:e, h], v[s:e, h],
                                  g[s:e, h], beta[s:e, h], S, gate)
                o[s:e, h] = O
            hT[n, h] = S
    return o, hT
