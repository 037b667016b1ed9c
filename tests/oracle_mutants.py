"""Deliberately wrong variants of the KDA recurrence (CPU, numpy).

Each mutant plants one plausible mistake.  The pin suite must reject every one
of them; that is the evidence that the pins constrain every term of the
oracle (a dropped term, a wrong sign, a swapped order, a transposed operand).
These run on the CPU only and are never used as a reference.
"""
import numpy as np

MUTATIONS = (
    "read_before_write",    # o_t read from the decayed state before the write
    "decay_after_write",    # write first, then decay
    "undecayed_delta",      # delta read uses S_{t-1} instead of Diag(a_t) S_{t-1}
    "transposed_read",      # r = S k instead of S^T k (needs dk == dv)
    "gate_sign",            # log a = -5 sigmoid(-g)
    "gate_scale",           # log a = -sigmoid(g): the 5 dropped
    "beta_on_v_only",       # u = beta v - S^T k
    "no_beta",              # u = v - S^T k
    "decay_on_value_axis",  # Diag(a) applied along dv instead of dk (dk == dv)
)


def forward(q, k, v, g, beta, cu_seqlens, h0=None, mutation=None):
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
            for t in range(cu[n], cu[n + 1]):
                gg = g[t, h]
                with np.errstate(over="ignore"):
                    sig = 1.0 / (1.0 + np.exp(-gg))
                    if mutation == "gate_sign":
                        sig = 1.0 / (1.0 + np.exp(gg))
                la = -sig if mutation == "gate_scale" else -5.0 * sig
                a = np.exp(la)
                kt, vt, qt, bt = k[t, h], v[t, h], q[t, h], beta[t, h]
                if mutation == "decay_on_value_axis":
                    Sd = S * a[None, :]
                else:
                    Sd = a[:, None] * S
                Sread = S if mutation == "undecayed_delta" else Sd
                if mutation == "transposed_read":
                    r = Sread @ kt
                else:
                    r = Sread.T @ kt
                if mutation == "beta_on_v_only":
                    u = bt * vt - r
                elif mutation == "no_beta":
                    u = vt - r
                else:
                    u = bt * (vt - r)
                if mutation == "decay_after_write":
                    S = a[:, None] * (S + np.outer(kt, u))
                else:
                    S = Sd + np.outer(kt, u)
                if mutation == "read_before_write":
                    o[t, h] = Sd.T @ qt
                else:
                    o[t, h] = S.T @ qt
            hT[n, h] = S
    return o, hT
