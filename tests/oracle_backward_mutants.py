"""Deliberately wrong variants of the KDA backward pass (CPU, numpy).

Each mutant plants one plausible mistake in the reverse sweep; the backward
pins must reject every one.  With mutation=None this is a plain restatement
of the same chain rule, used only to show that a rejection is caused by the
planted mistake.  Never used as a reference.
"""
import numpy as np

MUTATIONS = (
    "no_read_grad",        # o_t = S_t^T q_t does not feed dS_t
    "no_delta_read_grad",  # r = S'^T k does not feed dS'
    "dk_missing_read",     # dk lacks the S' dr term
    "dg_sign",             # dg with the wrong sign
    "dh0_undecayed",       # dS_{t-1} = dS' instead of Diag(a) dS'
    "dbeta_uses_v",        # dbeta = du . v instead of du . (v - r)
    "dq_from_decayed",     # dq = S' do instead of S_t do
    "dv_no_beta",          # dv = du instead of beta du
)


def _sigmoid(x):
    with np.errstate(over="ignore"):
        return np.where(x >= 0, 1.0 / (1.0 + np.exp(-np.abs(x))),
                        np.exp(-np.abs(x)) / (1.0 + np.exp(-np.abs(x))))


def backward(q, k, v, g, beta, cu_seqlens, h0=None, d_o=None, d_hT=None,
             mutation=None):
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    cu = [int(x) for x in cu_seqlens]
    T, H, dk = q.shape
    dv = v.shape[2]
    N = len(cu) - 1
    out = {"dq": np.zeros((T, H, dk)), "dk": np.zeros((T, H, dk)),
           "dv": np.zeros((T, H, dv)), "dg": np.zeros((T, H, dk)),
           "dbeta": np.zeros((T, H)), "dh0": np.zeros((N, H, dk, dv))}
    for n in range(N):
        for h in range(H):
            S = np.zeros((dk, dv)) if h0 is None else np.array(h0[n, h], dtype=np.float64)
            before = []
            for t in range(cu[n], cu[n + 1]):
                before.append(S.copy())
                a = np.exp(-5.0 * _sigmoid(g[t, h]))
                Sp = a[:, None] * S
                u = beta[t, h] * (v[t, h] - Sp.T @ k[t, h])
                S = Sp + np.outer(k[t, h], u)
            dS = np.zeros((dk, dv)) if d_hT is None else np.array(d_hT[n, h], dtype=np.float64)
            for t in range(cu[n + 1] - 1, cu[n] - 1, -1):
                P = before[t - cu[n]]
                s = _sigmoid(g[t, h])
                a = np.exp(-5.0 * s)
                Sp = a[:, None] * P
                kt, vt, qt, bt = k[t, h], v[t, h], q[t, h], beta[t, h]
                r = Sp.T @ kt
                u = bt * (vt - r)
                St = Sp + np.outer(kt, u)
                do = np.zeros(dv) if d_o is None else np.asarray(d_o[t, h], dtype=np.float64)
                out["dq"][t, h] = (Sp if mutation == "dq_from_decayed" else St) @ do
                if mutation != "no_read_grad":
                    dS = dS + np.outer(qt, do)
                du = dS.T @ kt
                dkk = dS @ u
                out["dbeta"][t, h] = du @ (vt if mutation == "dbeta_uses_v" else vt - r)
                out["dv"][t, h] = du if mutation == "dv_no_beta" else bt * du
                dr = -bt * du
                if mutation != "dk_missing_read":
                    dkk = dkk + Sp @ dr
                if mutation != "no_delta_read_grad":
                    dS = dS + np.outer(kt, dr)
                out["dk"][t, h] = dkk
                da = np.sum(dS * P, axis=1)
                dg = da * a * (-5.0 * s * (1.0 - s))
                out["dg"][t, h] = -dg if mutation == "dg_sign" else dg
                if mutation != "dh0_undecayed":
                    dS = a[:, None] * dS
            out["dh0"][n, h] = dS
    return out
