"""The token-level chain rule the backward kernel evaluates, checked on the CPU
against the fp64 backward oracle (no GPU, no library code).

Per token t, in reverse, with S the state before the token, a = exp(l(g)),
l(g) = -5 sigmoid(g), S' = Diag(a) S, w = v - S'^T k, u = beta w,
S_t = S' + k u^T, o_t = S_t^T q, and dS = dL/dS_t on entry:

    dq = S_t dO;  dS += q dO^T;  du = dS^T k;  dk = dS u - beta S' du;
    dv = beta du;  dbeta = du . w;  dS' = dS - beta k du^T;
    da_i = sum_j dS'_ij S_ij;  dg = da * a * l'(g);  dS_{t-1} = Diag(a) dS'

The kernel takes du in the same pass as S'^T k, before dS is updated, by
du = (dS + q dO^T)^T k = dS^T k + dO (q . k).  Both orders are checked here
against oracle.backward (pinned on its own by central differences, the
adjoint identity and closed forms) for L = <dO, O> + <dhT, hT>.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_60_b200 import inputs


def token_grads(S, q, k, v, g, beta, dO, dS, du_first):
    sig = 1.0 / (1.0 + np.exp(-g))
    a = np.exp(-5.0 * sig)
    Sp = a[:, None] * S
    w = v - Sp.T @ k
    u = beta * w
    St = Sp + np.outer(k, u)
    dq = St @ dO
    if du_first:
        du = dS.T @ k + dO * (q @ k)          # before dS takes q dO^T
        dS = dS + np.outer(q, dO)
    else:
        dS = dS + np.outer(q, dO)
        du = dS.T @ k
    dk = dS @ u - beta * (Sp @ du)
    dv = beta * du
    dbeta = du @ w
    dSp = dS - beta * np.outer(k, du)
    da = np.sum(dSp * S, axis=1)
    dg = da * a * (-5.0 * sig * (1.0 - sig))
    return dq, dk, dv, dg, dbeta, a[:, None] * dSp, St


def backward(q, k, v, g, beta, cu, h0, dO, dhT, du_first):
    T, H, dk = q.shape
    dv = v.shape[2]
    N = len(cu) - 1
    out = {n: np.zeros(s) for n, s in (("dq", (T, H, dk)), ("dk", (T, H, dk)),
                                       ("dv", (T, H, dv)), ("dg", (T, H, dk)),
                                       ("dbeta", (T, H)), ("dh0", (N, H, dk, dv)))}
    for n in range(N):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            states = [h0[n, h].copy()]                # S before each token
            for t in range(t0, t1):
                S = states[-1]
                a = np.exp(-5.0 / (1.0 + np.exp(-g[t, h])))
                Sp = a[:, None] * S
                states.append(Sp + np.outer(k[t, h], beta[t, h] * (v[t, h] - Sp.T @ k[t, h])))
            dS = dhT[n, h].copy()
            for t in range(t1 - 1, t0 - 1, -1):
                r = token_grads(states[t - t0], q[t, h], k[t, h], v[t, h], g[t, h],
                                beta[t, h], dO[t, h], dS, du_first)
                (out["dq"][t, h], out["dk"][t, h], out["dv"][t, h], out["dg"][t, h],
                 out["dbeta"][t, h], dS, _) = r
            out["dh0"][n, h] = dS
    return out


@pytest.mark.parametrize("du_first", [False, True])
def test_token_chain_rule_equals_backward_oracle(du_first):
    lens = [0, 1, 23, 40]
    H, d = 2, 16
    inp = inputs.make_prefill(lens, H, d, d, torch.float32, seed=31, h0_std=0.05)
    q, k, v, g, beta = (x.double().numpy() for x in (inp.q, inp.k, inp.v, inp.g, inp.beta))
    g = g - 3.0                                  # slower decay: the carried state matters
    cu = inp.cu_seqlens.numpy()
    h0 = inp.h0.double().numpy()
    rng = np.random.default_rng(32)
    dO = rng.standard_normal(v.shape)
    dhT = rng.standard_normal(h0.shape)
    got = backward(q, k, v, g, beta, cu, h0, dO, dhT, du_first)
    ref = oracle.backward(q, k, v, g, beta, cu, h0=h0, d_o=dO, d_hT=dhT)
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        scale = max(np.max(np.abs(ref[name])), 1e-300)
        err = np.max(np.abs(got[name] - ref[name])) / scale
        assert err < 1e-12, (name, err)
