"""The chunk form of the memory backward, written plainly in fp64 NumPy.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle``): it restates the
algorithm the GPU's chunked memory backward follows, so that the algebra can be
checked against the token recurrence's reverse mode (``oracle.gdn_backward``)
by a pin in tests/test_oracle.py.  Nothing here is shared with the CUDA code.

Forward, per chunk of C tokens with start state S0 (section 2.2.1 recurrence
S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t,
regrouped; l_t = sum of log alpha from the chunk start, g_t = e^{l_t}):
    A_ts = beta_t e^{l_t - l_s} k_t.k_s (s < t),   T = (I + A)^-1
    R    = diag(beta) V - diag(beta g) K S0^T,     U = T R
    O    = diag(g) Q S0^T + P U,   P_ts = e^{l_t - l_s} q_t.k_s (s <= t)
    S_C  = g_C S0 + U^T diag(D) K,   D_s = e^{l_C - l_s}
Backward, given dO and dS_C (the chain rule through the four lines above):
    dU = P^T dO + diag(D) K dS_C^T,   dR = T^T dU,   dA = -dR U^T (s < t)
    dS0 = dO^T (diag(g) Q - P W) + dS_C (g_C I - (diag(D) K)^T W),  W = T diag(beta g) K
and the token gradients below; dS_C of a chunk is dS0 of the next one.
"""
from __future__ import annotations

import numpy as np


def _chunk_forward_pieces(q, k, v, alpha, beta, S0, t0, n):
    Q, K, V = q[t0:t0 + n], k[t0:t0 + n], v[t0:t0 + n]
    be, al = beta[t0:t0 + n], alpha[t0:t0 + n]
    ell = np.cumsum(np.log(al))
    gam = np.exp(ell)
    E = np.exp(ell[:, None] - ell[None, :])
    KK = K @ K.T
    A = np.tril(be[:, None] * E * KK, -1)
    T = np.linalg.inv(np.eye(n) + A)
    R = be[:, None] * V - (be * gam)[:, None] * (K @ S0.T)
    U = T @ R
    return Q, K, V, be, al, ell, gam, E, KK, T, U


def gdn_backward_chunked(q, k, v, alpha, beta, dO, S0=None, dS_final=None, C=64):
    """One (batch, head): q, k [L, d_k], v, dO [L, d_v], alpha, beta [L] (float64).
    Returns dq, dk, dv, dalpha, dbeta, dS0 of the decayed-retrieval update form."""
    L, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, dtype=np.float64)
    nch = (L + C - 1) // C
    starts = []
    for c in range(nch):                       # chunk start states
        t0, n = c * C, min(C, L - c * C)
        starts.append(S.copy())
        Q, K, V, be, al, ell, gam, E, KK, T, U = _chunk_forward_pieces(q, k, v, alpha, beta, S, t0, n)
        S = gam[-1] * S + U.T @ (np.exp(ell[-1] - ell)[:, None] * K)
    dS = np.zeros((dv, dk)) if dS_final is None else np.array(dS_final, dtype=np.float64)
    ends = [None] * nch
    for c in reversed(range(nch)):             # gradients of the chunk end states
        t0, n = c * C, min(C, L - c * C)
        Q, K, V, be, al, ell, gam, E, KK, T, U = _chunk_forward_pieces(q, k, v, alpha, beta, starts[c], t0, n)
        W = T @ ((be * gam)[:, None] * K)
        P = np.tril(E) * (Q @ K.T)
        ends[c] = dS.copy()
        Kd = np.exp(ell[-1] - ell)[:, None] * K
        dS = gam[-1] * dS - (dS @ Kd.T) @ W + dO[t0:t0 + n].T @ (gam[:, None] * Q - P @ W)
    out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
           "dalpha": np.zeros(L), "dbeta": np.zeros(L), "dS0": dS}
    for c in range(nch):                       # token gradients of each chunk
        t0, n = c * C, min(C, L - c * C)
        S0c, dSC = starts[c], ends[c]
        Q, K, V, be, al, ell, gam, E, KK, T, U = _chunk_forward_pieces(q, k, v, alpha, beta, S0c, t0, n)
        dOc = dO[t0:t0 + n]
        D = np.exp(ell[-1] - ell)
        M = np.tril(E)
        QK = Q @ K.T
        P = M * QK
        dU = P.T @ dOc + D[:, None] * (K @ dSC.T)
        dR = T.T @ dU
        dA = np.tril(-dR @ U.T, -1)
        dOU = dOc @ U.T
        Emat = dA * be[:, None] * E
        S0k = K @ S0c.T
        out["dq"][t0:t0 + n] = gam[:, None] * (dOc @ S0c) + (M * dOU) @ K
        out["dk"][t0:t0 + n] = ((M * dOU).T @ Q + D[:, None] * (U @ dSC) - (be * gam)[:, None] * (dR @ S0c)
                                + (Emat + Emat.T) @ K)
        out["dv"][t0:t0 + n] = be[:, None] * dR
        out["dbeta"][t0:t0 + n] = (dR * V).sum(1) - gam * (dR * S0k).sum(1) + (dA * E * KK).sum(1)
        # derivative with respect to l_t, then log alpha_tau = sum_{t >= tau} dl_t
        dl = gam * (dOc * (Q @ S0c.T)).sum(1)
        dM = dOU * P
        dl += dM.sum(1) - dM.sum(0)
        dl[-1] += gam[-1] * (dSC * S0c).sum()
        dD = (U * (K @ dSC.T)).sum(1) * D
        dl[-1] += dD.sum()
        dl -= dD
        dl -= gam * be * (dR * S0k).sum(1)
        Am = dA * be[:, None] * E * KK
        dl += Am.sum(1) - Am.sum(0)
        out["dalpha"][t0:t0 + n] = np.cumsum(dl[::-1])[::-1] / al
    return out
