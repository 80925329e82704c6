"""NumPy twin of the oracle: a second, independent restatement in pure Python
loops (tiny inputs only).  Test infrastructure only.

Kairos (arXiv 2606.16533), section 2.2.1 (gated delta memory, Eq. (2)-(6),
o_t = S_t q_t) and section 2.2.2 (SWA Eq. (7), DSWA Eq. (8)); the causal window
and residue-class readings are the same as the C oracle's.
"""
from __future__ import annotations

import math

import numpy as np


def _f64(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:
        a = (a.astype(np.uint32) << 16).view(np.float32)
    return a.astype(np.float64)


def swa(q, k, v, w):
    """Causal window of w keys: query i attends to keys j with i - w < j <= i."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, L, H, dk = q.shape
    out = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            for i in range(L):
                keys = [j for j in range(L) if i - w < j <= i]
                logits = np.array([q[b, i, h] @ k[b, j, h] for j in keys]) / math.sqrt(dk)
                p = np.exp(logits - logits.max())
                p /= p.sum()
                out[b, i, h] = sum(pj * v[b, j, h] for pj, j in zip(p, keys))
    return out


def dswa(q, k, v, P, dilation, w):
    """Eq. (8) executed literally: gather each residue class of frames
    (f = g, g + dilation, ...) into its own sequence, run the causal window on
    it, scatter the rows back.  Works for ragged classes (F % dilation != 0)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, L, H, dk = q.shape
    F = -(-L // P)
    out = np.zeros(v.shape)
    for g in range(dilation):
        idx = [t for f in range(g, F, dilation) for t in range(f * P, min((f + 1) * P, L))]
        if not idx:
            continue
        o = swa(q[:, idx], k[:, idx], v[:, idx], w)
        out[:, idx] = o
    return out


def gdn(q, k, v, alpha, beta, S0=None):
    """S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    alpha, beta = np.asarray(alpha, np.float64), np.asarray(beta, np.float64)
    B, L, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, L, H, dv))
    Sf = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dv, dk)) if S0 is None else np.array(S0[b, h], dtype=np.float64)
            for t in range(L):
                kt, qt, vt = k[b, t, h], q[b, t, h], v[b, t, h]
                a, be = alpha[b, t, h], beta[b, t, h]
                S = a * S @ (np.eye(dk) - be * np.outer(kt, kt)) + be * np.outer(vt, kt)
                out[b, t, h] = S @ qt
            Sf[b, h] = S
    return out, Sf
