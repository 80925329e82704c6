"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Kairos (arXiv 2606.16533): section 2.2.1 (gated delta memory, Eq. (2)-(6),
o_t = S_t q_t), section 2.2.2 (SWA Eq. (7), DSWA Eq. (8)), section 2.3.2
(contraction, Eq. (18)).  The pages print no worked numeric example, so the
pins are closed forms, library routines, invariants, special cases and a
second independent restatement (``oracle.twin``).  Each is chosen so that a
plausible slip (dropped decay, wrong sign, transposed state, off-by-one
window, wrong residue class, wrong softmax scale) fails at least one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import twin
from workloads import WORKLOADS, make_inputs, bf16_bits, bf16_to_float32


def rnd(shape, seed, normalise=False):
    r = np.random.default_rng(seed).standard_normal(shape)
    if normalise:
        r /= np.linalg.norm(r, axis=-1, keepdims=True)
    return r.astype(np.float32)


def gates_ab(shape, seed):
    r = np.random.default_rng(seed)
    alpha = np.exp(-np.logaddexp(0, r.standard_normal(shape) + 2)).astype(np.float32)
    beta = (1 / (1 + np.exp(-r.standard_normal(shape)))).astype(np.float32)
    return alpha, beta


# --------------------------------------------------------------------------
# Sliding-window attention (Eq. (7), causal reading)
# --------------------------------------------------------------------------

def test_swa_full_window_equals_causal_sdpa():
    """w >= L: the window covers every earlier key -> full causal attention,
    compared with torch's fp64 scaled_dot_product_attention(is_causal=True)."""
    B, L, H, d = 2, 37, 3, 16
    q, k, v = rnd((B, L, H, d), 1), rnd((B, L, H, d), 2), rnd((B, L, H, d), 3)
    o = oracle.attention("swa", q, k, v, P=1, dilation=1, w=L + 5)
    t = lambda a: torch.from_numpy(a).double().permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-13)


def test_swa_band_equals_sdpa_with_band_mask():
    """Band window vs the library's masked softmax (boolean mask)."""
    B, L, H, d, w = 1, 50, 2, 8, 7
    q, k, v = rnd((B, L, H, d), 4), rnd((B, L, H, d), 5), rnd((B, L, H, d), 6)
    o = oracle.attention("swa", q, k, v, P=1, dilation=1, w=w)
    i = torch.arange(L)[:, None]
    j = torch.arange(L)[None, :]
    mask = (j <= i) & (j > i - w)
    t = lambda a: torch.from_numpy(a).double().permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=mask)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-13)


@pytest.mark.parametrize("w", [1, 3, 8])
def test_swa_uniform_logits_average_the_window(w):
    """q = 0 makes every logit equal: row i is the plain mean of the values of
    exactly min(i+1, w) most recent keys (self included)."""
    B, L, H, d = 1, 20, 1, 4
    q = np.zeros((B, L, H, d), np.float32)
    k = rnd((B, L, H, d), 7)
    v = rnd((B, L, H, 6), 8)
    o = oracle.attention("swa", q, k, v, P=1, dilation=1, w=w)
    for i in range(L):
        lo = max(0, i - w + 1)
        np.testing.assert_allclose(o[0, i, 0], v[0, lo:i + 1, 0].astype(np.float64).mean(0),
                                   rtol=0, atol=1e-14)


def test_swa_window_one_returns_own_value():
    B, L, H, d = 1, 9, 2, 4
    q, k, v = rnd((B, L, H, d), 9), rnd((B, L, H, d), 10), rnd((B, L, H, 3), 11)
    o = oracle.attention("swa", q, k, v, P=1, dilation=1, w=1)
    np.testing.assert_array_equal(o, v.astype(np.float64))


def test_softmax_rows_sum_to_one_constant_values():
    """Constant values pass through any softmax row unchanged."""
    B, L, H, d = 1, 30, 2, 8
    q, k = rnd((B, L, H, d), 12), rnd((B, L, H, d), 13)
    v = np.ones((B, L, H, 5), np.float32) * 3.0
    for kind, dil in (("swa", 1), ("dswa", 3)):
        o = oracle.attention(kind, q, k, v, P=4, dilation=dil, w=5)
        np.testing.assert_allclose(o, 3.0, rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# Dilated sliding-window attention (Eq. (8))
# --------------------------------------------------------------------------

@pytest.mark.parametrize("P,w", [(1, 5), (4, 6), (5, 13)])
def test_dswa_dilation_one_is_swa(P, w):
    """SWA is DSWA with d = 1 (section 2.2.2): identical results."""
    B, L, H, d = 1, 40, 2, 8
    q, k, v = rnd((B, L, H, d), 14), rnd((B, L, H, d), 15), rnd((B, L, H, d), 16)
    a = oracle.attention("dswa", q, k, v, P=P, dilation=1, w=w)
    b = oracle.attention("swa", q, k, v, P=P, dilation=1, w=w)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("P,dil,F,w", [(4, 2, 6, 5), (3, 4, 8, 7), (8, 3, 9, 10)])
def test_dswa_equals_literal_rearrange(P, dil, F, w):
    """F % d == 0: Eq. (8) executed literally -- reshape (B, F*P, D) into
    (B*d, F/d*P, D) with einops (residue classes of frames), then causal band
    attention per group with torch's SDPA -- equals the mask form."""
    import einops
    B, H, d = 2, 2, 8
    L = F * P
    q, k, v = rnd((B, L, H, d), 17), rnd((B, L, H, d), 18), rnd((B, L, H, d), 19)
    o = oracle.attention("dswa", q, k, v, P=P, dilation=dil, w=w)
    pat = "b (m g p) h d -> (b g) h (m p) d"
    rq, rk, rv = (einops.rearrange(torch.from_numpy(a).double(), pat, g=dil, p=P) for a in (q, k, v))
    n = rq.shape[2]
    i = torch.arange(n)[:, None]
    j = torch.arange(n)[None, :]
    mask = (j <= i) & (j > i - w)
    ro = torch.nn.functional.scaled_dot_product_attention(rq, rk, rv, attn_mask=mask)
    back = einops.rearrange(ro, "(b g) h (m p) d -> b (m g p) h d", g=dil, p=P)
    np.testing.assert_allclose(o, back.numpy(), rtol=0, atol=1e-13)


@pytest.mark.parametrize("P,dil,L,w", [(4, 3, 45, 6), (1, 4, 30, 3), (5, 2, 33, 8)])
def test_dswa_ragged_matches_twin(P, dil, L, w):
    """F % d != 0 and a partial last frame: the NumPy twin's gather/scatter
    route agrees with the mask form."""
    B, H, d = 1, 2, 6
    q, k, v = rnd((B, L, H, d), 20), rnd((B, L, H, d), 21), rnd((B, L, H, d), 22)
    o = oracle.attention("dswa", q, k, v, P=P, dilation=dil, w=w)
    np.testing.assert_allclose(o, twin.dswa(q, k, v, P, dil, w), rtol=0, atol=1e-13)


@pytest.mark.parametrize("P,dil,w", [(3, 4, 5), (8, 2, 20), (5, 3, 4), (1, 4, 7)])
def test_dswa_key_span_bound_is_a_superset(P, dil, w):
    """The restricted key scan used for long sequences gives the same rows as
    scanning every earlier key."""
    B, L, H, d = 1, 120, 1, 4
    q, k, v = rnd((B, L, H, d), 23), rnd((B, L, H, d), 24), rnd((B, L, H, d), 25)
    a = oracle.attention("dswa", q, k, v, P=P, dilation=dil, w=w)
    b = oracle.attention("dswa", q, k, v, P=P, dilation=dil, w=w, span=-1)
    np.testing.assert_array_equal(a, b)


def test_dswa_uniform_logits_average_residue_class():
    """q = 0: row i averages the values of its own frame class that lie within
    w rearranged positions; checked on frame-level indices by hand."""
    P, dil, w, L = 2, 3, 3, 24
    q = np.zeros((1, L, 1, 4), np.float32)
    k = rnd((1, L, 1, 4), 26)
    v = rnd((1, L, 1, 2), 27)
    o = oracle.attention("dswa", q, k, v, P=P, dilation=dil, w=w)
    # query t = 19: frame 9 (class 0), s = 1 -> class-0 frames 0,3,6,9 -> r = 7.
    # Keys with r in {5,6,7}: frame 6 s=1 (t=13), frame 9 s=0 (t=18), t=19.
    np.testing.assert_allclose(o[0, 19, 0], v[0, [13, 18, 19], 0].astype(np.float64).mean(0),
                               atol=1e-14)
    # query t = 4: frame 2 (class 2), s = 0, first frame of its class -> only itself.
    np.testing.assert_allclose(o[0, 4, 0], v[0, 4, 0], atol=1e-14)


# --------------------------------------------------------------------------
# Gated delta memory (section 2.2.1)
# --------------------------------------------------------------------------

def _gdn_case(B=1, L=24, H=2, dk=8, dv=5, seed=30):
    q, k = rnd((B, L, H, dk), seed, True), rnd((B, L, H, dk), seed + 1, True)
    v = rnd((B, L, H, dv), seed + 2)
    alpha, beta = gates_ab((B, L, H), seed + 3)
    return q, k, v, alpha, beta


def test_gdn_four_step_equals_matrix_form():
    """Retrieve / interpolate / remove / write (Eq. (2), (5) on the decayed
    state) equals alpha S (I - beta k k^T) + beta v k^T as a matrix product."""
    q, k, v, a, b = _gdn_case(dk=8, dv=8)
    S0 = np.random.default_rng(1).standard_normal((1, 2, 8, 8))
    o1, S1 = oracle.gdn(q, k, v, a, b, S0)
    o2, S2 = oracle.gdn(q, k, v, a, b, S0, matrix_form=True)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S1, S2, rtol=0, atol=1e-12)


def _states(q, k, v, a, b, S0, variant=0):
    """All states S_0..S_L by chaining one-token oracle calls."""
    L = q.shape[1]
    Ss = [S0]
    S = S0
    for t in range(L):
        _, S = oracle.gdn(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], a[:, t:t + 1],
                          b[:, t:t + 1], S, variant=variant)
        Ss.append(S)
    return Ss


def test_gdn_chained_single_steps_equal_one_shot():
    q, k, v, a, b = _gdn_case()
    S0 = np.random.default_rng(2).standard_normal((1, 2, 5, 8))
    Ss = _states(q, k, v, a, b, S0)
    _, S = oracle.gdn(q, k, v, a, b, S0)
    np.testing.assert_array_equal(Ss[-1], S)


def test_gdn_retrieval_identity():
    """S_t k_t = alpha_t (1 - beta_t |k_t|^2) S_{t-1} k_t + beta_t |k_t|^2 v_t;
    for unit k the decayed old association is kept with weight 1-beta and the
    new value written with weight beta."""
    q, k, v, a, b = _gdn_case()
    S0 = np.random.default_rng(3).standard_normal((1, 2, 5, 8))
    Ss = _states(q, k, v, a, b, S0)
    for t in range(q.shape[1]):
        for h in range(2):
            kt = k[0, t, h].astype(np.float64)
            kk = kt @ kt
            lhs = Ss[t + 1][0, h] @ kt
            rhs = (a[0, t, h] * (1 - b[0, t, h] * kk) * (Ss[t][0, h] @ kt)
                   + b[0, t, h] * kk * v[0, t, h])
            np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-12)


def test_gdn_exact_memorisation_alpha_beta_one():
    """alpha = beta = 1: after writing (k_t, v_t) the memory returns v_t for k_t
    (keys exactly unit: a power-of-two scaled basis-free choice, k = e_i)."""
    q, k, v, _, _ = _gdn_case()
    rng = np.random.default_rng(44)
    k = np.zeros_like(k)
    idx = rng.integers(0, k.shape[-1], size=k.shape[:-1])
    np.put_along_axis(k, idx[..., None], 1.0, axis=-1)
    ones = np.ones((1, q.shape[1], 2), np.float32)
    S0 = np.random.default_rng(4).standard_normal((1, 2, 5, 8))
    Ss = _states(q, k, v, ones, ones, S0)
    for t in range(q.shape[1]):
        np.testing.assert_allclose(Ss[t + 1][0, :, :, :] @ k[0, t, :, :, None].astype(np.float64),
                                   v[0, t, :, :, None], rtol=0, atol=1e-12)


def test_gdn_output_reads_updated_state():
    """o_t = S_t q_t with the state after the step-t update (step 4)."""
    q, k, v, a, b = _gdn_case()
    S0 = np.random.default_rng(5).standard_normal((1, 2, 5, 8))
    Ss = _states(q, k, v, a, b, S0)
    o, _ = oracle.gdn(q, k, v, a, b, S0)
    for t in range(q.shape[1]):
        np.testing.assert_allclose(o[0, t], np.einsum("hvk,hk->hv", Ss[t + 1][0], q[0, t]),
                                   rtol=0, atol=1e-12)


def test_gdn_single_token_closed_form():
    """From S_0 = 0 one step gives S_1 = beta v k^T, so o_1 = beta (k . q) v."""
    q, k, v, a, b = _gdn_case(L=1)
    o, S = oracle.gdn(q, k, v, a, b)
    for h in range(2):
        kq = float(k[0, 0, h].astype(np.float64) @ q[0, 0, h])
        bb, vv = np.float64(b[0, 0, h]), v[0, 0, h].astype(np.float64)
        np.testing.assert_allclose(o[0, 0, h], bb * kq * vv, rtol=0, atol=1e-14)
        np.testing.assert_allclose(S[0, h], bb * np.outer(vv, k[0, 0, h].astype(np.float64)),
                                   rtol=0, atol=1e-14)


def test_gdn_beta_zero_alpha_one_freezes_state():
    """beta = 0, alpha = 1: nothing is written or forgotten, S_t = S_0 and
    o_t = S_0 q_t."""
    q, k, v, _, _ = _gdn_case()
    L = q.shape[1]
    S0 = np.random.default_rng(6).standard_normal((1, 2, 5, 8))
    o, S = oracle.gdn(q, k, v, np.ones((1, L, 2), np.float32), np.zeros((1, L, 2), np.float32), S0)
    np.testing.assert_allclose(S, S0, rtol=0, atol=1e-13)  # remove-then-write rounds
    np.testing.assert_allclose(o[0], np.einsum("hvk,thk->thv", S0[0], q[0]), rtol=0, atol=1e-13)


def test_gdn_orthonormal_keys_reduce_to_linear_attention():
    """alpha = beta = 1 with mutually orthonormal keys (L <= d_k): the delta
    correction never fires, S_t = sum_{s<=t} v_s k_s^T, and the output is
    cumulative causal linear attention o_t = sum_{s<=t} (k_s . q_t) v_s."""
    L, dk, dv, H = 10, 16, 6, 2
    rng = np.random.default_rng(7)
    k = np.zeros((1, L, H, dk), np.float32)
    for h in range(H):
        Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
        k[0, :, h] = Qm[:, :L].T
    q = rnd((1, L, H, dk), 31)
    v = rnd((1, L, H, dv), 32)
    ones = np.ones((1, L, H), np.float32)
    o, _ = oracle.gdn(q, k, v, ones, ones)
    k64, q64, v64 = (a.astype(np.float64) for a in (k, q, v))
    for t in range(L):
        ref = np.einsum("sh,shv->hv", np.einsum("shk,hk->sh", k64[0, :t + 1], q64[0, t]),
                        v64[0, :t + 1])
        np.testing.assert_allclose(o[0, t], ref, rtol=0, atol=1e-6)


def test_gdn_step_is_contraction_with_factor_alpha():
    """The linear part of one step, S -> alpha S (I - beta k k^T), read off the
    oracle with v = 0 and S_0 = I, has spectral norm exactly alpha for unit k and
    beta in [0, 1] (section 2.3.2: contractive with rho = alpha < 1)."""
    rng = np.random.default_rng(8)
    dk = 12
    for trial in range(6):
        kv = rng.standard_normal(dk)
        kv /= np.linalg.norm(kv)
        k = kv.astype(np.float32).reshape(1, 1, 1, dk)
        v = np.zeros((1, 1, 1, dk), np.float32)
        a = np.float32(rng.uniform(0.05, 0.99))
        b = np.float32(rng.uniform(0, 1)) if trial else np.float32(1.0)
        _, M = oracle.gdn(k, k, v, np.full((1, 1, 1), a), np.full((1, 1, 1), b),
                          np.eye(dk)[None, None])
        np.testing.assert_allclose(np.linalg.norm(M[0, 0], 2), a, rtol=1e-12)


def test_gdn_contraction_of_state_difference():
    """Two runs from different S_0 on identical inputs:
    ||S_t - S'_t||_F <= (prod_{s<=t} alpha_s) ||S_0 - S'_0||_F (Eq. (18), xi = 0)."""
    q, k, v, a, b = _gdn_case(L=16, H=1)
    rng = np.random.default_rng(9)
    S0, S0p = rng.standard_normal((2, 1, 1, 5, 8))
    A = _states(q, k, v, a, b, S0)
    Bs = _states(q, k, v, a, b, S0p)
    bound = np.linalg.norm(S0 - S0p)
    for t in range(16):
        bound *= float(a[0, t, 0])
        assert np.linalg.norm(A[t + 1] - Bs[t + 1]) <= bound * (1 + 1e-12)


def test_gdn_state_norm_bound():
    """||S_t||_F <= alpha_t ||S_{t-1}||_F + beta_t ||v_t||, hence bounded."""
    q, k, v, a, b = _gdn_case(L=30, H=1)
    S0 = np.random.default_rng(10).standard_normal((1, 1, 5, 8)) * 10
    Ss = _states(q, k, v, a, b, S0)
    for t in range(30):
        lhs = np.linalg.norm(Ss[t + 1])
        rhs = a[0, t, 0] * np.linalg.norm(Ss[t]) + b[0, t, 0] * np.linalg.norm(v[0, t, 0].astype(np.float64))
        assert lhs <= rhs * (1 + 1e-12)


def test_gdn_pages_variant_contraction_factor():
    """The equations as printed (Eq. (6): retrieval from the undecayed state)
    have linear part S -> S (alpha I - beta k k^T) with spectral norm
    max(alpha, |alpha - beta|) for unit k."""
    rng = np.random.default_rng(11)
    dk = 10
    for _ in range(5):
        kv = rng.standard_normal(dk)
        kv /= np.linalg.norm(kv)
        k = kv.astype(np.float32).reshape(1, 1, 1, dk)
        a, b = np.float32(rng.uniform(0.05, 0.99)), np.float32(rng.uniform(0, 1))
        _, M = oracle.gdn(k, k, np.zeros_like(k), np.full((1, 1, 1), a), np.full((1, 1, 1), b),
                          np.eye(dk)[None, None], variant=1)
        np.testing.assert_allclose(np.linalg.norm(M[0, 0], 2), max(a, abs(float(a) - float(b))),
                                   rtol=1e-12)


@pytest.mark.parametrize("C", [1, 7, 16, 64, 200])
def test_gdn_chunked_equals_recurrent(C):
    """The chunk regrouping (decay ratios, unit-lower solve, WY-style state
    coupling) reproduces the token recurrence in fp64."""
    q, k, v, a, b = _gdn_case(B=2, L=200, H=2, dk=16, dv=12)
    S0 = np.random.default_rng(12).standard_normal((2, 2, 12, 16))
    o1, S1 = oracle.gdn(q, k, v, a, b, S0)
    o2, S2 = oracle.gdn_chunked(q, k, v, a, b, C, S0)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-12)


def test_gdn_chunked_slow_decay():
    """Chunk form with alpha ~ 0.98 (long memory) still matches."""
    q, k, v, _, b = _gdn_case(B=1, L=150, H=1, dk=16, dv=16)
    a = np.full(b.shape, 0.98, np.float32)
    o1, S1 = oracle.gdn(q, k, v, a, b)
    o2, S2 = oracle.gdn_chunked(q, k, v, a, b, 64)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-11)
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-11)


# --------------------------------------------------------------------------
# Second restatement, streaming, combination
# --------------------------------------------------------------------------

@pytest.mark.parametrize("P", [1, 4, 8])
def test_twin_agrees_with_c_oracle(P):
    B, L, H, d = 1, 48, 2, 8
    q, k = rnd((B, L, H, d), 40, True), rnd((B, L, H, d), 41, True)
    v = rnd((B, L, H, d), 42)
    a, b = gates_ab((B, L, H), 43)
    np.testing.assert_allclose(oracle.attention("swa", q, k, v, P, 1, 9), twin.swa(q, k, v, 9),
                               rtol=0, atol=1e-13)
    np.testing.assert_allclose(oracle.attention("dswa", q, k, v, P, 4, 5),
                               twin.dswa(q, k, v, P, 4, 5), rtol=0, atol=1e-13)
    o1, S1 = oracle.gdn(q, k, v, a, b)
    o2, S2 = twin.gdn(q, k, v, a, b)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S1, S2, rtol=0, atol=1e-12)


def test_streaming_steps_equal_one_shot():
    """Carrying S and the key history across appends gives the one-shot rows
    and state exactly (same per-row arithmetic)."""
    wl = WORKLOADS["tiny_fp32"].with_(L=96, P=8, H=2, d_k=16, d_v=16, swa_window=12,
                                      dswa_window=10, dilation=3)
    inp = make_inputs(wl, seed=3)
    full = oracle.forward(inp)
    B, L, H = wl.B, wl.L, wl.H
    S = None
    for t0 in range(0, L, 20):
        t1 = min(L, t0 + 20)
        rows = np.array([(b * t1 + t) * H + h for b in range(B) for t in range(t0, t1)
                         for h in range(H)])
        sl = lambda a: np.ascontiguousarray(a[:, :t1])
        for kind, dil, w in (("swa", 1, wl.swa_window), ("dswa", wl.dilation, wl.dswa_window)):
            part = oracle.attention_rows(kind, sl(inp.q), sl(inp.k), sl(inp.v), wl.P, dil, w, rows)
            np.testing.assert_array_equal(part.reshape(B, t1 - t0, H, -1), full[kind][:, t0:t1])
        seg = lambda a: np.ascontiguousarray(a[:, t0:t1])
        o, S = oracle.gdn(seg(inp.q), seg(inp.k), seg(inp.v), seg(inp.alpha), seg(inp.beta), S)
        np.testing.assert_array_equal(o, full["gdn"][:, t0:t1])
    np.testing.assert_array_equal(S, full["S"])


def test_gates_isolate_branches():
    wl = WORKLOADS["tiny_fp32"].with_(L=40, P=4)
    inp = make_inputs(wl, seed=5)
    full = oracle.forward(inp)
    for i, name in enumerate(("swa", "dswa", "gdn")):
        g = np.zeros_like(inp.gates)
        g[:, i] = 1.0
        inp2 = make_inputs(wl, seed=5)
        inp2.gates = g
        np.testing.assert_array_equal(oracle.forward(inp2)["out"], full[name])


# --------------------------------------------------------------------------
# Input generator (no arithmetic of the method)
# --------------------------------------------------------------------------

def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1e-3, 3.0e38], np.float64)
    bits = bf16_bits(x)
    back = bf16_to_float32(bits)
    assert back[0] == 1.0 and back[1] == 1.0          # tie -> even (down)
    assert back[2] == 1.0 + 4 * 2 ** -8                # tie -> even (up)
    assert back[3] == -2.5
    assert abs(back[4] - 1e-3) <= 2 ** -9 * 1e-3
    assert np.all(torch.from_numpy(back).to(torch.bfloat16).float().numpy() == back)


def test_inputs_deterministic_and_distributed():
    wl = WORKLOADS["clip_4k"].with_(L=512)
    a = make_inputs(wl)
    b = make_inputs(wl)
    for n in ("q", "k", "v", "alpha", "beta", "gates"):
        np.testing.assert_array_equal(getattr(a, n), getattr(b, n))
    qn = np.linalg.norm(a.as_float32("q").astype(np.float64), axis=-1)
    assert np.all(np.abs(qn - 1) < 1e-2)
    assert 0.1 < a.alpha.mean() < 0.2 and a.alpha.max() < 1
    assert 0.3 < a.beta.mean() < 0.7


# --------------------------------------------------------------------------
# Centred windows and rotary embedding (the bidirectional reading of Eq. (7),
# RoPE on the sliding-window blocks)
# --------------------------------------------------------------------------

def _rand_qkv(B, L, H, d, seed=0):
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal((B, L, H, d)).astype(np.float32) for _ in range(3))


def _masked_softmax_attention(q, k, v, admit):
    """Dense softmax attention with an explicit [L, L] admission matrix
    (numpy library routines; a check independent of the oracle's loops)."""
    s = np.einsum("blhd,bmhd->bhlm", q.astype(np.float64), k.astype(np.float64)) / math.sqrt(q.shape[-1])
    s = np.where(admit[None, None], s, -np.inf)
    p = np.exp(s - s.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    return np.einsum("bhlm,bmhd->blhd", p, v.astype(np.float64))


def test_centred_window_wider_than_sequence_is_bidirectional_attention():
    q, k, v = _rand_qkv(1, 37, 2, 8)
    got = oracle.attention("swa", q, k, v, 1, 1, 1000, centred=True)
    want = _masked_softmax_attention(q, k, v, np.ones((37, 37), bool))
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)


def test_centred_window_band_matches_explicit_mask():
    L, w = 50, 9  # |i - j| <= 4
    q, k, v = _rand_qkv(1, L, 2, 8, seed=1)
    i = np.arange(L)
    admit = np.abs(i[:, None] - i[None, :]) <= w // 2
    got = oracle.attention("swa", q, k, v, 1, 1, w, centred=True)
    np.testing.assert_allclose(got, _masked_softmax_attention(q, k, v, admit), rtol=0, atol=1e-13)


def test_centred_half_window_zero_returns_own_value():
    q, k, v = _rand_qkv(1, 20, 3, 4, seed=2)
    got = oracle.attention("dswa", q, k, v, 4, 2, 1, centred=True)
    np.testing.assert_array_equal(got, v.astype(np.float64))


def test_centred_dswa_wide_window_is_attention_within_frame_class():
    P, dil, L = 5, 3, 40  # frames 0..7, classes f mod 3
    q, k, v = _rand_qkv(1, L, 2, 8, seed=3)
    f = np.arange(L) // P
    admit = (f[:, None] % dil) == (f[None, :] % dil)
    got = oracle.attention("dswa", q, k, v, P, dil, 10 * L, centred=True)
    np.testing.assert_allclose(got, _masked_softmax_attention(q, k, v, admit), rtol=0, atol=1e-13)


def test_rope_single_pair_scores_are_cosines_of_the_position_gap():
    # d = 2: q_t = k_t = (1, 0) and base irrelevant (theta_0 = 1), so
    # s_ij = cos(i - j) / sqrt(2) exactly; v_t = t picks out the weights.
    L = 12
    q = np.zeros((1, L, 1, 2), np.float32)
    q[..., 0] = 1.0
    k = q.copy()
    v = np.arange(L, dtype=np.float32).reshape(1, L, 1, 1) * np.ones((1, 1, 1, 2), np.float32)
    got = oracle.attention("swa", q, k, v, 1, 1, 1000, centred=True, rope_base=10000.0)
    i = np.arange(L)
    s = np.cos(i[:, None] - i[None, :]) / math.sqrt(2.0)
    p = np.exp(s - s.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    np.testing.assert_allclose(got[0, :, 0, 0], p @ i, rtol=0, atol=1e-12)


def test_rope_scores_depend_only_on_relative_position():
    # prepending tokens shifts every position by c; rows whose window does not
    # reach the prefix must come out the same
    c, L, w = 7, 30, 9
    q, k, v = _rand_qkv(1, L, 2, 16, seed=4)
    jq, jk, jv = _rand_qkv(1, c, 2, 16, seed=5)
    cat = lambda a, b: np.concatenate([a, b], axis=1)
    base = oracle.attention("swa", q, k, v, 1, 1, w, centred=True, rope_base=500.0)
    shifted = oracle.attention("swa", cat(jq, q), cat(jk, k), cat(jv, v), 1, 1, w, centred=True,
                               rope_base=500.0)[:, c:]
    rows = slice(w // 2, L - w // 2)
    np.testing.assert_allclose(shifted[:, rows], base[:, rows], rtol=0, atol=1e-12)
    # and rotation is not the identity: without it the outputs differ
    plain = oracle.attention("swa", q, k, v, 1, 1, w, centred=True)
    assert np.abs(plain - base).max() > 1e-3


# --------------------------------------------------------------------------
# Backward pass: reverse-mode derivatives of the forward definitions
# --------------------------------------------------------------------------

def _central_difference(fn, arr, idx, eps=1e-3):
    """d fn / d arr[idx] by a central difference taken on the float32 values the
    oracle actually reads (the step is measured after rounding)."""
    a = arr.copy()
    a[idx] += eps
    hi, f_hi = float(a[idx]), fn(a)
    a = arr.copy()
    a[idx] -= eps
    lo, f_lo = float(a[idx]), fn(a)
    return (f_hi - f_lo) / (hi - lo)


_PROBES4 = [(0, 0, 0, 0), (0, 3, 1, 2), (0, 7, 0, 1), (0, 12, 1, 3)]


@pytest.mark.parametrize("kind,P,dil,w,centred,rope", [
    ("swa", 1, 1, 4, False, 0.0), ("dswa", 2, 2, 3, False, 0.0), ("swa", 1, 1, 5, True, 100.0),
    ("dswa", 3, 2, 4, True, 10.0), ("swa", 1, 1, 30, False, 0.0)])
def test_attention_backward_matches_central_differences(kind, P, dil, w, centred, rope):
    q, k, v = (rnd((1, 13, 2, 4), s) for s in (1, 2, 3))
    dO = np.random.default_rng(4).standard_normal((1, 13, 2, 4))
    dq, dk, dv = oracle.attention_backward(kind, q, k, v, P, dil, w, dO, centred=centred,
                                           rope_base=rope)
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in _PROBES4:
            def loss(a):
                qq, kk, vv = {"q": (a, k, v), "k": (q, a, v), "v": (q, k, a)}[name]
                o = oracle.attention(kind, qq, kk, vv, P, dil, w, centred=centred, rope_base=rope)
                return float((o * dO).sum())
            assert abs(_central_difference(loss, arr, idx) - grad[idx]) < 1e-6, (name, idx)


def test_attention_backward_single_key_and_invariants():
    q, k, v = (rnd((2, 20, 3, 8), s) for s in (5, 6, 7))
    dO = np.random.default_rng(8).standard_normal((2, 20, 3, 8))
    # w = 1: o = v, so dv = dO and nothing reaches q or k
    dq, dk, dv = oracle.attention_backward("swa", q, k, v, 1, 1, 1, dO)
    assert np.abs(dq).max() == 0 and np.abs(dk).max() == 0
    np.testing.assert_allclose(dv, dO, rtol=0, atol=1e-15)
    # softmax rows sum to one: sum_j dv_j = sum_i dO_i; logits are shift invariant
    # per query: sum_j dk_j = 0 (each query's ds sums to zero)
    for kind, P, dil, w in (("swa", 1, 1, 6), ("dswa", 4, 2, 5)):
        dq, dk, dv = oracle.attention_backward(kind, q, k, v, P, dil, w, dO)
        np.testing.assert_allclose(dv.sum(axis=1), dO.sum(axis=1), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)


@pytest.mark.parametrize("variant", [0, 1])
@pytest.mark.parametrize("L", [13, 150])
def test_gdn_backward_matches_central_differences(variant, L):
    """L = 150 crosses the oracle's 64-step recompute segments."""
    q = rnd((1, L, 2, 4), 11)
    k = rnd((1, L, 2, 4), 12, normalise=True)
    v = rnd((1, L, 2, 4), 13)
    r = np.random.default_rng(14)
    alpha = r.uniform(0.5, 0.99, (1, L, 2)).astype(np.float32)
    beta = r.uniform(0.1, 0.9, (1, L, 2)).astype(np.float32)
    S0 = r.standard_normal((1, 2, 4, 4)) * 0.3
    dSf = r.standard_normal((1, 2, 4, 4))
    dO = r.standard_normal((1, L, 2, 4))
    g = oracle.gdn_backward(q, k, v, alpha, beta, dO, S0, dSf, variant)

    def loss(qq=q, kk=k, vv=v, aa=alpha, bb=beta, SS=S0):
        o, S = oracle.gdn(qq, kk, vv, aa, bb, SS, variant=variant)
        return float((o * dO).sum() + (S * dSf).sum())
    ts = [0, 5, L // 2, L - 1]
    for name, arr, grad in (("qq", q, g["dq"]), ("kk", k, g["dk"]), ("vv", v, g["dv"])):
        for t in ts:
            idx = (0, t, t % 2, (3 * t) % 4)
            n = _central_difference(lambda a: loss(**{name: a}), arr, idx)
            assert abs(n - grad[idx]) < 1e-6 * (1 + abs(n)), (name, idx, n, grad[idx])
    for name, arr, grad in (("aa", alpha, g["dalpha"]), ("bb", beta, g["dbeta"])):
        for t in ts:
            idx = (0, t, (t + 1) % 2)
            n = _central_difference(lambda a: loss(**{name: a}), arr, idx, eps=1e-4)
            assert abs(n - grad[idx]) < 1e-6 * (1 + abs(n)), (name, idx, n, grad[idx])
    for idx in ((0, 0, 0, 0), (0, 1, 2, 3)):
        a = S0.copy()
        a[idx] += 1e-6
        f_hi = loss(SS=a)
        a[idx] -= 2e-6
        n = (f_hi - loss(SS=a)) / 2e-6
        assert abs(n - g["dS0"][idx]) < 1e-6 * (1 + abs(n))


@pytest.mark.parametrize("variant", [0, 1])
def test_gdn_backward_frozen_state_closed_form(variant):
    """beta = 0, alpha = 1 freezes the state (S_t = S0, o_t = S0 q_t).  Then
    dq_t = S0^T dO_t, dk = dv = 0, dS0 = dS_final + sum_t dO_t q_t^T, and with
    G_t = dS_final + sum_{s>=t} dO_s q_s^T: dalpha_t = <G_t, S0> and
    dbeta_t = (G_t k_t) . (v_t - S0 k_t)."""
    B, L, H, d = 1, 9, 2, 5
    q, v = rnd((B, L, H, d), 21), rnd((B, L, H, d), 23)
    k = rnd((B, L, H, d), 22, normalise=True)
    alpha = np.ones((B, L, H), np.float32)
    beta = np.zeros((B, L, H), np.float32)
    r = np.random.default_rng(24)
    S0, dSf = r.standard_normal((B, H, d, d)), r.standard_normal((B, H, d, d))
    dO = r.standard_normal((B, L, H, d))
    g = oracle.gdn_backward(q, k, v, alpha, beta, dO, S0, dSf, variant)
    q64, k64, v64 = (x.astype(np.float64) for x in (q, k, v))
    np.testing.assert_allclose(g["dq"], np.einsum("bhvk,blhv->blhk", S0, dO), atol=1e-12)
    assert np.abs(g["dk"]).max() == 0 and np.abs(g["dv"]).max() == 0
    np.testing.assert_allclose(g["dS0"], dSf + np.einsum("blhv,blhk->bhvk", dO, q64), atol=1e-12)
    for t in range(L):
        G = dSf + np.einsum("blhv,blhk->bhvk", dO[:, t:], q64[:, t:])
        np.testing.assert_allclose(g["dalpha"][:, t], np.einsum("bhvk,bhvk->bh", G, S0), atol=1e-11)
        Gk = np.einsum("bhvk,bhk->bhv", G, k64[:, t])
        resid = v64[:, t] - np.einsum("bhvk,bhk->bhv", S0, k64[:, t])
        np.testing.assert_allclose(g["dbeta"][:, t], (Gk * resid).sum(-1), atol=1e-11)


def test_layer_backward_gates_and_sum_match_central_differences():
    wl = WORKLOADS["tiny_fp32"].with_(L=24, H=2, d_k=4, d_v=4, P=2, swa_window=5, dswa_window=3,
                                      dilation=2)
    inp = make_inputs(wl, seed=3)
    dout = np.random.default_rng(5).standard_normal((1, 24, 2, 4))
    g = oracle.backward(inp, dout)

    def loss_with(**over):
        import dataclasses
        return float((oracle.forward(dataclasses.replace(inp, **over))["out"] * dout).sum())
    for idx in ((0, 0), (1, 1), (0, 2), (1, 2)):
        n = _central_difference(lambda a: loss_with(gates=a), inp.gates, idx)
        assert abs(n - g["dgates"][idx]) < 1e-6 * (1 + abs(n))
    # q feeds all three branches
    for idx in ((0, 3, 0, 1), (0, 20, 1, 3)):
        n = _central_difference(lambda a: loss_with(q=a), inp.q, idx)
        assert abs(n - g["dq"][idx]) < 1e-6 * (1 + abs(n))


@pytest.mark.parametrize("C,L", [(64, 150), (16, 70), (64, 64)])
def test_chunked_memory_backward_equals_recurrent_reverse_mode(C, L):
    """The chunk form of the memory backward (the algorithm the GPU follows)
    reproduces the token recurrence's reverse mode, including a ragged last chunk."""
    r = np.random.default_rng(31)
    q = rnd((1, L, 1, 8), 32)
    k = rnd((1, L, 1, 8), 33, normalise=True)
    v = rnd((1, L, 1, 8), 34)
    alpha = r.uniform(0.05, 0.99, (1, L, 1)).astype(np.float32)
    beta = r.uniform(0.05, 0.95, (1, L, 1)).astype(np.float32)
    S0 = r.standard_normal((1, 1, 8, 8)) * 0.3
    dSf = r.standard_normal((1, 1, 8, 8))
    dO = r.standard_normal((1, L, 1, 8))
    ref = oracle.gdn_backward(q, k, v, alpha, beta, dO, S0, dSf, 0)
    f = lambda a: a[0, :, 0].astype(np.float64)
    got = oracle.gdn_backward_chunked(f(q), f(k), f(v), f(alpha), f(beta), dO[0, :, 0], S0[0, 0], dSf[0, 0], C)
    for name in ("dq", "dk", "dv", "dalpha", "dbeta"):
        np.testing.assert_allclose(got[name], ref[name][0, :, 0], rtol=1e-9, atol=1e-11, err_msg=name)
    np.testing.assert_allclose(got["dS0"], ref["dS0"][0, 0], rtol=1e-9, atol=1e-11)


def test_e4m3_rounding_follows_the_format():
    """E4M3 (4 exponent bits, bias 7, 3 mantissa bits): representable values stay,
    ties go to the even mantissa, the subnormal spacing is 2^-9, and values past
    the largest finite 448 saturate."""
    r = oracle.fp8.e4m3_round
    for x in (0.0, 1.0, 1.125, 448.0, 240.0, 2.0 ** -6, 2.0 ** -9, -3.5, 0.875):
        assert r(x) == x
    assert r(1.0625) == 1.0 and r(1.1875) == 1.25          # ties to even
    assert r(3 * 2.0 ** -10) == 2.0 ** -8                  # subnormal tie to even (code 2)
    assert r(2.0 ** -11) == 0.0 and r(2.0 ** -10 + 2.0 ** -14) == 2.0 ** -9
    assert r(464.0) == 448.0 and r(1000.0) == 448.0 and r(-1e6) == -448.0
    assert r(447.0) == 448.0 and r(420.0) == 416.0         # spacing 32 in [256, 448]


def test_e4m3_rounding_matches_torch_float8():
    """In range, the model agrees with torch's float8_e4m3fn conversion (a library
    routine implementing the same format) on random and near-tie values."""
    x = np.concatenate([np.random.default_rng(41).standard_normal(20000) * 30,
                        np.random.default_rng(42).uniform(-2.0 ** -5, 2.0 ** -5, 5000)])
    x = x[np.abs(x) <= 440].astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.fp8.e4m3_round(x), ref)


def test_quantize_tiles_scale_and_error_bound():
    """Per 128-row tile: the largest magnitude maps to 448 exactly, and every
    element is within half an e4m3 spacing (relative 2^-4) of its input, or within
    the subnormal half-spacing 2^-10 * scale."""
    x = (np.random.default_rng(43).standard_normal((1, 300, 2, 16)) *
         np.linspace(0.1, 10, 300)[None, :, None, None]).astype(np.float32)
    deq, sc = oracle.fp8.quantize_tiles(x, Pseg=100)
    assert sc.shape == (3, 2, 1)
    for s in range(3):
        for h in range(2):
            tile = x[0, 100 * s:100 * (s + 1), h]
            assert sc[s, h, 0] == np.float32(np.abs(tile).max()) / np.float32(448.0)
            err = np.abs(deq[0, 100 * s:100 * (s + 1), h].astype(np.float64) - tile)
            bound = np.maximum(np.abs(tile) * 2.0 ** -4, 2.0 ** -10 * sc[s, h, 0]) * (1 + 1e-6)
            assert (err <= bound).all()
