"""ctypes front end of ``hlta_oracle.c`` (test infrastructure only)."""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hlta_oracle.c")
_LIB = os.path.join(_HERE, "libhlta_oracle.so")
_lib = None

_F32, _BF16 = 0, 1


def library_path() -> str:
    return _LIB


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE: no -ffast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        vp, dp, fp = ctypes.c_void_p, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_float)
        i, l = ctypes.c_int, ctypes.c_long
        lib.oracle_attention.argtypes = [i, i, i, i, i, i, i, i, i, vp, vp, vp, i, l,
                                         ctypes.POINTER(ctypes.c_longlong), l, dp]
        lib.oracle_attention.restype = i
        lib.oracle_attention_centred.argtypes = [i, ctypes.c_double, i, i, i, i, i, i, i, i, vp, vp, vp, i,
                                                 l, ctypes.POINTER(ctypes.c_longlong), l, dp]
        lib.oracle_attention_centred.restype = i
        lib.oracle_gdn.argtypes = [i, i, i, i, i, vp, vp, vp, i, fp, fp, dp, dp, dp, i, i]
        lib.oracle_gdn.restype = i
        lib.oracle_gdn_chunked.argtypes = [i, i, i, i, i, vp, vp, vp, i, fp, fp, dp, dp, dp, i]
        lib.oracle_gdn_chunked.restype = i
        lib.oracle_attention_backward.argtypes = [i, i, ctypes.c_double, i, i, i, i, i, i, i, i,
                                                  vp, vp, vp, i, dp, dp, dp, dp]
        lib.oracle_attention_backward.restype = i
        lib.oracle_gdn_backward.argtypes = [i, i, i, i, i, vp, vp, vp, i, fp, fp, dp, dp, dp, dp, dp,
                                            dp, dp, dp, dp, i]
        lib.oracle_gdn_backward.restype = i
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = i
        _lib = lib
    return _lib


def num_threads() -> int:
    return _load().oracle_num_threads()


def _tensor(a: np.ndarray):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return a, _BF16
    if a.dtype != np.float32:
        a = a.astype(np.float32)
    return a, _F32


def _dptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def dswa_span(P: int, dilation: int, w: int) -> int:
    """A key distance that every key of the dilated window stays within.

    A key j of query i (same frame class) satisfies i - j = dilation*g*P + s_i - s_j
    with g*P <= r(i) - r(j) + s_j - s_i < w + P, so i - j < dilation * (w + P)."""
    return dilation * (w + P)


def attention_rows(kind: str, q, k, v, P: int, dilation: int, w: int, rows=None,
                   span: int | None = None, centred: bool = False,
                   rope_base: float = 0.0) -> np.ndarray:
    """Softmax attention rows under the SWA ("swa") or DSWA ("dswa") mask.

    q, k: [B, L, H, d_k], v: [B, L, H, d_v] (uint16 bf16 bits or float32).
    rows: int64 row ids (b*L + t)*H + h, or None for all rows.  Returns
    [nrows, d_v] float64 (or [B, L, H, d_v] when rows is None).
    span: None chooses a provable bound; -1 examines every key.
    centred: the centred window |r(i) - r(j)| <= w // 2 instead of the causal
    one; rope_base > 0 rotates q and k by their token positions first
    (oracle_attention_centred in hlta_oracle.c).
    """
    lib = _load()
    q, dt = _tensor(q)
    k, dt2 = _tensor(k)
    v, dt3 = _tensor(v)
    assert dt == dt2 == dt3
    B, L, H, dk = q.shape
    dv = v.shape[-1]
    kind_i = {"swa": 0, "dswa": 1}[kind]
    if span is None:
        if centred:
            span = w // 2 if kind == "swa" else dswa_span(P, dilation, w // 2)
        else:
            span = w - 1 if kind == "swa" else dswa_span(P, dilation, w)
    if rows is None:
        n = B * L * H
        rp = None
        out = np.empty((B, L, H, dv), dtype=np.float64)
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows.size
        rp = rows.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong))
        out = np.empty((n, dv), dtype=np.float64)
    if centred or rope_base > 0.0:
        if not centred:
            raise ValueError("rotary embedding is provided with the centred window only")
        rc = lib.oracle_attention_centred(kind_i, float(rope_base), B, L, H, dk, dv, P, dilation, w,
                                          q.ctypes.data, k.ctypes.data, v.ctypes.data, dt, n, rp, span,
                                          _dptr(out))
    else:
        rc = lib.oracle_attention(kind_i, B, L, H, dk, dv, P, dilation, w,
                                  q.ctypes.data, k.ctypes.data, v.ctypes.data, dt, n, rp, span,
                                  _dptr(out))
    if rc != 0:
        raise ValueError("oracle_attention: bad arguments")
    return out


def attention(kind, q, k, v, P, dilation, w, span=None, centred=False, rope_base=0.0):
    return attention_rows(kind, q, k, v, P, dilation, w, None, span, centred, rope_base)


def _gdn_common(q, k, v, alpha, beta, S0):
    q, dt = _tensor(q)
    k, _ = _tensor(k)
    v, _ = _tensor(v)
    alpha = np.ascontiguousarray(alpha, dtype=np.float32)
    beta = np.ascontiguousarray(beta, dtype=np.float32)
    B, L, H, dk = q.shape
    dv = v.shape[-1]
    if S0 is not None:
        S0 = np.ascontiguousarray(S0, dtype=np.float64)
        assert S0.shape == (B, H, dv, dk)
    fptr = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
    return q, k, v, dt, fptr(alpha), fptr(beta), S0, (B, L, H, dk, dv)


def gdn(q, k, v, alpha, beta, S0=None, variant: int = 0, matrix_form: bool = False,
        want_out: bool = True):
    """Gated delta memory by the token recurrence.  Returns (out, S_final)."""
    lib = _load()
    q, k, v, dt, ap, bp, S0, (B, L, H, dk, dv) = _gdn_common(q, k, v, alpha, beta, S0)
    S = np.empty((B, H, dv, dk), dtype=np.float64)
    out = np.empty((B, L, H, dv), dtype=np.float64) if want_out else None
    rc = lib.oracle_gdn(B, L, H, dk, dv, q.ctypes.data, k.ctypes.data, v.ctypes.data, dt,
                        ap, bp, _dptr(S0), _dptr(S), _dptr(out), variant, int(matrix_form))
    if rc != 0:
        raise ValueError("oracle_gdn: bad arguments")
    return out, S


def gdn_chunked(q, k, v, alpha, beta, chunk: int, S0=None):
    """Gated delta memory by the chunk regrouping.  Returns (out, S_final)."""
    lib = _load()
    q, k, v, dt, ap, bp, S0, (B, L, H, dk, dv) = _gdn_common(q, k, v, alpha, beta, S0)
    S = np.empty((B, H, dv, dk), dtype=np.float64)
    out = np.empty((B, L, H, dv), dtype=np.float64)
    rc = lib.oracle_gdn_chunked(B, L, H, dk, dv, q.ctypes.data, k.ctypes.data, v.ctypes.data,
                                dt, ap, bp, _dptr(S0), _dptr(S), _dptr(out), chunk)
    if rc != 0:
        raise ValueError("oracle_gdn_chunked: bad arguments")
    return out, S


def forward(inp, S0=None, branches=("swa", "dswa", "gdn"), variant=0):
    """The whole layer: out = g_swa[h]*SWA + g_dswa[h]*DSWA + g_gdn[h]*GDN.

    inp: a ``workloads.Inputs``.  The branch combination (a per-head weighted
    sum) is the specification's; the pages leave it open.  variant selects the
    memory update form of ``gdn`` (0: decayed retrieval, 1: Eq. (2)/(6) as
    printed).
    Returns dict with 'out' [B,L,H,d_v], per-branch outputs and 'S'.
    """
    wl = inp.wl
    res = {}
    g = inp.gates.astype(np.float64)
    total = 0.0
    if "swa" in branches:
        res["swa"] = attention("swa", inp.q, inp.k, inp.v, wl.P, 1, wl.swa_window)
        total = total + g[None, None, :, 0, None] * res["swa"]
    if "dswa" in branches:
        res["dswa"] = attention("dswa", inp.q, inp.k, inp.v, wl.P, wl.dilation, wl.dswa_window)
        total = total + g[None, None, :, 1, None] * res["dswa"]
    o, S = gdn(inp.q, inp.k, inp.v, inp.alpha, inp.beta, S0, variant=variant)
    res["S"] = S
    if "gdn" in branches:
        res["gdn"] = o
        total = total + g[None, None, :, 2, None] * o
    res["out"] = total
    return res


def attention_backward(kind: str, q, k, v, P: int, dilation: int, w: int, dO, centred: bool = False,
                       rope_base: float = 0.0):
    """Derivatives (dq, dk, dv) of ``attention`` given dO = dLoss/dO [B,L,H,d_v]
    (oracle_attention_backward in hlta_oracle.c).  float64 arrays."""
    lib = _load()
    q, dt = _tensor(q)
    k, _ = _tensor(k)
    v, _ = _tensor(v)
    B, L, H, dk_ = q.shape
    dv_ = v.shape[-1]
    dO = np.ascontiguousarray(dO, dtype=np.float64)
    assert dO.shape == (B, L, H, dv_)
    dq = np.empty((B, L, H, dk_))
    dk = np.empty((B, L, H, dk_))
    dv = np.empty((B, L, H, dv_))
    rc = lib.oracle_attention_backward({"swa": 0, "dswa": 1}[kind], int(centred), float(rope_base),
                                       B, L, H, dk_, dv_, P, dilation, w, q.ctypes.data, k.ctypes.data,
                                       v.ctypes.data, dt, _dptr(dO), _dptr(dq), _dptr(dk), _dptr(dv))
    if rc != 0:
        raise ValueError("oracle_attention_backward: bad arguments")
    return dq, dk, dv


def gdn_backward(q, k, v, alpha, beta, dO, S0=None, dS_final=None, variant: int = 0):
    """Derivatives of ``gdn`` given dO [B,L,H,d_v] and the gradient of the final
    state dS_final [B,H,d_v,d_k] (None: zero).  Returns a dict of float64 arrays
    dq, dk, dv, dalpha, dbeta, dS0 (oracle_gdn_backward in hlta_oracle.c)."""
    lib = _load()
    q, k, v, dt, ap, bp, S0, (B, L, H, dk_, dv_) = _gdn_common(q, k, v, alpha, beta, S0)
    dO = np.ascontiguousarray(dO, dtype=np.float64)
    assert dO.shape == (B, L, H, dv_)
    if dS_final is not None:
        dS_final = np.ascontiguousarray(dS_final, dtype=np.float64)
        assert dS_final.shape == (B, H, dv_, dk_)
    r = {"dq": np.empty((B, L, H, dk_)), "dk": np.empty((B, L, H, dk_)), "dv": np.empty((B, L, H, dv_)),
         "dalpha": np.empty((B, L, H)), "dbeta": np.empty((B, L, H)), "dS0": np.empty((B, H, dv_, dk_))}
    rc = lib.oracle_gdn_backward(B, L, H, dk_, dv_, q.ctypes.data, k.ctypes.data, v.ctypes.data, dt, ap,
                                 bp, _dptr(S0), _dptr(dO), _dptr(dS_final), _dptr(r["dq"]),
                                 _dptr(r["dk"]), _dptr(r["dv"]), _dptr(r["dalpha"]), _dptr(r["dbeta"]),
                                 _dptr(r["dS0"]), variant)
    if rc != 0:
        raise ValueError("oracle_gdn_backward: bad arguments")
    return r


def backward(inp, dout, S0=None, dS_final=None, branches=("swa", "dswa", "gdn"), variant=0,
             centred=False, rope_base=0.0):
    """Derivatives of the whole layer out = sum_b g[h, b] O_b given dout =
    dLoss/dout [B,L,H,d_v] and dS_final (gradient of the final memory state).

    Each branch receives dO_b = g[h, b] dout; dgates[h, b] = sum over batch,
    tokens and channels of dout * O_b.  Returns a dict of float64 arrays: dq,
    dk, dv, dalpha, dbeta (zero when the memory branch is not selected), dgates
    [H, 3] and dS0 (None when the memory branch is not selected).
    """
    wl = inp.wl
    dout = np.asarray(dout, dtype=np.float64)
    g = inp.gates.astype(np.float64)
    B, L, H = wl.B, wl.L, wl.H
    res = {"dq": np.zeros((B, L, H, wl.d_k)), "dk": np.zeros((B, L, H, wl.d_k)),
           "dv": np.zeros((B, L, H, wl.d_v)), "dalpha": np.zeros((B, L, H)),
           "dbeta": np.zeros((B, L, H)), "dgates": np.zeros((H, 3)), "dS0": None}
    kw = dict(centred=centred, rope_base=rope_base)
    for col, (name, dil, w) in enumerate((("swa", 1, wl.swa_window),
                                          ("dswa", wl.dilation, wl.dswa_window))):
        if name not in branches:
            continue
        o = attention(name, inp.q, inp.k, inp.v, wl.P, dil, w, **kw)
        res["dgates"][:, col] = np.einsum("blhc,blhc->h", dout, o)
        dq, dk, dv = attention_backward(name, inp.q, inp.k, inp.v, wl.P, dil, w,
                                        g[None, None, :, col, None] * dout, **kw)
        res["dq"] += dq
        res["dk"] += dk
        res["dv"] += dv
    if "gdn" in branches:
        o, _ = gdn(inp.q, inp.k, inp.v, inp.alpha, inp.beta, S0, variant=variant)
        res["dgates"][:, 2] = np.einsum("blhc,blhc->h", dout, o)
        r = gdn_backward(inp.q, inp.k, inp.v, inp.alpha, inp.beta, g[None, None, :, 2, None] * dout,
                         S0, dS_final, variant)
        for n in ("dq", "dk", "dv", "dalpha", "dbeta"):
            res[n] += r[n]
        res["dS0"] = r["dS0"]
    return res
