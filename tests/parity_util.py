"""Helpers shared by the GPU parity tests: upload seeded inputs, run the CUDA
library through its C ABI, and compute oracle rows for comparison."""
from __future__ import annotations

import numpy as np

import oracle
from workloads import Inputs, bf16_to_float32

# Tolerances (the specification's): bf16 max-abs <= 2e-2 and relative L2 <= 5e-3;
# fp32 relative L2 <= 1e-4.
TOL = {"bf16": {"max_abs": 2e-2, "rel_l2": 5e-3}, "fp32": {"max_abs": None, "rel_l2": 1e-4}}


def to_device(inp: Inputs):
    import torch
    dev = "cuda"

    def t(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(a).to(dev)
    return {n: t(getattr(inp, n)) for n in ("q", "k", "v", "alpha", "beta", "gates")}


def to_numpy64(t):
    import torch
    if t.dtype == torch.bfloat16:
        return bf16_to_float32(t.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


def run_gpu(layer, dev_inputs, S0=None, want_state=False, branches=7):
    import torch
    c = layer.cfg
    S_out = torch.empty((c.B, c.H, c.d_v, c.d_k), dtype=torch.float32, device="cuda") if want_state else None
    out = layer.forward(dev_inputs["q"], dev_inputs["k"], dev_inputs["v"], dev_inputs["alpha"],
                        dev_inputs["beta"], dev_inputs["gates"], S0=S0, S_out=S_out, branches=branches)
    torch.cuda.synchronize()
    return out, S_out


def sample_rows(wl, n: int, seed: int = 0) -> np.ndarray:
    """Row ids (b*L + t)*H + h: the first and last tokens, tokens around frame
    boundaries and window edges, and n random rows."""
    rng = np.random.default_rng(seed)
    L, H, B, P = wl.L, wl.H, wl.B, wl.P
    ts = set(range(min(L, 3))) | set(range(max(0, L - 3), L))
    for f in (1, 2, wl.dilation - 1, wl.dilation, wl.dilation + 1, wl.frames - 1):
        for off in (-1, 0, 1, P // 2):
            t = f * P + off
            if 0 <= t < L:
                ts.add(t)
    for w in (wl.swa_window, wl.dswa_window, 64, 128):
        for off in (-1, 0, 1):
            if 0 <= w + off < L:
                ts.add(w + off)
    rows = [(b * L + t) * H + h for t in sorted(ts) for b in range(B) for h in (0, H - 1)]
    rows += list(rng.integers(0, B * L * H, size=n))
    return np.unique(np.array(rows, dtype=np.int64))


def oracle_rows(inp: Inputs, rows, gdn_out=None, branches=("swa", "dswa", "gdn"), centred=False,
                rope_base=0.0):
    """Oracle layer output at the given rows ([n, d_v] float64).  gdn_out: a full
    oracle GDN output [B,L,H,d_v] (computed when None and GDN is selected).
    centred / rope_base select the centred attention window and the rotary
    embedding of the attention branches."""
    wl = inp.wl
    g = inp.gates.astype(np.float64)
    h = rows % wl.H
    res = np.zeros((rows.size, wl.d_v))
    kw = dict(centred=centred, rope_base=rope_base)
    if "swa" in branches:
        res += g[h, 0, None] * oracle.attention_rows("swa", inp.q, inp.k, inp.v, wl.P, 1,
                                                     wl.swa_window, rows, **kw)
    if "dswa" in branches:
        res += g[h, 1, None] * oracle.attention_rows("dswa", inp.q, inp.k, inp.v, wl.P,
                                                     wl.dilation, wl.dswa_window, rows, **kw)
    if "gdn" in branches:
        if gdn_out is None:
            gdn_out, _ = oracle.gdn(inp.q, inp.k, inp.v, inp.alpha, inp.beta)
        res += g[h, 2, None] * gdn_out.reshape(-1, wl.d_v)[rows]
    return res


def errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = got - ref
    return {"max_abs": float(np.abs(diff).max()) if diff.size else 0.0,
            "rel_l2": float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))}


def assert_close(got, ref, dtype, what=""):
    e = errors(got, ref)
    tol = TOL[dtype]
    msg = f"{what}: {e} vs tolerance {tol}"
    assert e["rel_l2"] <= tol["rel_l2"], msg
    if tol["max_abs"] is not None:
        assert e["max_abs"] <= tol["max_abs"], msg
    return e
