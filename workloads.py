"""Seeded synthetic inputs for the Hybrid Linear Temporal Attention forward pass.

This module is shared by the fp64 oracle (``oracle/``), the CUDA path
(``hybrid_linear_temporal_b200``), the tests and ``bench.py``.  It holds the
workload shapes and the value distributions only -- none of the layer's
arithmetic -- so that both sides see bit-identical inputs without sharing any
code of the method itself.

Shapes follow the Kairos paper (arXiv 2606.16533), section 2.2.2: a latent
video of F frames with P tokens each is flattened to a causal sequence of
L = F * P tokens, token t = f * P + s.  The synthetic workloads stand in for
latent video; no dataset is involved.

Distributions (fp64 draws, cast once).  Every tensor is drawn in blocks of
4096 tokens per batch element, each block from its own generator
``default_rng(SeedSequence(seed, spawn_key=(tensor, b, block)))`` with tensor ids
q=0, k=1, v=2, beta=3, alpha=4, gates=5, so values do not depend on how many
threads generate them:

* q, k ~ N(0, 1), then L2-normalised per (token, head)
* v ~ N(0, 1)
* beta = sigmoid(N(0, 1))
* alpha = exp(-softplus(N(0, 1) + shift)), shift = 2 (4 for the long-horizon
  workload); ``alpha_mode="slow"`` is a stress variant with shift = -4
  (alpha ~ 0.98) that exercises long memory
* gates ~ U(0, 1) per head, three per head (SWA, DSWA, GDN)
* stress variant ``q_scale``: q is multiplied by q_scale after normalising,
  which sharpens the softmax (logit std ~ 0.0078 * q_scale at d = 128) while
  the keys stay unit, so the memory stays contractive

bf16 tensors are stored as ``uint16`` bit patterns (round-to-nearest-even of
the fp64 draw); ``as_float32`` gives their exact values.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os

import numpy as np

# Draw block: tensors are generated in independently seeded blocks of tokens,
# so the long workloads never hold fp64 copies of a whole tensor and blocks can
# be drawn in parallel.
_BLOCK_TOKENS = 4096
_TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "beta": 3, "alpha": 4, "gates": 5}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d_k: int
    d_v: int
    L: int                 # tokens per sequence (one-shot) or total (streaming)
    P: int                 # tokens per latent frame
    swa_window: int
    dswa_window: int
    dilation: int
    chunk: int = 64
    dtype: str = "bf16"    # "bf16" or "fp32"
    alpha_shift: float = 2.0
    stream_steps: int = 0  # >0: L tokens arrive in this many equal appends
    seed: int = 0

    @property
    def frames(self) -> int:
        return -(-self.L // self.P)

    @property
    def step_tokens(self) -> int:
        return self.L // self.stream_steps if self.stream_steps else self.L

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: tiny fp32 check, short bf16 clip, the 480P-shaped
# rollout (headline), streaming rollout and long horizon.
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", B=1, H=2, d_k=64, d_v=64, L=256, P=1,
                          swa_window=32, dswa_window=32, dilation=4, dtype="fp32"),
    "clip_4k": Workload("clip_4k", B=1, H=16, d_k=128, d_v=128, L=4096, P=256,
                        swa_window=256, dswa_window=256, dilation=4),
    "rollout_480p": Workload("rollout_480p", B=1, H=24, d_k=128, d_v=128, L=32760, P=1560,
                             swa_window=1560, dswa_window=1560, dilation=8),
    "stream_480p": Workload("stream_480p", B=4, H=24, d_k=128, d_v=128, L=120 * 1560, P=1560,
                            swa_window=1560, dswa_window=1560, dilation=8, stream_steps=120),
    "long_131k": Workload("long_131k", B=1, H=24, d_k=128, d_v=128, L=131040, P=1560,
                          swa_window=1560, dswa_window=3120, dilation=16, alpha_shift=4.0),
}
ORDER = ["tiny_fp32", "clip_4k", "rollout_480p", "stream_480p", "long_131k"]


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64/fp32 values to bf16 (nearest, ties to even); return uint16 bits.

    fp64 input is first rounded to fp32 (nearest), then fp32 to bf16."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + (0x7FFF + ((u >> 16) & 1))) >> 16).astype(np.uint16)


def bf16_to_float32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Inputs:
    """Host tensors of one workload.

    q, k: [B, L, H, d_k]; v: [B, L, H, d_v] -- uint16 bf16 bits or float32.
    alpha, beta: [B, L, H] float32.  gates: [H, 3] float32 (SWA, DSWA, GDN).
    """
    wl: Workload
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    alpha: np.ndarray
    beta: np.ndarray
    gates: np.ndarray

    def as_float32(self, name: str) -> np.ndarray:
        a = getattr(self, name)
        return bf16_to_float32(a) if a.dtype == np.uint16 else a


def _block_rng(seed, tensor, b, block):
    return np.random.default_rng(np.random.SeedSequence(seed, spawn_key=(_TENSOR_IDS[tensor], b, block)))


def _parallel(fn, jobs):
    workers = min(len(jobs), os.cpu_count() or 1, 16)
    if workers <= 1:
        for j in jobs:
            fn(*j)
        return
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        list(ex.map(lambda j: fn(*j), jobs))


def _normal_tensor(seed, name, B, L, H, d, normalise, dtype, scale=1.0):
    out = np.empty((B, L, H, d), dtype=np.uint16 if dtype == "bf16" else np.float32)

    def block(b, blk):
        t0 = blk * _BLOCK_TOKENS
        n = min(_BLOCK_TOKENS, L - t0)
        x = _block_rng(seed, name, b, blk).standard_normal((n, H, d))
        if normalise:
            x /= np.linalg.norm(x, axis=-1, keepdims=True)
        if scale != 1.0:
            x *= scale
        out[b, t0:t0 + n] = bf16_bits(x) if dtype == "bf16" else x.astype(np.float32)
    _parallel(block, [(b, blk) for b in range(B) for blk in range(-(-L // _BLOCK_TOKENS))])
    return out


def _scalar_tensor(seed, name, B, L, H, fn):
    out = np.empty((B, L, H), dtype=np.float32)
    for b in range(B):
        for blk in range(-(-L // _BLOCK_TOKENS)):
            t0 = blk * _BLOCK_TOKENS
            n = min(_BLOCK_TOKENS, L - t0)
            out[b, t0:t0 + n] = fn(_block_rng(seed, name, b, blk).standard_normal((n, H)))
    return out


def make_inputs(wl: Workload, seed: int | None = None, alpha_mode: str = "default",
                normalise_qk: bool = True, q_scale: float = 1.0) -> Inputs:
    """Draw the inputs of ``wl`` (see the module docstring for the recipe)."""
    seed = wl.seed if seed is None else seed
    B, L, H = wl.B, wl.L, wl.H
    q = _normal_tensor(seed, "q", B, L, H, wl.d_k, normalise_qk, wl.dtype, q_scale)
    k = _normal_tensor(seed, "k", B, L, H, wl.d_k, normalise_qk, wl.dtype)
    v = _normal_tensor(seed, "v", B, L, H, wl.d_v, False, wl.dtype)
    beta = _scalar_tensor(seed, "beta", B, L, H, lambda z: 1.0 / (1.0 + np.exp(-z)))
    shift = {"default": wl.alpha_shift, "slow": -4.0}[alpha_mode]
    alpha = _scalar_tensor(seed, "alpha", B, L, H, lambda z: np.exp(-np.logaddexp(0.0, z + shift)))
    gates = _block_rng(seed, "gates", 0, 0).uniform(0.0, 1.0, (H, 3)).astype(np.float32)
    return Inputs(wl, q, k, v, alpha, beta, gates)


def band_pairs(n: int, w: int) -> int:
    """Number of (query, key) pairs of a causal window of w keys over n tokens."""
    if n <= w:
        return n * (n + 1) // 2
    return w * (w + 1) // 2 + (n - w) * w


def dswa_pairs(L: int, P: int, w: int, dilation: int) -> int:
    """(query, key) pairs of the dilated window: a causal window of w keys over
    each residue class of frames (frames f = g, g + dilation, ...)."""
    F = -(-L // P)
    tot = 0
    for g in range(dilation):
        n = sum(min(P, L - f * P) for f in range(g, F, dilation))
        tot += band_pairs(n, w)
    return tot


def backward_work(wl: Workload) -> dict:
    """Flops and HBM bytes of one backward pass of ``wl`` (all three branches).

    Attention: 10 * d flops per in-band (query, key) pair (the logits again,
    dO.v, and the three products for dq, dk, dv).  Memory branch, chunk form per
    chunk of C tokens: 32*C^2*d + 22*C*d^2 + (2/3)*C^3 (the products of the
    per-chunk prep, the two state scans and the token gradients).
    Bytes: q, k, v, dout read, dq, dk, dv written, alpha, beta, dalpha, dbeta.
    """
    eb = 2 if wl.dtype == "bf16" else 4
    d = wl.d_k
    B, H, L, C = wl.B, wl.H, wl.L, wl.chunk
    swa = 10 * d * band_pairs(L, wl.swa_window) * B * H
    dswa = 10 * d * dswa_pairs(L, wl.P, wl.dswa_window, wl.dilation) * B * H
    nch = math.ceil(L / C)
    gdn = nch * (32 * C * C * d + 22 * C * d * d + (2 * C ** 3) // 3) * B * H
    bytes_ = B * L * H * (7 * d * eb + 16)
    return {"swa_flops": swa, "dswa_flops": dswa, "gdn_flops": gdn, "flops": swa + dswa + gdn,
            "bytes": bytes_}


def algorithmic_work(wl: Workload) -> dict:
    """Flops and HBM bytes the method needs for one forward pass of ``wl``.

    Attention: 4 * d flops per in-band (query, key) pair.  GDN: the chunk form,
    10*C^2*d + 6*C*d^2 + (2/3)*C^3 per chunk of C tokens (d = d_k = d_v).
    Bytes: q, k, v and out once, alpha and beta once.
    """
    eb = 2 if wl.dtype == "bf16" else 4
    d = wl.d_k
    B, H, L, C = wl.B, wl.H, wl.L, wl.chunk
    swa = 4 * d * band_pairs(L, wl.swa_window) * B * H
    dswa = 4 * d * dswa_pairs(L, wl.P, wl.dswa_window, wl.dilation) * B * H
    nch = math.ceil(L / C)
    gdn = nch * (10 * C * C * d + 6 * C * d * d + (2 * C ** 3) // 3) * B * H
    bytes_ = B * L * H * (3 * d * eb + wl.d_v * eb + 8)
    return {"swa_flops": swa, "dswa_flops": dswa, "gdn_flops": gdn,
            "flops": swa + dswa + gdn, "bytes": bytes_,
            "gdn_bytes": B * L * H * (3 * d * eb + wl.d_v * eb + 8)}
