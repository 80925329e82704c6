"""e4m3 quantization model for the FP8 attention logits (test infrastructure only).

The OCP 8-bit floating-point format E4M3: 4 exponent bits (bias 7), 3 mantissa
bits, subnormals down to 2^-9, largest finite value 448 = 1.75 * 2^8.  Rounding
is to nearest, ties to even, and out-of-range values saturate to +-448.

``quantize_tiles`` is the per-tile scaling the FP8 path reads as the pages'
"FP8 attention quantization": one scale per 128-row tile of a head inside a
segment (the whole sequence for SWA, one frame for DSWA), scale = max|x| / 448.
The scale and the scaled value are formed in float32 (scale = amax / 448,
y = x * (1 / scale)), so that the e4m3 codes are decided in the same precision
the GPU uses.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_round(y) -> np.ndarray:
    """Nearest e4m3 value of each element (ties to even, saturating), float64."""
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), E4M3_MAX)
    # exponent of the binade; below 2^-6 the spacing stays 2^-9 (subnormals)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    quantum = np.exp2(e - 3.0)
    return np.sign(y) * np.minimum(np.round(a / quantum) * quantum, E4M3_MAX)


def quantize_tiles(x: np.ndarray, Pseg: int, rows: int = 128):
    """x: [B, L, H, d] float32 (L a multiple of Pseg).  Returns (codes * scale as
    float32 [B, L, H, d], scales [B * L / Pseg, H, ceil(Pseg / rows)] float32)."""
    x = np.asarray(x, dtype=np.float32)
    B, L, H, d = x.shape
    segs = L // Pseg
    nblk = -(-Pseg // rows)
    out = np.empty_like(x)
    scales = np.empty((B * segs, H, nblk), dtype=np.float32)
    for b in range(B):
        for s in range(segs):
            for blk in range(nblk):
                t0 = s * Pseg + blk * rows
                t1 = min(t0 + rows, (s + 1) * Pseg)
                for h in range(H):
                    tile = x[b, t0:t1, h]
                    amax = np.float32(np.abs(tile).max())
                    scale = amax / np.float32(E4M3_MAX) if amax > 0 else np.float32(1.0)
                    inv = np.float32(1.0) / scale
                    codes = e4m3_round((tile * inv).astype(np.float32))
                    out[b, t0:t1, h] = (codes * np.float64(scale)).astype(np.float32)
                    scales[b * segs + s, h, blk] = scale
    return out, scales
