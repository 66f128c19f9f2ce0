"""RMSNorm and partial RoPE (oracle side).

[deep-read] "其他稳定性细节": queries and compressed KV are RMS-normalised before
the main attention; only the last 64 dims carry RoPE, and the attention
output is rotated back by the query position.  [notes] "细节": every query
head and the shared KV are RMS-normalised separately; RoPE is on the last 64
of 512 dims.  The model-spec table gives RoPE theta 160000 for the
compressed branch.

R11 (reading): RoFormer pairing of adjacent dims (2i, 2i+1) inside the RoPE
slice, frequency theta^(-2i/d_rope), the same theta for queries, SWA tokens
and compressed entries, no YaRN rescaling.
"""
from __future__ import annotations

import numpy as np


def rmsnorm(x, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) over the last axis (unit weight)."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def inv_freq(d_rope: int, theta: float) -> np.ndarray:
    return theta ** (-np.arange(0, d_rope, 2, dtype=np.float64) / d_rope)


def rope(x, pos, d_rope: int, theta: float, sign: float = 1.0) -> np.ndarray:
    """Rotate the last ``d_rope`` dims of x [..., d] by angle sign*pos*freq_i
    on adjacent pairs; ``pos`` broadcasts against x's leading axes."""
    x = np.array(x, dtype=np.float64, copy=True)
    if d_rope == 0:
        return x
    d = x.shape[-1]
    pos = np.asarray(pos, dtype=np.float64)
    ang = sign * pos[..., None] * inv_freq(d_rope, theta)      # [..., d_rope/2]
    c, s = np.cos(ang), np.sin(ang)
    x0 = x[..., d - d_rope::2].copy()
    x1 = x[..., d - d_rope + 1::2].copy()
    x[..., d - d_rope::2] = x0 * c - x1 * s
    x[..., d - d_rope + 1::2] = x0 * s + x1 * c
    return x
