"""KV compression by softmax-gated pooling (oracle side).

[deep-read] "CSA：4× 压缩之后再 top-k", equation C_i^comp: entry i of a CSA
layer pools, channel by channel, the current block of m tokens (branch a,
tokens m*i .. m*(i+1)-1, values C^a, weights S^a) and the previous block
(branch b, tokens m*(i-1) .. m*i-1, values C^b, weights S^b); the weights
come from a per-channel softmax, so the window spans 2m tokens at stride m
and there are about n/m entries.  [notes] "CSA": the two windows overlap by
half.  [news] "一、CSA与HCA" and [summary] "Hybrid CSA + HCA Attention":
the pooling weights are a softmax gate with a learned position bias.
[deep-read] "HCA：128× 压缩后保留 dense 全局视野": HCA uses m' = 128 and no
overlap.  [deep-read] "其他稳定性细节": compressed KV is RMS-normalised, and
its last 64 dims carry RoPE.

Readings:
  R1  gate logits are Z + B[r] (Z a linear projection of the token, B the
      learned bias of window position r); ONE softmax per channel over all
      window positions, so branches a and b share the normalisation.
  R2  window tokens outside [0, L) are left out of the softmax (no zero
      padding); an incomplete last block still yields an entry, which is not
      visible to queries until the block completes (R3).
  R6  the indexer-key compressor has the same form with its own C, Z, B and
      no RMSNorm, no RoPE.
  RoPE position of entry i is m*i (the first token of its block).
"""
from __future__ import annotations

import numpy as np

from .rope import rmsnorm, rope


def window(i: np.ndarray, m: int, overlap: bool):
    """Token index [n, R] and window position [R] of every entry in ``i``."""
    i = np.asarray(i, dtype=np.int64)
    if overlap:
        r = np.arange(2 * m, dtype=np.int64)
        tok = m * (i[:, None] - 1) + r[None, :]
    else:
        r = np.arange(m, dtype=np.int64)
        tok = m * i[:, None] + r[None, :]
    return tok, r


def pool(entries, m: int, overlap: bool, L: int, Ca, Za, bias, Cb=None, Zb=None):
    """Softmax-gated pooled vectors e [n, c] for entry indices ``entries``.

    ``Ca, Za, Cb, Zb`` are callables tok[...] -> [..., c] (or arrays indexed by
    absolute token) giving the branch-a / branch-b values and gate logits.
    """
    def _g(A):
        if callable(A):
            return A
        arr = np.asarray(A, dtype=np.float64)
        return lambda t: arr[t]
    Ca, Za = _g(Ca), _g(Za)
    if overlap:
        Cb, Zb = _g(Cb), _g(Zb)
    tok, r = window(entries, m, overlap)
    present = (tok >= 0) & (tok < L)
    safe = np.where(present, tok, 0)
    if overlap:
        is_a = (r >= m)[None, :]
        vals = np.where(is_a[..., None], Ca(safe), Cb(safe))
        logit = np.where(is_a[..., None], Za(safe), Zb(safe))
    else:
        vals = Ca(safe)
        logit = Za(safe)
    logit = logit + np.asarray(bias, dtype=np.float64)[r][None, :, :]
    logit = np.where(present[..., None], logit, -np.inf)
    mx = np.max(logit, axis=1, keepdims=True)
    w = np.exp(logit - mx)
    w = w / np.sum(w, axis=1, keepdims=True)
    return np.sum(w * np.where(present[..., None], vals, 0.0), axis=1)


def finish_main(e, entries, m: int, d_rope: int, theta: float, eps: float = 1e-6,
                apply_rmsnorm: bool = True, apply_rope: bool = True):
    """Main-path post-processing: RMSNorm, then RoPE at position m*i."""
    out = rmsnorm(e, eps) if apply_rmsnorm else np.asarray(e, dtype=np.float64)
    if apply_rope:
        out = rope(out, m * np.asarray(entries, dtype=np.int64), d_rope, theta)
    return out


def n_entries(L: int, m: int) -> int:
    """Entries emitted for L tokens: ceil(L / m) (invariant I3)."""
    return -(-int(L) // int(m))


def n_visible(p, m: int):
    """R3: entry i is visible to the query at p iff m*(i+1)-1 <= p."""
    return (np.asarray(p, dtype=np.int64) + 1) // m
