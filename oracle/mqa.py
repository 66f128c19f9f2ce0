"""Shared-KV multi-query attention with a sliding window and a sink (oracle).

[deep-read] model-spec table: 64 (Flash) / 128 (Pro) query heads of dim 512
over ONE shared KV head.  [deep-read] "CSA 与 HCA": one 512-dim compressed
entry serves as both key and value for every query head; the last 128 raw
tokens are attended uncompressed.  [deep-read] "其他稳定性细节": a learnable
per-head sink lets the weights sum to less than one, and the output's RoPE
dims are rotated back by the query position.  [notes] "细节": the sink adds
exp(z'_h) to each head's softmax denominator.

For query head h with prepared query q_h and key set {k_j}:
    s_hj = scale * q_h . k_j
    a_hj = exp(s_hj) / (exp(z_h) + sum_l exp(s_hl))
    o_h  = R(-p) applied to the RoPE dims of  sum_j a_hj k_j      (V == K)

Readings:
  R4  the window is tokens max(0, p-n_win+1) .. p (the query's own token
      included); a token's KV is RMSNorm(C^a_t) with RoPE at t, stored in the
      entry format; window tokens are not de-duplicated against entries.
  R5  scale = 1/sqrt(d).
  R7  the output rotation is R(-p) on the last d_rope dims.
  R10 with the FP8 KV format the query's 448 non-RoPE dims are coded E4M3
      with one power-of-two scale per (query, head) and its RoPE dims bf16;
      both sides attend with the coded query.
"""
from __future__ import annotations

import numpy as np

from . import codecs
from .rope import rmsnorm, rope


def prepare_query(Q, p, d_rope: int, theta: float, fp8: bool, apply_rmsnorm: bool = False,
                  eps: float = 1e-6) -> np.ndarray:
    """Q [H, d] -> the query the scores use: [RMSNorm], RoPE at p, [R10 coding]."""
    q = rmsnorm(Q, eps) if apply_rmsnorm else np.asarray(Q, dtype=np.float64)
    q = rope(q, np.full(q.shape[0], p), d_rope, theta)
    if fp8:
        codes, rbits, s = codecs.quantize_kv(q, d_rope)
        q = codecs.dequantize_kv(codes, rbits, s)
    return q


def attend(q, keys, scale: float, sink=None, return_weights: bool = False):
    """q [H, d], keys [n, d] (V == K), sink [H] or None -> (o [H, d], lse [H])."""
    q = np.asarray(q, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    s = scale * (q @ keys.T)                                     # [H, n]
    terms = [s]
    if sink is not None:
        terms.append(np.asarray(sink, dtype=np.float64)[:, None])
    allv = np.concatenate(terms, axis=1)
    mx = np.max(allv, axis=1, keepdims=True)
    mx = np.where(np.isfinite(mx), mx, 0.0)
    den = np.sum(np.exp(allv - mx), axis=1, keepdims=True)      # includes the sink
    a = np.exp(s - mx) / den
    o = a @ keys
    lse = (np.log(den) + mx)[:, 0]
    if return_weights:
        sink_share = 1.0 - np.sum(a, axis=1)
        return o, lse, a, sink_share
    return o, lse


def finish_output(o, p, d_rope: int, theta: float) -> np.ndarray:
    """R7: rotate the RoPE dims of o back by the query position."""
    o = np.asarray(o, dtype=np.float64)
    return rope(o, np.full(o.shape[0], p), d_rope, theta, sign=-1.0)


def window_tokens(p: int, n_win: int) -> np.ndarray:
    """R4: raw tokens attended by the query at p."""
    return np.arange(max(0, p - n_win + 1), p + 1, dtype=np.int64)
