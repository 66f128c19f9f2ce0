"""Lightning indexer scores and top-k selection (oracle side).

[deep-read] "CSA：4× 压缩之后再 top-k": the indexer compresses the history 4x
on its own, scores every compressed key with 64 indexer query heads through
a ReLU similarity, and sums the heads with input-dependent head weights;
Flash keeps 512 entries, Pro 1024 (model-spec table).  [summary] "Hybrid CSA
+ HCA Attention": low-rank query, ReLU score.  [deep-read] "FP4 QAT、可恢复
rollout 与百万 Token RL": the indexer QK path is MXFP4.

    s_i = sum_h w_h * max(0, q_h . k_i)        for every visible key i

Readings:
  R3   only keys of completed blocks are visible: i < floor((p+1)/m).
  R13  the k largest scores; exact ties go to the lower index; the result is
       listed in ascending index order and padded with -1 when fewer than k
       keys are visible.
"""
from __future__ import annotations

import numpy as np


def scores(qI, w, keys) -> np.ndarray:
    """qI [H_I, d_I], w [H_I], keys [n, d_I] (dequantised) -> s [n] (fp64)."""
    qI = np.asarray(qI, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    dots = keys @ qI.T                                   # [n, H_I]
    return np.maximum(dots, 0.0) @ np.asarray(w, dtype=np.float64)


def topk(s, n_vis: int, k: int) -> np.ndarray:
    """R13 selection over s[:n_vis] -> int64 [k], ascending, -1 padded."""
    s = np.asarray(s, dtype=np.float64)[: int(n_vis)]
    idx = np.arange(len(s), dtype=np.int64)
    order = np.lexsort((idx, -s))                        # by -s, then by index
    chosen = np.sort(order[: min(k, len(s))])
    out = np.full(k, -1, dtype=np.int64)
    out[: len(chosen)] = chosen
    return out
