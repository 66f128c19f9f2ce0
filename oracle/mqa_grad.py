"""Backward of the shared-KV MQA (oracle; TEST INFRASTRUCTURE ONLY, see the
package header: only tests/, smoke() and bench.py's CPU legs may use it).

[deep-read] "Deterministic backward": the sparse attention's backward gives
every SM its own gradient buffer and sums the buffers in a fixed order, so
that the entry gradients (an entry is read by every query that selects it)
do not depend on the order of atomic additions.  This module states what that
backward computes, in fp64, from the forward of ``oracle.mqa.attend``:

    s_hj = scale * q_h . k_j,   a_hj = exp(s_hj) / (exp(z_h) + sum_l exp(s_hl)),
    o_h  = sum_j a_hj k_j                                   (V == K)

Given dO = dL/do (before the output's inverse RoPE, which is a rotation; its
backward rotates dO forward by the query position):

    dA_hj = dO_h . k_j
    D_h   = sum_j a_hj dA_hj = dO_h . o_h
    dS_hj = a_hj (dA_hj - D_h)                  (softmax with the sink as one
    dz_h  = -(1 - sum_j a_hj) D_h                 more logit carrying no value)
    dq_h  = scale * sum_j dS_hj k_j
    dk_j  = scale * sum_h dS_hj q_h  +  sum_h a_hj dO_h   (key path + value path)

Readings (the pages give the determinism requirement, not these formulas; the
formulas are the chain rule of the forward above): the differentiable inputs
are the prepared query (after RMSNorm, RoPE and coding) and the stored rows
as the forward reads them (the coding's own gradient, e.g. a straight-through
estimator in quantisation-aware training, is outside this backward); the
entry gradients of a batch are summed over its queries in query order.
"""
from __future__ import annotations

import numpy as np

from .mqa import attend
from .rope import rope


def attend_backward(q, keys, scale: float, dO, sink=None):
    """Gradients of ``attend``: q [H, d], keys [n, d], dO [H, d], sink [H] or
    None -> (dq [H, d], dkeys [n, d], dsink [H] or None, dS [H, n])."""
    q = np.asarray(q, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    o, _, a, sink_share = attend(q, keys, scale, sink, return_weights=True)
    dA = dO @ keys.T                                    # [H, n]
    D = np.sum(dO * o, axis=1, keepdims=True)           # [H, 1]
    dS = a * (dA - D)
    dq = scale * (dS @ keys)
    dkeys = scale * (dS.T @ q) + a.T @ dO
    dsink = None if sink is None else -sink_share * D[:, 0]
    return dq, dkeys, dsink, dS


def output_rotation_backward(dO_out, p, d_rope: int, theta: float) -> np.ndarray:
    """dL/do from dL/d(output): the output is R(-p) o on the RoPE dims, whose
    transpose is R(+p)."""
    return rope(np.asarray(dO_out, dtype=np.float64), np.full(len(dO_out), p), d_rope, theta)


def sparse_backward(qs, sel, entries, window_rows, scale: float, dOs, sink=None):
    """Backward of a batch of sparse MQA queries over one cache.

    qs [nq, H, d] prepared queries; sel: per query the entry indices it
    attends (-1 skipped); entries [N, d]; window_rows: per query its window
    rows [w, d]; dOs [nq, H, d].  Returns (dq [nq, H, d], dentries [N, d]
    summed over the queries in query order, dwindow: per query [w, d],
    dsink [H] summed over the queries or None)."""
    entries = np.asarray(entries, dtype=np.float64)
    nq = len(qs)
    dq = np.zeros((nq,) + np.shape(qs[0]), dtype=np.float64)
    dent = np.zeros_like(entries)
    dwin = []
    dsink = None if sink is None else np.zeros(len(sink), dtype=np.float64)
    for i in range(nq):
        rows = np.asarray(sel[i], dtype=np.int64)
        rows = rows[rows >= 0]
        win = np.asarray(window_rows[i], dtype=np.float64).reshape(-1, entries.shape[1])
        keys = np.concatenate([entries[rows], win], 0)
        dqi, dk, dz, _ = attend_backward(qs[i], keys, scale, dOs[i], sink)
        dq[i] = dqi
        np.add.at(dent, rows, dk[: len(rows)])
        dwin.append(dk[len(rows):])
        if dsink is not None:
            dsink += dz
    return dq, dent, dwin, dsink
