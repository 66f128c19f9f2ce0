"""Whole-step compositions of the oracle stages for the five workloads.

A decode step for the query at position p of one sequence (call stacks of
[deep-read] "CSA：4× 压缩之后再 top-k" and "HCA：128× 压缩后保留 dense 全局视野",
with the state split of "异构 KV cache 与磁盘前缀复用"):
  1. the new token's raw compressor inputs join the uncompressed tail; its
     own KV (RMSNorm, RoPE at p, coded) joins the sliding window (R4);
  2. if (p+1) % m == 0 the block is complete and one entry (and, for CSA,
     one indexer key) is pooled from the tail and appended;
  3. CSA: indexer scores over the visible keys, then top-k;
  4. shared-KV MQA over the selected (CSA) or all visible (HCA) entries plus
     the window tokens, with the sink; the output's RoPE dims are rotated
     back by -p.

The decode histories are synthetic entries (``synth.decode_layer_inputs``)
that are only coded here, never pooled.
"""
from __future__ import annotations

import numpy as np

from . import codecs
from .compress import finish_main, n_visible, pool
from .indexer import scores as index_scores, topk
from .mqa import attend, finish_output, prepare_query, window_tokens
from .rope import rmsnorm, rope


def store_kv(v, ly):
    """Entry vectors -> (stored form, dequantised fp64 values)."""
    if ly.kv_fp8:
        codes, rbits, s = codecs.quantize_kv(v, ly.d_rope)
        return (codes, rbits, s), codecs.dequantize_kv(codes, rbits, s)
    v32 = codecs.f32(v)
    return (v32.astype(np.float32),), v32


def store_key(v, ly):
    """Indexer key / query vectors -> (stored form, dequantised fp64 values)."""
    if ly.idx_fp4:
        codes, sf = codecs.quantize_mxfp4(v)
        return (codecs.pack_e2m1(codes), sf), codecs.dequantize_mxfp4(codes, sf)
    v32 = codecs.f32(v)
    return (v32.astype(np.float32),), v32


def token_kv(C_t, t, ly, eps=1e-6):
    """R4: the window KV of raw token t (values C^a_t): RMSNorm, RoPE at t."""
    return rope(rmsnorm(C_t, eps), np.asarray(t), ly.d_rope, ly.rope_theta)


def decode_layer(inp: dict, ly, seqs, need_scores: bool = False) -> dict:
    """One decode step of one layer for the sequences ``seqs``."""
    p, ring, m = inp["p"], inp["ring"], ly.m
    t0 = p - ring + 1                      # token held in tail row 0
    complete = (p + 1) % m == 0
    i_new = (p + 1) // m - 1
    n_vis = int(n_visible(p, m))
    scale = 1.0 / np.sqrt(ly.d)
    out = {k: [] for k in ("entry_new", "entry_new_val", "key_new", "key_new_val", "swa_new",
                           "swa_new_val", "scores", "idx", "out", "lse")}
    for b in seqs:
        hist = inp["hist_entries"][b]
        n_hist = hist.shape[0]
        tail = lambda nm: (lambda t, arr=inp["tail_" + nm][b]: np.asarray(arr, np.float64)[t - t0])
        new_val = None
        if complete:
            if ly.kind == "csa":
                e = pool(np.array([i_new]), m, True, p + 1, tail("Ca"), tail("Za"), inp["bias"],
                         tail("Cb"), tail("Zb"))
            else:
                e = pool(np.array([i_new]), m, False, p + 1, tail("C"), tail("Z"), inp["bias"])
            e = finish_main(e, np.array([i_new]), m, ly.d_rope, ly.rope_theta)
            st, new_val = store_kv(e, ly)
            out["entry_new"].append(st)
            out["entry_new_val"].append(new_val[0])

        def entries(rows):
            """Stored (dequantised) entries for the given entry indices."""
            rows = np.asarray(rows, dtype=np.int64)
            old = rows[rows < n_hist]
            _, val = store_kv(hist[old], ly)
            res = np.empty((len(rows), ly.d))
            res[rows < n_hist] = val
            if np.any(rows >= n_hist):
                res[rows >= n_hist] = new_val[0]
            return res
        # window: synthetic history rows for tokens p-n_win+1 .. p-1, then token p
        ca_p = inp["tail_Ca" if ly.kind == "csa" else "tail_C"][b][ring - 1]
        st, swa_p = store_kv(token_kv(ca_p[None, :], np.array([p]), ly), ly)
        out["swa_new"].append(st)
        out["swa_new_val"].append(swa_p[0])
        toks = window_tokens(p, ly.n_win)
        hist_rows = toks[:-1] - (p - (ly.n_win - 1))
        _, swa_hist_val = store_kv(inp["swa_hist"][b][hist_rows], ly)
        swa_val = np.concatenate([swa_hist_val, swa_p], axis=0)
        if ly.kind == "csa":
            _, kval = store_key(inp["hist_keys"][b], ly)
            if complete:
                itail = lambda nm: (lambda t, arr=inp["itail_" + nm][b]: np.asarray(arr, np.float64)[t - t0])
                k = pool(np.array([i_new]), m, True, p + 1, itail("Ca"), itail("Za"), inp["ibias"],
                         itail("Cb"), itail("Zb"))
                kst, kv = store_key(k, ly)
                out["key_new"].append(kst)
                out["key_new_val"].append(kv[0])
                kval = np.concatenate([kval, kv], axis=0)
            _, qv = store_key(inp["qI"][b], ly)
            s = index_scores(qv, inp["w"][b], kval[:n_vis])
            idx = topk(s, n_vis, ly.top_k)
            out["scores"].append(s)
            out["idx"].append(idx)
            sel = entries(idx[idx >= 0])
        else:
            sel = entries(np.arange(n_vis))
        q = prepare_query(inp["Q"][b], p, ly.d_rope, ly.rope_theta, ly.kv_fp8)
        keys = np.concatenate([sel, swa_val], axis=0)
        o, lse = attend(q, keys, scale, inp["sink"])
        out["out"].append(finish_output(o, p, ly.d_rope, ly.rope_theta))
        out["lse"].append(lse)
    return out


def tiny_layer(inp: dict, w, query_rows=None) -> dict:
    """The tiny fp32 CSA layer: projections, pooling of every entry and key,
    window KV of every token, then the queries at ``inp['positions']``."""
    ly = w.layers[0]
    x = np.asarray(inp["x"], dtype=np.float64)
    C = x @ inp["W_kv"]
    Z = x @ inp["W_z"]
    CI = x @ inp["W_kvI"]
    ZI = x @ inp["W_zI"]
    L = w.L
    n_ent = -(-L // ly.m)
    ii = np.arange(n_ent)
    # R1: one W_kv / W_z serve both branches in this layer
    ents = finish_main(pool(ii, ly.m, True, L, C, Z, inp["bias"], C, Z), ii, ly.m, ly.d_rope,
                       ly.rope_theta)
    keys = pool(ii, ly.m, True, L, CI, ZI, inp["ibias"], CI, ZI)
    swa = token_kv(C, np.arange(L), ly)
    positions = inp["positions"] if query_rows is None else inp["positions"][query_rows]
    res = dict(entries=ents, keys=keys, swa=swa, scores=[], idx=[], out=[], lse=[], qI=[], w=[],
               Q=[])
    scale = 1.0 / np.sqrt(ly.d)
    for p in positions:
        xp = x[p]
        qI = ((xp @ inp["W_dq"]) @ inp["W_uq"]).reshape(ly.H_I, ly.d_I)
        wh = xp @ inp["W_w"]
        n_vis = int(n_visible(p, ly.m))
        s = index_scores(qI, wh, keys[:n_vis])
        idx = topk(s, n_vis, ly.top_k)
        Q = (xp @ inp["W_q"]).reshape(ly.H, ly.d)
        q = prepare_query(Q, p, ly.d_rope, ly.rope_theta, False, apply_rmsnorm=True)
        kk = np.concatenate([ents[idx[idx >= 0]], swa[window_tokens(int(p), ly.n_win)]], axis=0)
        o, lse = attend(q, kk, scale, inp["sink"])
        res["scores"].append(s)
        res["idx"].append(idx)
        res["out"].append(finish_output(o, p, ly.d_rope, ly.rope_theta))
        res["lse"].append(lse)
        res["qI"].append(qI)
        res["w"].append(wh)
        res["Q"].append(Q)
    return res
