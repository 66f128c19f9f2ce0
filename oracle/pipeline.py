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
    out = {k: [] for k in ("entry_new", "entry_new_val", "entry_new_raw", "key_new",
                           "key_new_val", "key_new_raw", "swa_new", "swa_new_val", "swa_new_raw",
                           "scores", "idx", "out", "lse")}
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
            out["entry_new_raw"].append(e[0])
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
        swa_raw = token_kv(ca_p[None, :], np.array([p]), ly)
        st, swa_p = store_kv(swa_raw, ly)
        out["swa_new_raw"].append(swa_raw[0])
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
                out["key_new_raw"].append(k[0])
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
               Q=[], q=[])
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
        res["q"].append(q)
    return res


PREFILL_COLS = ("Ca", "Cb", "Za", "Zb", "ICa", "ICb", "IZa", "IZb", "C", "Z")


def prefill_columns(csa, hca) -> dict:
    """Column range of each projected array in the prefill pair's projection
    output: the CSA main arrays (Ca, Cb, Za, Zb; d columns each), the CSA
    indexer arrays (ICa, ICb, IZa, IZb; d_I each), the HCA arrays (C, Z; d each)."""
    widths = [csa.d] * 4 + [csa.d_I] * 4 + [hca.d] * 2
    out, c0 = {}, 0
    for nm, wd in zip(PREFILL_COLS, widths):
        out[nm] = (c0, c0 + wd)
        c0 += wd
    return out


def prefill_pair(w, x, W, qin_csa: dict, qin_hca: dict, query_rows) -> dict:
    """Chunked prefill of a CSA + HCA layer pair ([deep-read] "CSA：4× 压缩之后再
    top-k", "HCA：128× 压缩后保留 dense 全局视野"): the raw tokens x [L, d_model]
    are projected by W into the compressor inputs of both layers; every
    complete entry / indexer key is pooled from them and every token's window
    KV is its own RMSNorm'd, RoPE'd C^a (R4); then each query at position
    prefix + row (rows ``query_rows``) runs the indexer + top-k + sparse MQA
    (CSA) and the dense MQA over all visible entries (HCA).  ``qin_csa`` /
    ``qin_hca`` hold the per-query inputs of those rows, in that order.

    Only the projections a query needs are formed: the indexer arrays and the
    HCA arrays of every token, the CSA main arrays of the selected entries'
    windows and of the window tokens.  Returns per-query lists plus, for every
    CSA key, CSA entry and HCA entry that was formed, its stored (dequantised)
    value and its value before coding."""
    csa, hca = w.layers
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    cols = prefill_columns(csa, hca)
    L = w.L
    proj_cache = {}

    def proj(nm, rows=None):
        """Projection of array ``nm`` for token rows (all tokens when None)."""
        c0, c1 = cols[nm]
        if rows is None:
            if nm not in proj_cache:
                proj_cache[nm] = x @ W[:, c0:c1]
            return proj_cache[nm]
        return x[np.asarray(rows)] @ W[:, c0:c1]

    def lookup(arr_rows, arr):
        """(token -> row) view of a projection restricted to some tokens."""
        pos = {int(t): i for i, t in enumerate(arr_rows)}
        return lambda t: arr[np.vectorize(pos.__getitem__)(t)]

    scale_c, scale_h = 1.0 / np.sqrt(csa.d), 1.0 / np.sqrt(hca.d)
    # CSA indexer keys of every complete entry
    n_csa = L // csa.m
    ii = np.arange(n_csa)
    keys = pool(ii, csa.m, True, L, proj("ICa"), proj("IZa"), qin_csa["ibias"],
                proj("ICb"), proj("IZb"))
    _, key_val = store_key(keys, csa)
    # HCA entries of every complete block
    n_hca = L // hca.m
    jj = np.arange(n_hca)
    hca_ent = finish_main(pool(jj, hca.m, False, L, proj("C"), proj("Z"), qin_hca["bias"]),
                          jj, hca.m, hca.d_rope, hca.rope_theta)
    _, hca_val = store_kv(hca_ent, hca)
    out = {"hca_raw": hca_ent, "csa_raw": {}, "detail": []}
    out.update({k: [] for k in ("positions", "scores", "idx", "csa_out", "csa_lse", "hca_out",
                           "hca_lse", "csa_entries")})
    out["key_val"] = key_val
    out["key_raw"] = keys
    out["hca_val"] = hca_val
    csa_cache = {}
    for r, row in enumerate(query_rows):
        p = w.prefix + int(row)
        out["positions"].append(p)
        # ---- CSA: indexer, top-k, sparse MQA
        nv = int(n_visible(p, csa.m))
        _, qv = store_key(np.asarray(qin_csa["qI"][r], dtype=np.float64), csa)
        s = index_scores(qv, qin_csa["w"][r], key_val[:nv])
        idx = topk(s, nv, csa.top_k)
        sel = idx[idx >= 0]
        need = [i for i in sel.tolist() if i not in csa_cache]
        if need:
            need = np.asarray(need)
            toks = np.unique(np.concatenate([np.arange(csa.m * (i - 1), csa.m * (i + 1))
                                             for i in need]))
            toks = toks[(toks >= 0) & (toks < L)]
            arrs = {nm: lookup(toks, proj(nm, toks)) for nm in ("Ca", "Za", "Cb", "Zb")}
            e = finish_main(pool(need, csa.m, True, L, arrs["Ca"], arrs["Za"], qin_csa["bias"],
                                 arrs["Cb"], arrs["Zb"]), need, csa.m, csa.d_rope, csa.rope_theta)
            _, ev = store_kv(e, csa)
            for i, v, raw in zip(need.tolist(), ev, e):
                csa_cache[i] = v
                out["csa_raw"][i] = raw
        wt = window_tokens(p, csa.n_win)
        _, swa_c = store_kv(token_kv(proj("Ca", wt), wt, csa), csa)
        keys_c = np.concatenate([np.stack([csa_cache[i] for i in sel.tolist()])
                                 if len(sel) else np.zeros((0, csa.d)), swa_c], axis=0)
        q = prepare_query(qin_csa["Q"][r], p, csa.d_rope, csa.rope_theta, csa.kv_fp8)
        o, lse, a_c, _ = attend(q, keys_c, scale_c, qin_csa["sink"], return_weights=True)
        det = dict(csa_sel=sel, csa_win=wt, csa_keys=keys_c, csa_q=q, csa_a=a_c, csa_o=o)
        out["scores"].append(s)
        out["idx"].append(idx)
        out["csa_out"].append(finish_output(o, p, csa.d_rope, csa.rope_theta))
        out["csa_lse"].append(lse)
        # ---- HCA: dense MQA over the visible entries + window
        nvh = int(n_visible(p, hca.m))
        wt = window_tokens(p, hca.n_win)
        _, swa_h = store_kv(token_kv(proj("C", wt), wt, hca), hca)
        keys_h = np.concatenate([hca_val[:nvh], swa_h], axis=0)
        qh = prepare_query(qin_hca["Q"][r], p, hca.d_rope, hca.rope_theta, hca.kv_fp8)
        o, lse, a_h, _ = attend(qh, keys_h, scale_h, qin_hca["sink"], return_weights=True)
        det.update(hca_n=nvh, hca_win=wt, hca_keys=keys_h, hca_q=qh, hca_a=a_h, hca_o=o)
        out["detail"].append(det)
        out["hca_out"].append(finish_output(o, p, hca.d_rope, hca.rope_theta))
        out["hca_lse"].append(lse)
    out["csa_entries"] = csa_cache
    return out
