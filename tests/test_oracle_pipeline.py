"""Pins of the oracle's whole-step compositions: causality (a query never
depends on later tokens), batch independence, and the decode-state
bookkeeping (the tail ring and window history address the right tokens)."""
import dataclasses

import numpy as np

import synth
from oracle import codecs, compress, pipeline


def _tiny(L=300, nq=6):
    w = synth.scaled(synth.WORKLOADS["tiny_csa_fp32"], L=L, n_queries=nq, name="tiny_small")
    return w, synth.tiny_inputs(w)


def test_tiny_layer_is_causal():
    w, inp = _tiny()
    base = pipeline.tiny_layer(inp, w)
    p_first = int(inp["positions"][0])
    inp2 = dict(inp)
    x = inp["x"].copy()
    x[p_first + 1:] += 5.0 * np.random.default_rng(0).standard_normal(x[p_first + 1:].shape)
    inp2["x"] = x
    alt = pipeline.tiny_layer(inp2, w)
    assert np.allclose(base["out"][0], alt["out"][0], atol=1e-12)
    assert np.array_equal(base["idx"][0], alt["idx"][0])
    assert not np.allclose(base["out"][-1], alt["out"][-1])


def test_tiny_layer_shapes_and_selection():
    w, inp = _tiny()
    ly = w.layers[0]
    r = pipeline.tiny_layer(inp, w)
    assert r["entries"].shape == (compress.n_entries(w.L, 4), ly.d)
    for p, s, idx in zip(inp["positions"], r["scores"], r["idx"]):
        nv = int(compress.n_visible(p, 4))
        assert len(s) == nv and len(idx) == ly.top_k
        sel = idx[idx >= 0]
        assert np.all(np.diff(sel) > 0) and np.all(sel < nv)
        kth = np.sort(s)[::-1][min(ly.top_k, nv) - 1]
        assert np.all(s[sel] >= kth)


def _decode(kind, L, B=2):
    base = synth.WORKLOADS["csa_flash_128k" if kind == "csa" else "hca_flash_128k"]
    w = synth.scaled(base, B=B, L=L, top_k=16, name="small")
    return w, synth.decode_layer_inputs(w, 0)


def test_decode_tail_ring_addresses_the_right_tokens():
    for kind, L in (("csa", 4 * 50), ("hca", 128 * 3)):
        w, inp = _decode(kind, L)
        ly = w.layers[0]
        p, ring = inp["p"], inp["ring"]
        r = pipeline.decode_layer(inp, ly, [1])
        i_new = (p + 1) // ly.m - 1
        # rebuild the entry from full-length token arrays placed at absolute positions
        full = {}
        for nm in (["Ca", "Za", "Cb", "Zb"] if kind == "csa" else ["C", "Z"]):
            arr = np.zeros((p + 1, ly.d))
            arr[p - ring + 1:] = inp["tail_" + nm][1]
            full[nm] = arr
        if kind == "csa":
            e = compress.pool(np.array([i_new]), 4, True, p + 1, full["Ca"], full["Za"], inp["bias"],
                              full["Cb"], full["Zb"])
        else:
            e = compress.pool(np.array([i_new]), 128, False, p + 1, full["C"], full["Z"], inp["bias"])
        e = compress.finish_main(e, np.array([i_new]), ly.m, ly.d_rope, ly.rope_theta)
        _, val = pipeline.store_kv(e, ly)
        assert np.array_equal(val[0], r["entry_new_val"][0])


def test_decode_batch_independence():
    w, inp = _decode("csa", 4 * 40, B=3)
    ly = w.layers[0]
    r_all = pipeline.decode_layer(inp, ly, [0, 1, 2])
    inp2 = dict(inp)
    for key in ("hist_entries", "hist_keys", "Q", "qI"):
        arr = inp[key].copy()
        arr[0] = -arr[0]
        inp2[key] = arr
    r_alt = pipeline.decode_layer(inp2, ly, [0, 1, 2])
    for b in (1, 2):
        assert np.array_equal(r_all["out"][b], r_alt["out"][b])
        assert np.array_equal(r_all["idx"][b], r_alt["idx"][b])


def test_decode_window_holds_own_token():
    """R4: the query's own token is in its window: with every other key driven
    out by a huge negative score, the output is that token's KV."""
    w, inp = _decode("hca", 128 * 2, B=1)
    ly = dataclasses.replace(w.layers[0], n_win=1)
    inp = dict(inp)
    inp["sink"] = np.full(ly.H, -1e9)
    r = pipeline.decode_layer(inp, ly, [0])
    p = inp["p"]
    # with n_win = 1 the window is exactly token p; compare against an
    # attention over the entries plus that single token
    kv = pipeline.token_kv(inp["tail_C"][0][-1][None, :], np.array([p]), ly)
    _, kv_val = pipeline.store_kv(kv, ly)
    assert np.allclose(kv_val[0], r["swa_new_val"][0])


def test_tiny_layer_query_construction_closed_form():
    """The low-rank indexer query x_p W_dq W_uq reshaped to [H_I, d_I] (head
    major), the head weights x_p W_w and the MQA query x_p W_q reshaped to
    [H, d], pinned with one-hot weights: with x_p = e_0, W_dq = e_0 -> e_j,
    W_uq = e_j -> e_(h0*d_I + c0), W_w = 0.75 e_0 -> e_h0 and
    W_q = e_0 -> e_(h1*d + c1), the indexer query is the one-hot at (h0, c0),
    the scores are 0.75 * max(0, k_i[c0]) for every visible key, and the MQA
    query before RMSNorm is the one-hot at (h1, c1) (after RMSNorm,
    1/sqrt(1/d + eps) there; RoPE leaves a non-RoPE dim alone).  A transposed reshape or a
    swapped head / dim order lands the one-hot elsewhere."""
    w, inp = _tiny(L=200, nq=3)
    ly = w.layers[0]
    r, h0, c0, h1, c1 = 5, 2, 11, 9, 17
    assert c1 < ly.d - ly.d_rope
    inp = dict(inp)
    x = inp["x"].copy()
    for p in inp["positions"]:
        x[p] = 0.0
        x[p, 0] = 1.0
    inp["x"] = x
    W_dq = np.zeros_like(inp["W_dq"])
    W_dq[0, r] = 1.0
    W_uq = np.zeros_like(inp["W_uq"])
    W_uq[r, h0 * ly.d_I + c0] = 1.0
    W_w = np.zeros_like(inp["W_w"])
    W_w[0, h0] = 0.75
    W_q = np.zeros_like(inp["W_q"])
    W_q[0, h1 * ly.d + c1] = 1.0
    inp.update(W_dq=W_dq, W_uq=W_uq, W_w=W_w, W_q=W_q)
    res = pipeline.tiny_layer(inp, w)
    for n, p in enumerate(inp["positions"]):
        want_q = np.zeros((ly.H_I, ly.d_I))
        want_q[h0, c0] = 1.0
        assert np.array_equal(res["qI"][n], want_q)
        want_w = np.zeros(ly.H_I)
        want_w[h0] = 0.75
        assert np.allclose(res["w"][n], want_w, rtol=0, atol=1e-15)
        nv = int(compress.n_visible(p, ly.m))
        assert np.allclose(res["scores"][n], 0.75 * np.maximum(res["keys"][:nv, c0], 0.0),
                           rtol=0, atol=1e-12)
        want_Q = np.zeros((ly.H, ly.d))
        want_Q[h1, c1] = 1.0
        assert np.array_equal(res["Q"][n], want_Q)
        q = res["q"][n]
        assert abs(q[h1, c1] - 1.0 / np.sqrt(1.0 / ly.d + 1e-6)) < 1e-12     # RMSNorm, eps 1e-6
        assert np.count_nonzero(np.abs(q) > 1e-9) == 1
