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
