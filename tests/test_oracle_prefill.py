"""CPU checks of the prefill composition: the projections it forms on demand
for a subset of tokens agree with the full projection, and its pieces fit
together (causal key counts, ascending selections, window sizes)."""
import numpy as np

import synth
from oracle.compress import finish_main, pool
from oracle.pipeline import PREFILL_COLS, prefill_columns, prefill_pair, store_kv

W_TINY = synth.scaled(synth.WORKLOADS["flash_prefill_64k"], L=700, n_queries=300, prefix=400,
                      top_k=32, H=4, name="prefill_tiny")


def _tiny():
    w = W_TINY
    x = synth.prefill_x(w)[:, :64]
    W = synth.prefill_weight(w)[:64]
    return w, x, W


def test_columns_tile_the_projection():
    csa, hca = synth.WORKLOADS["flash_prefill_64k"].layers
    cols = prefill_columns(csa, hca)
    assert list(cols) == list(PREFILL_COLS)
    spans = sorted(cols.values())
    assert spans[0][0] == 0
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] == 4 * csa.d + 4 * csa.d_I + 2 * hca.d


def test_on_demand_projection_matches_full():
    w, x, W = _tiny()
    csa, hca = w.layers
    rows = [0, 5, 299]
    q0 = synth.prefill_queries(w, 0, rows=rows)
    q1 = synth.prefill_queries(w, 1, rows=rows)
    ref = prefill_pair(w, x, W, q0, q1, rows)
    cols = prefill_columns(csa, hca)
    full = {nm: x.astype(np.float64) @ W[:, c0:c1].astype(np.float64) for nm, (c0, c1) in cols.items()}
    for i, got in ref["csa_entries"].items():
        e = finish_main(pool(np.array([i]), csa.m, True, w.L, full["Ca"], full["Za"], q0["bias"],
                             full["Cb"], full["Zb"]), np.array([i]), csa.m, csa.d_rope, csa.rope_theta)
        _, want = store_kv(e, csa)
        assert np.array_equal(got, want[0]), i
    for n, r in enumerate(rows):
        p = w.prefix + r
        nv = (p + 1) // csa.m
        sel = ref["idx"][n]
        kk = min(csa.top_k, nv)
        assert len(ref["scores"][n]) == nv
        assert np.all(np.diff(sel[:kk]) > 0) and np.all(sel[kk:] == -1)
        assert np.all(np.isfinite(ref["csa_out"][n])) and np.all(np.isfinite(ref["hca_out"][n]))
    assert len(ref["hca_val"]) == w.L // hca.m and len(ref["key_val"]) == w.L // csa.m
