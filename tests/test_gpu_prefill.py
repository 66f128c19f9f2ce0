"""Chunked prefill of the V4-Flash CSA + HCA pair through the C-ABI, against
``oracle.pipeline.prefill_pair`` (the config of 65536 new tokens on a 65536
prefix, scaled so that the oracle finishes in seconds: L = 4000 tokens, 2000
new on a 2000 prefix, d_model 4096; the scale keeps ragged key tiles, a
partial HCA block and more than one internal query chunk).

Every step runs in the library: the projection of the raw tokens, the pooling
of every entry and indexer key, the window KV of every token, the indexer +
top-k of every query, the sparse (CSA) and dense (HCA) MQA of every query.
Sampled queries, entries and keys are compared with the oracle."""
import numpy as np
import pytest
import torch

import synth
from oracle import codecs
from oracle.pipeline import prefill_columns, prefill_pair
from tests.gpu_util import (R16_TOL, check_coded_row, check_topk, code_rows, coding_bound, desc_for,
                            dev, r16, r16_excess, read_keys, read_kv, v4)

pytestmark = pytest.mark.gpu

W5 = synth.scaled(synth.WORKLOADS["flash_prefill_64k"], L=4000, n_queries=2000, prefix=2000,
                  name="flash_prefill_scaled")
ROWS = [0, 1, 127, 1023, 1024, 1500, 1998, 1999]      # sampled query rows


@pytest.fixture(scope="module")
def run():
    v = v4()
    w = W5
    csa, hca = w.layers
    L, n = w.L, w.n_queries
    x = synth.prefill_x(w)
    W = synth.prefill_weight(w)
    q0 = synth.prefill_queries(w, 0)
    q1 = synth.prefill_queries(w, 1)
    cols = prefill_columns(csa, hca)
    ncol = W.shape[1]
    # a0: projection of every token
    X, Wt = dev(x, torch.bfloat16), dev(W, torch.bfloat16)
    Y = torch.empty(L, ncol, dtype=torch.float32, device="cuda")
    v.project(X, Wt, Y)
    arr = {nm: Y[:, c0:c1] for nm, (c0, c1) in cols.items()}
    dc, dh = desc_for(csa), desc_for(hca)
    one = lambda val: torch.full((1,), val, dtype=torch.int64, device="cuda")
    common = dict(in_rows=L, in_seq_stride=L * ncol, in_row_stride=ncol, seq_len=one(L),
                  entry_begin=one(0))

    def rows_of(fmt, c, n_rows, d_rope=64):
        out = torch.zeros(1, n_rows, v.row_bytes(fmt, c, d_rope), dtype=torch.uint8, device="cuda")
        sc = (torch.zeros(1, n_rows, dtype=torch.float32, device="cuda") if fmt == v.E4M3_BF16ROPE
              else torch.zeros(1, n_rows, c // 32, dtype=torch.uint8, device="cuda"))
        return out, sc
    # a1: CSA entries, CSA indexer keys, HCA entries, window KV of every token
    n_c, n_h = L // csa.m, L // hca.m
    rows_c = (n_c + 127) // 128 * 128
    kv_c, kvs_c = rows_of(v.E4M3_BF16ROPE, csa.d, rows_c)
    v.compress(dc, m=csa.m, overlap=True, c=csa.d, Ca=arr["Ca"], Za=arr["Za"], Cb=arr["Cb"],
               Zb=arr["Zb"], bias=dev(q0["bias"]), n_entries=n_c, complete_only=True,
               out_dtype=v.E4M3_BF16ROPE, out=kv_c, out_scale=kvs_c, out_rows=rows_c, **common)
    keys, keys_sf = rows_of(v.MXFP4, csa.d_I, rows_c, 0)
    v.compress(dc, m=csa.m, overlap=True, c=csa.d_I, Ca=arr["ICa"], Za=arr["IZa"], Cb=arr["ICb"],
               Zb=arr["IZb"], bias=dev(q0["ibias"]), n_entries=n_c, complete_only=True,
               out_dtype=v.MXFP4, out=keys, out_scale=keys_sf, out_rows=rows_c,
               apply_rmsnorm=False, apply_rope=False, **common)
    rows_h = max(128, (n_h + 127) // 128 * 128)
    kv_h, kvs_h = rows_of(v.E4M3_BF16ROPE, hca.d, rows_h)
    v.compress(dh, m=hca.m, overlap=False, c=hca.d, Ca=arr["C"], Za=arr["Z"], bias=dev(q1["bias"]),
               n_entries=n_h, complete_only=True, out_dtype=v.E4M3_BF16ROPE, out=kv_h,
               out_scale=kvs_h, out_rows=rows_h, **common)
    swa_c, swas_c = rows_of(v.E4M3_BF16ROPE, csa.d, L)
    v.compress(dc, m=1, overlap=False, c=csa.d, Ca=arr["Ca"], Za=None, n_entries=L,
               out_dtype=v.E4M3_BF16ROPE, out=swa_c, out_scale=swas_c, out_rows=L, **common)
    swa_h, swas_h = rows_of(v.E4M3_BF16ROPE, hca.d, L)
    v.compress(dh, m=1, overlap=False, c=hca.d, Ca=arr["C"], Za=None, n_entries=L,
               out_dtype=v.E4M3_BF16ROPE, out=swa_h, out_scale=swas_h, out_rows=L, **common)
    # a2-a4: indexer queries, indexer + top-k of every query
    pos = dev(np.arange(w.prefix, L), torch.int64)
    seq = torch.zeros(n, dtype=torch.int32, device="cuda")
    qI, qI_sf = code_rows(dc, dev(q0["qI"].reshape(1, n * csa.H_I, csa.d_I)), v.MXFP4)
    qI, qI_sf = qI.reshape(n, csa.H_I, -1), qI_sf.reshape(n, csa.H_I, -1)
    idx = torch.full((n, csa.top_k), -1, dtype=torch.int32, device="cuda")
    ws_c = v.workspace(dc, n, rows_c)
    v.index_topk(dc, qI=qI, qI_sf=qI_sf, w=dev(q0["w"]), q_pos=pos, q_seq=seq, B=1, keys=keys,
                 keys_sf=keys_sf, key_rows=rows_c, max_vis=n_c, idx_out=idx, ws=ws_c)
    # a5-a7: sparse MQA (CSA) and dense MQA (HCA) of every query
    out_c = torch.zeros(n, csa.H, csa.d, dtype=torch.bfloat16, device="cuda")
    lse_c = torch.zeros(n, csa.H, dtype=torch.float32, device="cuda")
    v.sparse_mqa(dc, Q=dev(q0["Q"], torch.bfloat16), q_pos=pos, q_seq=seq, B=1, kv=kv_c,
                 kv_scale=kvs_c, kv_rows=rows_c, swa=swa_c, swa_scale=swas_c, swa_rows=L, idx=idx,
                 out=out_c, ws=ws_c, sink=dev(q0["sink"]), lse=lse_c)
    out_h = torch.zeros(n, hca.H, hca.d, dtype=torch.bfloat16, device="cuda")
    lse_h = torch.zeros(n, hca.H, dtype=torch.float32, device="cuda")
    ws_h = v.workspace(dh, n, rows_h)
    v.dense_mqa(dh, Q=dev(q1["Q"], torch.bfloat16), q_pos=pos, q_seq=seq, B=1, kv=kv_h,
                kv_scale=kvs_h, kv_rows=rows_h, swa=swa_h, swa_scale=swas_h, swa_rows=L,
                max_vis=n_h, out=out_h, ws=ws_h, sink=dev(q1["sink"]), lse=lse_h)
    torch.cuda.synchronize()
    assert v.device_status(ws_c) == 0 and v.device_status(ws_h) == 0
    ref = prefill_pair(w, x, W, synth.prefill_queries(w, 0, rows=ROWS),
                       synth.prefill_queries(w, 1, rows=ROWS), ROWS)
    return dict(v=v, w=w, Y=Y.cpu().numpy(), x=x, W=W, kv_c=kv_c.cpu().numpy(),
                kvs_c=kvs_c.cpu().numpy(), keys=keys.cpu().numpy(), keys_sf=keys_sf.cpu().numpy(),
                kv_h=kv_h.cpu().numpy(), kvs_h=kvs_h.cpu().numpy(), idx=idx.cpu().numpy(),
                swa_c=swa_c.cpu().numpy(), swas_c=swas_c.cpu().numpy(), swa_h=swa_h.cpu().numpy(),
                swas_h=swas_h.cpu().numpy(),
                out_c=out_c.float().cpu().numpy(), lse_c=lse_c.cpu().numpy(),
                out_h=out_h.float().cpu().numpy(), lse_h=lse_h.cpu().numpy(), ref=ref, q0=q0)


def test_prefill_projection_rows(run):
    x, W, Y = run["x"], run["W"], run["Y"]
    for r in (0, 1, 1999, 2000, 3999):
        want = x[r].astype(np.float64) @ W.astype(np.float64)
        assert np.max(np.abs(Y[r] - want)) <= 1e-4 * max(1.0, np.max(np.abs(want))), r


def test_prefill_entries_and_keys(run):
    v, ref = run["v"], run["ref"]
    # every CSA key, every HCA entry, the CSA entries the sampled queries selected
    kgot = read_keys(run["keys"][0, : len(ref["key_val"])], run["keys_sf"][0, : len(ref["key_val"])],
                     v.MXFP4)
    assert r16(kgot, ref["key_val"]) <= R16_TOL
    hgot = read_kv(run["kv_h"][0, : len(ref["hca_val"])], run["kvs_h"][0, : len(ref["hca_val"])],
                   v.E4M3_BF16ROPE)
    for j in range(len(ref["hca_val"])):
        check_coded_row(hgot[j], ref["hca_val"][j], ref["hca_raw"][j], what=("hca entry", j))
    for i, want in list(ref["csa_entries"].items())[:256]:
        got = read_kv(run["kv_c"][0, i], run["kvs_c"][0, i], v.E4M3_BF16ROPE)
        check_coded_row(got, want, ref["csa_raw"][i], what=("csa entry", i))


def test_prefill_topk_and_outputs(run):
    v, ref, w = run["v"], run["ref"], run["w"]
    csa = w.layers[0]
    kgot = read_keys(run["keys"][0, : len(ref["key_val"])], run["keys_sf"][0, : len(ref["key_val"])],
                     v.MXFP4)
    dk = np.abs(kgot - ref["key_val"])          # coding decisions taken differently
    for n, r in enumerate(ROWS):
        p = ref["positions"][n]
        nv = (p + 1) // csa.m
        extra = None
        if dk[:nv].any():
            qv = codecs.dequantize_mxfp4(*codecs.quantize_mxfp4(run["q0"]["qI"][r]))
            extra = np.abs(qv) @ dk[:nv].T
            extra = run["q0"]["w"][r] @ extra
        check_topk(run["idx"][r], ref["scores"][n], nv, csa.top_k, extra)
        # outputs: R16 on what the two sides' (valid, differently rounded)
        # stored key codes do not explain
        det = ref["detail"][n]
        gk = lambda rows, sc, sel: read_kv(rows[0, sel], sc[0, sel], v.E4M3_BF16ROPE)
        kc = np.concatenate([gk(run["kv_c"], run["kvs_c"], det["csa_sel"]),
                             gk(run["swa_c"], run["swas_c"], det["csa_win"])], axis=0)
        bc = coding_bound(det["csa_keys"], kc, det["csa_a"], det["csa_q"], det["csa_o"],
                          1 / np.sqrt(csa.d))
        ec = r16_excess(run["out_c"][r], ref["csa_out"][n], bc)
        assert ec <= R16_TOL, ("csa out", r, ec, r16(run["out_c"][r], ref["csa_out"][n]))
        assert np.max(np.abs(run["lse_c"][r] - ref["csa_lse"][n])) <= 5e-2, ("csa lse", r)
        hca = w.layers[1]
        kh = np.concatenate([gk(run["kv_h"], run["kvs_h"], np.arange(det["hca_n"])),
                             gk(run["swa_h"], run["swas_h"], det["hca_win"])], axis=0)
        bh = coding_bound(det["hca_keys"], kh, det["hca_a"], det["hca_q"], det["hca_o"],
                          1 / np.sqrt(hca.d))
        eh = r16_excess(run["out_h"][r], ref["hca_out"][n], bh)
        assert eh <= R16_TOL, ("hca out", r, eh, r16(run["out_h"][r], ref["hca_out"][n]))
        assert np.max(np.abs(run["lse_h"][r] - ref["hca_lse"][n])) <= 5e-2, ("hca lse", r)


def test_prefill_selection_valid_for_every_query(run):
    idx, w = run["idx"], run["w"]
    k = w.layers[0].top_k
    for r in range(w.n_queries):
        nv = (w.prefix + r + 1) // w.layers[0].m
        kk = min(k, nv)
        sel = idx[r, :kk]
        assert np.all(idx[r, kk:] == -1) and np.all(np.diff(sel) > 0)
        assert sel[0] >= 0 and sel[-1] < nv
