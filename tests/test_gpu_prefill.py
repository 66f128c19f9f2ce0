"""Chunked prefill of the V4-Flash CSA + HCA pair through the C-ABI, checked
stage-wise against the oracle (tests/parity.py): at a scaled size (L = 4000:
2000 new tokens on a 2000-token prefix, every query checked) and at the full
size of 65536 new tokens on a 65536 prefix (at least 1024 stratified query
rows, sampled entries and keys; selection validity for every query).

Every step runs in the library (bench.PrefillPair): the projection of the raw
tokens, the pooling of every entry and indexer key, the window KV of every
token, the indexer + top-k of every query, the sparse (CSA) and dense (HCA)
MQA of every query.  The checks, each on the GPU's own checked output of the
stage before:
  a0  projection rows against x @ W in float64;
  a1  entries, keys and window rows as valid codings of the oracle's pooling
      (or RMSNorm + RoPE) of the GPU's projected rows;
  a3  the oracle's scores of the keys the GPU stored, with the indexer queries
      the GPU stored: the GPU's selection (a4) within the top-k tie rule;
  a6  the oracle's attention over the rows the GPU stored and the entries it
      selected: outputs within 2e-2 max-abs / RMS, LSE within 1e-3."""
import numpy as np
import pytest
import torch

import synth
from oracle import compress as ocomp, indexer as oidx, mqa as omqa
from oracle.pipeline import token_kv
from tests.gpu_util import (check_output, check_stored_keys, check_stored_kv, check_topk,
                            oracle_attention, read_keys, read_kv)

pytestmark = pytest.mark.gpu

FULL = synth.WORKLOADS["flash_prefill_64k"]
SCALED = synth.scaled(FULL, L=4000, n_queries=2000, prefix=2000, name="flash_prefill_scaled")


def _run(w):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bench import PrefillPair
    pp = PrefillPair(w, out_dtype=torch.float32)     # parity on the fp32 outputs
    pp.prefix_state()
    pp.step()
    torch.cuda.synchronize()
    assert pp.v.device_status(pp.ws_c) == 0 and pp.v.device_status(pp.ws_h) == 0
    return pp


@pytest.fixture(scope="module")
def scaled():
    pp = _run(SCALED)
    yield pp
    del pp
    torch.cuda.empty_cache()


@pytest.fixture(scope="module")
def full():
    pp = _run(FULL)
    yield pp
    del pp
    torch.cuda.empty_cache()


def _stratified(n, P, k_uniform, seed):
    """Query rows: the first and last, rows around CSA / HCA block boundaries
    and chunk boundaries of 1024 queries, and uniform draws."""
    rows = {0, 1, 2, 3, n - 2, n - 1}
    for b in (4, 128, 1024, 4096):
        for r in range(b - 1 - (P % b), n, max(b, n // 8)):
            rows.update({r, min(n - 1, r + 1)})
    rng = np.random.default_rng(seed)
    rows.update(rng.choice(n, size=min(n, k_uniform), replace=False).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < n))


def _proj_rows(pp, rows):
    return pp.Y[torch.from_numpy(np.asarray(rows)).long().cuda()].double().cpu().numpy()


def check_projection(pp, rows):
    x = pp.x[torch.from_numpy(np.asarray(rows)).long().cuda()].float().cpu().numpy()
    W = pp.W.float().cpu().numpy().astype(np.float64)
    got = _proj_rows(pp, rows)
    want = x.astype(np.float64) @ W
    # bf16 inputs, fp32 accumulation over K = d_model terms
    tol = 1e-4 * max(1.0, float(np.max(np.abs(want))))
    assert np.max(np.abs(got - want)) <= tol


def check_entries(pp, csa_ent, hca_ent, tokens):
    """Stored CSA entries, CSA keys, HCA entries and window rows against the
    oracle's pooling / token KV of the GPU's projected rows (stage-wise)."""
    v, csa, hca, L = pp.v, pp.csa, pp.hca, pp.w.L
    cols = pp.cols

    def arrays(ents, m, overlap, names):
        tok = ocomp.window(np.asarray(ents), m, overlap)[0]
        toks = np.unique(tok[(tok >= 0) & (tok < L)])
        Yt = _proj_rows(pp, toks)
        pos = np.full(L, -1, dtype=np.int64)
        pos[toks] = np.arange(len(toks))
        return [(lambda t, c=cols[nm]: Yt[pos[t], c[0]:c[1]]) for nm in names]
    Ca, Cb, Za, Zb = arrays(csa_ent, csa.m, True, ("Ca", "Cb", "Za", "Zb"))
    raw = ocomp.finish_main(ocomp.pool(csa_ent, csa.m, True, L, Ca, Za, pp.bias_c.cpu().numpy(),
                                       Cb, Zb), csa_ent, csa.m, csa.d_rope, csa.rope_theta)
    sel = torch.from_numpy(np.asarray(csa_ent)).long().cuda()
    check_stored_kv(pp.kv_c[0][sel], pp.kvs_c[0][sel], v.E4M3_BF16ROPE, raw, what="csa entries")
    ICa, ICb, IZa, IZb = arrays(csa_ent, csa.m, True, ("ICa", "ICb", "IZa", "IZb"))
    kraw = ocomp.pool(csa_ent, csa.m, True, L, ICa, IZa, pp.ibias.cpu().numpy(), ICb, IZb)
    check_stored_keys(pp.keys[0][sel], pp.keys_sf[0][sel], v.MXFP4, kraw, "csa keys")
    C, Z = arrays(hca_ent, hca.m, False, ("C", "Z"))
    hraw = ocomp.finish_main(ocomp.pool(hca_ent, hca.m, False, L, C, Z, pp.bias_h.cpu().numpy()),
                             hca_ent, hca.m, hca.d_rope, hca.rope_theta)
    hs = torch.from_numpy(np.asarray(hca_ent)).long().cuda()
    check_stored_kv(pp.kv_h[0][hs], pp.kvs_h[0][hs], v.E4M3_BF16ROPE, hraw, what="hca entries")
    Yt = _proj_rows(pp, tokens)
    ts = torch.from_numpy(np.asarray(tokens)).long().cuda()
    for ly, col, swa, sc in ((csa, "Ca", pp.swa_c, pp.swas_c), (hca, "C", pp.swa_h, pp.swas_h)):
        c0, c1 = cols[col]
        traw = token_kv(Yt[:, c0:c1], np.asarray(tokens), ly)
        check_stored_kv(swa[0][ts], sc[0][ts], v.E4M3_BF16ROPE, traw, what=("window", col))


def check_queries(pp, rows):
    """Indexer + top-k, sparse MQA and dense MQA of the query rows, on the
    GPU's stored keys, entries and window rows."""
    v, csa, hca, w = pp.v, pp.csa, pp.hca, pp.w
    P = w.prefix
    nk = w.L // csa.m
    keys = read_keys(pp.keys[0, :nk], pp.keys_sf[0, :nk], v.MXFP4)
    rt = torch.from_numpy(np.asarray(rows)).long().cuda()
    qv = read_keys(pp.qI[rt], pp.qI_sf[rt], v.MXFP4)
    wI = pp.wI[rt].cpu().numpy()
    idx = pp.idx[rt].cpu().numpy()
    Qc, Qh = pp.Q_c[rt].float().cpu().numpy(), pp.Q_h[rt].float().cpu().numpy()
    oc, lc = pp.out_c[rt].float().cpu().numpy(), pp.lse_c[rt].cpu().numpy()
    oh, lh = pp.out_h[rt].float().cpu().numpy(), pp.lse_h[rt].cpu().numpy()
    sink_c, sink_h = pp.sink_c.cpu().numpy(), pp.sink_h.cpu().numpy()
    nh = w.L // hca.m
    ent_h = read_kv(pp.kv_h[0, :nh], pp.kvs_h[0, :nh], v.E4M3_BF16ROPE)
    swaps = 0
    for n, r in enumerate(rows):
        p = P + int(r)
        nv = (p + 1) // csa.m
        s = oidx.scores(qv[n], wI[n], keys[:nv])
        swaps += check_topk(idx[n], s, nv, csa.top_k)
        sel = idx[n][idx[n] >= 0]
        st = torch.from_numpy(sel).long().cuda()
        win = omqa.window_tokens(p, csa.n_win)
        wt = torch.from_numpy(win).long().cuda()
        kc = np.concatenate([read_kv(pp.kv_c[0][st], pp.kvs_c[0][st], v.E4M3_BF16ROPE),
                             read_kv(pp.swa_c[0][wt], pp.swas_c[0][wt], v.E4M3_BF16ROPE)], 0)
        o, lse = oracle_attention(Qc[n], p, kc, sink_c, csa, True)
        check_output(oc[n], o, lc[n], lse, False, ("csa query", int(r)))
        nvh = (p + 1) // hca.m
        kh = np.concatenate([ent_h[:nvh],
                             read_kv(pp.swa_h[0][wt], pp.swas_h[0][wt], v.E4M3_BF16ROPE)], 0)
        o, lse = oracle_attention(Qh[n], p, kh, sink_h, hca, True)
        check_output(oh[n], o, lh[n], lse, False, ("hca query", int(r)))
    return swaps


def check_selection_valid(pp):
    w, csa = pp.w, pp.csa
    idx = pp.idx.cpu().numpy()
    nv = (w.prefix + np.arange(w.n_queries) + 1) // csa.m
    kk = np.minimum(csa.top_k, nv)
    col = np.arange(csa.top_k)[None, :]
    valid = col < kk[:, None]
    assert np.all(idx[~valid] == -1)
    assert np.all(idx[valid] >= 0) and np.all((idx < nv[:, None])[valid])
    d = np.diff(idx, axis=1)
    assert np.all(d[valid[:, 1:]] > 0)


# ------------------------------------------------------------------ scaled (every query)

def test_scaled_projection(scaled):
    check_projection(scaled, [0, 1, 1999, 2000, 3999])


def test_scaled_entries_keys_and_window(scaled):
    w = scaled.w
    check_entries(scaled, np.arange(w.L // 4), np.arange(w.L // 128), np.arange(w.L))


def test_scaled_every_query(scaled):
    check_queries(scaled, np.arange(scaled.w.n_queries))
    check_selection_valid(scaled)


def test_scaled_bf16_outputs_are_rounded_fp32(scaled):
    """The same step with bf16 outputs gives the bf16 rounding of the fp32
    outputs, bit for bit (the step is idempotent)."""
    f32 = (scaled.out_c.clone(), scaled.out_h.clone())
    scaled.out_c = torch.zeros(f32[0].shape, dtype=torch.bfloat16, device="cuda")
    scaled.out_h = torch.zeros(f32[1].shape, dtype=torch.bfloat16, device="cuda")
    scaled.step()
    torch.cuda.synchronize()
    assert torch.equal(scaled.out_c, f32[0].to(torch.bfloat16))
    assert torch.equal(scaled.out_h, f32[1].to(torch.bfloat16))
    scaled.out_c, scaled.out_h = f32


# ------------------------------------------------------------------ full size (sampled)

def test_full_projection_and_entries(full):
    w = full.w
    rng = np.random.default_rng(5)
    check_projection(full, [0, 1, w.prefix - 1, w.prefix, w.L - 1] +
                     rng.choice(w.L, 11, replace=False).tolist())
    nc, nh = w.L // 4, w.L // 128
    ce = np.unique(np.concatenate([[0, 1, w.prefix // 4 - 1, w.prefix // 4, nc - 1],
                                   rng.choice(nc, 251, replace=False)]))
    te = np.unique(np.concatenate([[0, w.prefix - 1, w.prefix, w.L - 1],
                                   rng.choice(w.L, 252, replace=False)]))
    check_entries(full, ce, np.arange(nh), te)


def test_full_stratified_queries(full):
    rows = _stratified(full.w.n_queries, full.w.prefix, 1000, 7)
    assert len(rows) >= 1024
    check_queries(full, rows)
    check_selection_valid(full)
