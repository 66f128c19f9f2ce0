"""Paged compressed caches ([deep-read] "异构 KV cache 与磁盘前缀复用": a
classical block cache over blocks of lcm(4, 128) = 128 raw tokens, i.e. 32 CSA
entries and 32 indexer keys, or one HCA entry, a block).  The same data is
stored once per sequence (contiguous) and once scattered over a shuffled pool
of blocks behind a block table; every call must give the same result both
ways: the indexer's scores and selection and the sparse MQA bit for bit (the
same arithmetic on the same rows), the dense MQA (whose paged rows are
gathered, so its key splits fall elsewhere and its f16 split partials round
differently: 2^-11 relative) within 5e-3 of the output's RMS, and
the decode step's appended rows at their blocks' slots.  The paged results
are also checked against the oracle, and a table entry outside the pool must
be caught by the kernels (status bit, no access)."""
import numpy as np
import pytest
import torch

import synth
from oracle import compress as ocomp, indexer as oidx, mqa as omqa
from tests.gpu_util import (DecodeState, check_output, check_topk, code_rows, desc_for, dev,
                            oracle_attention, read_keys, read_kv, v4)

pytestmark = pytest.mark.gpu

BLOCK_TOKENS = 128          # raw tokens a block covers
ST_BAD_INDEX = 1 << 1
# paged against per-sequence dense MQA: the same keys split over other CTAs,
# merged from f16 partials (2^-11 relative each): about 1e-3 of the RMS apart
SPLIT_TOL = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _table(rng, B, bps, spare):
    """A block table of B x bps distinct blocks drawn from a shuffled pool of
    B * bps + spare blocks (int32 [B][bps]) and the pool size."""
    n = B * bps + spare
    return rng.permutation(n)[: B * bps].reshape(B, bps).astype(np.int32), n


def _scatter(rows, table, epb, n_blocks):
    """Per-sequence rows [B][bps * epb][...] -> pool [n_blocks * epb][...] in
    which logical block i of sequence b sits at block table[b][i]."""
    B, bps = table.shape
    pool = torch.zeros((n_blocks * epb,) + tuple(rows.shape[2:]), dtype=rows.dtype,
                       device=rows.device)
    for b in range(B):
        for i in range(bps):
            pb = int(table[b, i])
            pool[pb * epb:(pb + 1) * epb] = rows[b, i * epb:(i + 1) * epb]
    return pool


def _pool_row(table, epb, b, e):
    return int(table[b, e // epb]) * epb + e % epb


@pytest.mark.parametrize("H_I,one_seq", [(64, False), (128, False), (64, True)])
def test_paged_index_topk_matches_contiguous(H_I, one_seq):
    v = v4()
    rng = np.random.default_rng(H_I + one_seq)
    epb, bps = 32, 150                          # 4800 keys a sequence
    B = 1 if one_seq else 3
    N, k, d_I = epb * bps, 64, 128
    keys = rng.standard_normal((B, N, d_I)).astype(np.float32)
    if one_seq:     # consecutive queries of one sequence: the paired form
        positions = np.array([4 * N - 1, 4 * N - 6, 4 * 700 + 3, 4 * 700 + 4, 9, 4 * 33])
        q_seq = np.zeros(len(positions), np.int32)
    else:           # block edges: the last key of a block, the first of the next
        positions = np.array([4 * N - 1, 4 * 32 * 7 - 1, 4 * 32 * 7 + 3, 2, 4 * N - 5, 4 * 3001])
        q_seq = np.array([0, 1, 2, 0, 2, 1], dtype=np.int32)
    nq = len(positions)
    qI = rng.standard_normal((nq, H_I, d_I)).astype(np.float32)
    w = rng.uniform(-0.2, 1, (nq, H_I)).astype(np.float32)
    ly = synth.Layer("csa", 4, 16, 512, 64, 128, H_I, d_I, k, idx_fp4=True)
    desc = desc_for(ly)
    krows, ksf = code_rows(desc, dev(keys), v.MXFP4)
    qrows, qsf = code_rows(desc, dev(qI.reshape(1, nq * H_I, d_I)), v.MXFP4)
    qrows, qsf = qrows.reshape(nq, H_I, -1), qsf.reshape(nq, H_I, -1)
    table, n_blocks = _table(rng, B, bps, 7)
    pk, psf = _scatter(krows, table, epb, n_blocks), _scatter(ksf, table, epb, n_blocks)
    res = []
    for paged in (False, True):
        idx = torch.full((nq, k), -9, dtype=torch.int32, device="cuda")
        scores = torch.zeros(nq, N, dtype=torch.float32, device="cuda")
        ws = v.workspace(desc, nq, N)
        kw = dict(keys=pk, keys_sf=psf, key_rows=n_blocks * epb,
                  block_table=dev(table, torch.int32)) if paged else \
            dict(keys=krows, keys_sf=ksf, key_rows=N)
        v.index_topk(desc, qI=qrows, qI_sf=qsf, w=dev(w), q_pos=dev(positions, torch.int64),
                     q_seq=dev(q_seq, torch.int32), B=B, max_vis=N, idx_out=idx,
                     scores_out=scores, ws=ws, **kw)
        torch.cuda.synchronize()
        assert v.device_status(ws) == 0
        res.append((idx.cpu().numpy(), scores.cpu().numpy()))
    assert np.array_equal(res[0][1], res[1][1])
    assert np.array_equal(res[0][0], res[1][0])
    # and the oracle on the keys as stored
    kd = read_keys(krows, ksf, v.MXFP4)
    qd = read_keys(qrows, qsf, v.MXFP4)
    for q in range(nq):
        nv = int(ocomp.n_visible(positions[q], 4))
        s = oidx.scores(qd[q], w[q], kd[q_seq[q], :nv])
        scale = max(1.0, float(np.max(np.abs(s)))) if nv else 1.0
        assert np.max(np.abs(res[1][1][q, :nv] - s), initial=0.0) <= 1e-5 * scale
        check_topk(res[1][0][q], s, nv, k)


def test_paged_index_bad_table_entry_is_caught():
    """A visible block whose table entry lies outside the pool: the kernel
    skips its loads and records ST_BAD_INDEX; the next good call succeeds."""
    v = v4()
    rng = np.random.default_rng(3)
    epb, bps, H_I, d_I, k = 32, 40, 64, 128, 32
    N = epb * bps
    keys = rng.standard_normal((1, N, d_I)).astype(np.float32)
    qI = rng.standard_normal((1, H_I, d_I)).astype(np.float32)
    ly = synth.Layer("csa", 4, 16, 512, 64, 128, H_I, d_I, k, idx_fp4=True)
    desc = desc_for(ly)
    krows, ksf = code_rows(desc, dev(keys), v.MXFP4)
    qrows, qsf = code_rows(desc, dev(qI), v.MXFP4)
    table, n_blocks = _table(rng, 1, bps, 0)
    pk, psf = _scatter(krows, table, epb, n_blocks), _scatter(ksf, table, epb, n_blocks)
    bad = table.copy()
    bad[0, 5] = n_blocks + 100
    idx = torch.full((1, k), -9, dtype=torch.int32, device="cuda")
    ws = v.workspace(desc, 1, N)
    kw = dict(qI=qrows.reshape(1, H_I, -1), qI_sf=qsf.reshape(1, H_I, -1),
              w=dev(np.ones((1, H_I), np.float32)), q_pos=dev(np.array([4 * N - 1]), torch.int64),
              B=1, keys=pk, keys_sf=psf, key_rows=n_blocks * epb, max_vis=N, idx_out=idx, ws=ws)
    v.index_topk(desc, block_table=dev(bad, torch.int32), **kw)
    code, bits = v.device_status_code(ws)
    assert bits & ST_BAD_INDEX and code == 6          # V4A_ERR_DEVICE_CHECK
    v.workspace_init(ws)
    v.index_topk(desc, block_table=dev(table, torch.int32), **kw)
    torch.cuda.synchronize()
    assert v.device_status(ws) == 0


@pytest.mark.parametrize("sparse", [True, False])
def test_paged_mqa_matches_contiguous(sparse):
    v = v4()
    rng = np.random.default_rng(17 + sparse)
    m = 4 if sparse else 128
    epb = BLOCK_TOKENS // m
    B, H, d, d_rope, n_win, k = 3, 128, 512, 64, 128, 96
    bps = 24 if sparse else 700                    # 768 CSA entries / 700 HCA entries a sequence
    N = epb * bps
    ly = synth.Layer("csa" if sparse else "hca", m, H, d, d_rope, n_win, 4, 32, k)
    desc = desc_for(ly)
    fmt = v.E4M3_BF16ROPE
    ents = rng.standard_normal((B, N, d)).astype(np.float32)
    swa_rows = 256
    swa_vals = rng.standard_normal((B, swa_rows, d)).astype(np.float32)
    kv, kv_sc = code_rows(desc, dev(ents), fmt, d_rope=d_rope)
    swa, swa_sc = code_rows(desc, dev(swa_vals), fmt, d_rope=d_rope)
    positions = np.array([m * N - 1, m * 300 + 1, 5, m * 10, m * N - 2, 200])
    q_seq = np.array([0, 1, 2, 2, 1, 0], dtype=np.int32)
    nq = len(positions)
    Q = synth.bf16_values(rng.standard_normal((nq, H, d)).astype(np.float32))
    sink = rng.standard_normal(H).astype(np.float32)
    idx = np.full((nq, k), -1, dtype=np.int32)
    for q in range(nq):
        nv = int(ocomp.n_visible(positions[q], m))
        sel = np.sort(rng.choice(nv, size=min(k, nv), replace=False)) if nv else np.zeros(0, int)
        idx[q, : len(sel)] = sel
    table, n_blocks = _table(rng, B, bps, 5)
    pkv, psc = _scatter(kv, table, epb, n_blocks), _scatter(kv_sc, table, epb, n_blocks)
    outs = []
    for paged in (False, True):
        out = torch.zeros(nq, H, d, dtype=torch.float32, device="cuda")
        lse = torch.zeros(nq, H, dtype=torch.float32, device="cuda")
        ws = v.workspace(desc, nq, N)
        cache = dict(kv=pkv, kv_scale=psc, kv_rows=n_blocks * epb,
                     block_table=dev(table, torch.int32)) if paged else \
            dict(kv=kv, kv_scale=kv_sc, kv_rows=N)
        kw = dict(Q=dev(Q, torch.bfloat16), q_pos=dev(positions, torch.int64),
                  q_seq=dev(q_seq, torch.int32), B=B, swa=swa, swa_scale=swa_sc,
                  swa_rows=swa_rows, out=out, ws=ws, sink=dev(sink), lse=lse, **cache)
        if sparse:
            v.sparse_mqa(desc, idx=dev(idx, torch.int32), **kw)
        else:
            v.dense_mqa(desc, max_vis=N, **kw)
        torch.cuda.synchronize()
        assert v.device_status(ws) == 0
        outs.append((out.cpu().numpy(), lse.cpu().numpy()))
    if sparse:
        assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    else:
        rms = float(np.sqrt(np.mean(outs[0][0] ** 2)))
        assert np.max(np.abs(outs[0][0] - outs[1][0])) <= SPLIT_TOL * rms
        assert np.max(np.abs(outs[0][1] - outs[1][1])) <= SPLIT_TOL
    e_val = read_kv(kv, kv_sc, fmt, d, d_rope)
    s_val = read_kv(swa, swa_sc, fmt, d, d_rope)
    for q in range(nq):
        p, b = int(positions[q]), int(q_seq[q])
        nv = int(ocomp.n_visible(p, m))
        rows = idx[q][idx[q] >= 0] if sparse else np.arange(nv)
        toks = omqa.window_tokens(p, n_win)
        keys = np.concatenate([e_val[b, rows], s_val[b, toks % swa_rows]], 0)
        o, l = oracle_attention(Q[q], p, keys, sink, ly, True)
        check_output(outs[1][0][q], o, outs[1][1][q], l, False, ("query", q))


@pytest.mark.parametrize("kind,L", [("csa", 4 * 3000), ("hca", 128 * 40)])
def test_paged_decode_step_matches_contiguous(kind, L):
    """One decode step on paged caches against the same step on the per-sequence
    caches: the same selection, the same (CSA) or SPLIT_TOL-close (HCA)
    output, and the appended entry (and indexer key) at its block's slot."""
    v = v4()
    base = synth.WORKLOADS["csa_flash_128k" if kind == "csa" else "hca_flash_128k"]
    w = synth.scaled(base, B=3, L=L, top_k=64, name=f"paged_{kind}")
    inp = synth.decode_layer_inputs(w, 0)
    st = DecodeState(w, 0, inp)
    lay = st.lay
    epb = BLOCK_TOKENS // lay.m
    bps = lay.kv_rows // epb
    rng = np.random.default_rng(len(kind))
    table, n_blocks = _table(rng, st.B, bps, 9)
    bt = dev(table, torch.int32)
    # the paged copy of every cache, taken before the contiguous step
    pkv, psc = _scatter(lay.kv, table, epb, n_blocks), _scatter(lay.kv_scale, table, epb, n_blocks)
    rings = {n: getattr(lay, n).clone() for n in ("tail", "swa", "swa_scale") if getattr(lay, n) is not None}
    if st.csa:
        rings["itail"] = lay.itail.clone()
        pk, psf = _scatter(lay.keys, table, epb, n_blocks), _scatter(lay.keys_sf, table, epb, n_blocks)
    st.step()
    torch.cuda.synchronize()
    assert v.device_status(st.ws) == 0
    out_c, lse_c = lay.out.clone(), lay.lse.clone()
    idx_c = lay.idx.clone() if st.csa else None
    # the same step on the paged caches (fresh copies of the rings)
    for n, t in rings.items():
        getattr(lay, n).copy_(t)
    out_p = torch.zeros_like(lay.out)
    lse_p = torch.zeros_like(lay.lse)
    kw = {}
    if st.csa:
        idx_p = torch.full_like(lay.idx, -9)
        kw = dict(x_idx=lay.x_idx, itail=lay.itail, ibias=lay.ibias, keys=pk, keys_sf=psf,
                  key_rows=n_blocks * epb, qI=lay.qI, qI_sf=lay.qI_sf, w=lay.w, idx_out=idx_p)
    v.workspace_init(lay.ws)
    v.decode(lay.desc, pos=lay.pos, x_main=lay.x_main, tail=lay.tail, bias=lay.bias, kv=pkv,
             kv_scale=psc, kv_rows=n_blocks * epb, swa=lay.swa, swa_scale=lay.swa_scale,
             swa_rows=lay.swa_rows, Q=lay.Q, out=out_p, ws=lay.ws, max_vis=st.max_vis,
             sink=lay.sink, lse=lse_p, block_table=bt, **kw)
    torch.cuda.synchronize()
    assert v.device_status(lay.ws) == 0
    if st.csa:
        assert torch.equal(idx_p, idx_c)
        assert torch.equal(out_p, out_c) and torch.equal(lse_p, lse_c)
    else:
        rms = float(out_c.float().pow(2).mean().sqrt())
        assert float((out_p.float() - out_c.float()).abs().max()) <= SPLIT_TOL * rms
        assert float((lse_p - lse_c).abs().max()) <= SPLIT_TOL
    # the entry (and key) this step completed, at its block's slot
    p = int(inp["p"])
    if (p + 1) % lay.m == 0:
        e = (p + 1) // lay.m - 1
        for b in range(st.B):
            r = _pool_row(table, epb, b, e)
            assert torch.equal(pkv[r], lay.kv[b, e]) and torch.equal(psc[r], lay.kv_scale[b, e])
            if st.csa:
                assert torch.equal(pk[r], lay.keys[b, e]) and torch.equal(psf[r], lay.keys_sf[b, e])
