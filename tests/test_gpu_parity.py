"""GPU parity: every stage of the CUDA path, called through the C ABI, against
the fp64 CPU oracle on the same seeded inputs - small cases that span several
tiles with ragged tails, the edge cases (first entries, partial windows,
fewer visible keys than k, no sink), and the five workloads at full size with
sampled sequences."""
import numpy as np
import pytest
import torch

import synth
from oracle import codecs, compress as ocomp, indexer as oidx, mqa as omqa, pipeline
from tests.gpu_util import (F32_ABS_TOL, LSE_ABS_TOL, R16_TOL, DecodeState, check_output,
                            check_stored_keys, check_stored_kv, check_topk, code_rows,
                            check_bf16_output_is_rounded_fp32, compare_decode, desc_for, dev,
                            oracle_attention, r16, read_keys, read_kv, v4)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


# ------------------------------------------------------------------ coding (bit-exact)

def test_coding_is_bit_exact():
    v = v4()
    rng = np.random.default_rng(11)
    vals = rng.standard_normal((3, 300, 512)).astype(np.float32)
    vals[0, :50] *= 1e-3
    vals[1, :50] *= 1e3
    vals[2, 7] = 0.0
    vals[2, 8, :448] = 0.0
    d = v.layer_desc(v.HCA, 128, 64, 512, 64)
    rows, sc = code_rows(d, dev(vals), v.E4M3_BF16ROPE)
    codes, rbits, s = codecs.quantize_kv(vals.astype(np.float64), 64)
    g = rows.cpu().numpy()
    assert np.array_equal(g[..., :448], codes)
    assert np.array_equal(g[..., 448:].copy().view(np.uint16), rbits)
    assert np.array_equal(sc.cpu().numpy(), s)
    # MXFP4 (128 channels), including an all-zero block and saturating blocks
    kv = rng.standard_normal((2, 700, 128)).astype(np.float32)
    kv[0, 3, :32] = 0.0
    kv[1, 5] *= 1e-30
    rows, sf = code_rows(d, dev(kv), v.MXFP4)
    c2, sf2 = codecs.quantize_mxfp4(kv.astype(np.float64))
    assert np.array_equal(rows.cpu().numpy(), codecs.pack_e2m1(c2))
    assert np.array_equal(sf.cpu().numpy(), sf2)
    rows, _ = code_rows(d, dev(kv), v.F32)
    assert np.array_equal(rows.cpu().numpy().view(np.float32), kv)


# ------------------------------------------------------------------ compression

@pytest.mark.parametrize("kind,m,L,fmt,c,ring", [
    ("csa", 4, 4 * 37 + 3, "e4m3", 512, None),
    ("csa", 4, 4 * 200, "mxfp4", 128, None),
    ("csa", 4, 4 * 61 + 1, "f32", 128, None),
    ("hca", 128, 128 * 5 + 77, "e4m3", 512, None),
    ("hca", 128, 128 * 3, "f32", 64, None),
    ("csa", 4, 4 * 50, "e4m3", 512, 8),      # tail ring input
    ("hca", 128, 128 * 4, "e4m3", 512, 128),
])
@pytest.mark.parametrize("in_bf16", [False, True])
def test_compress_parity(kind, m, L, fmt, c, ring, in_bf16):
    v = v4()
    rng = np.random.default_rng(L + c)
    B = 2
    overlap = kind == "csa"
    arrs = {nm: rng.standard_normal((B, L, c)).astype(np.float32) for nm in ("Ca", "Za", "Cb", "Zb")}
    if in_bf16:
        arrs = {k: synth.bf16_values(a) for k, a in arrs.items()}
    bias = (rng.standard_normal((2 * m if overlap else m, c)) * 0.1).astype(np.float32)
    n_ent = ocomp.n_entries(L, m)
    if ring is None:
        e0, n_e, rows_in = 0, n_ent, L
        dev_arrs = {k: dev(a, torch.bfloat16 if in_bf16 else torch.float32) for k, a in arrs.items()}
    else:
        # only the last complete block, read from a ring of `ring` rows
        e0, n_e, rows_in = L // m - 1, 1, ring
        rr = {}
        for k, a in arrs.items():
            r = np.zeros((B, ring, c), dtype=np.float32)
            for t in range(L - ring, L):
                r[:, t % ring] = a[:, t]
            rr[k] = dev(r, torch.bfloat16 if in_bf16 else torch.float32)
        dev_arrs = rr
    fmt_id = {"e4m3": v.E4M3_BF16ROPE, "mxfp4": v.MXFP4, "f32": v.F32}[fmt]
    norm_rope = fmt != "mxfp4"
    d_rope = 64 if c == 512 else (32 if c >= 64 else 0)
    desc = v.layer_desc(v.CSA if overlap else v.HCA, m, 16, 512, d_rope)
    out_rows = n_ent + 3
    rb = v.row_bytes(fmt_id, c, d_rope)
    out = torch.zeros(B, out_rows, rb, dtype=torch.uint8, device="cuda")
    sc = (torch.zeros(B, out_rows, dtype=torch.float32, device="cuda") if fmt == "e4m3" else
          torch.zeros(B, out_rows, c // 32, dtype=torch.uint8, device="cuda") if fmt == "mxfp4"
          else None)
    lens = torch.full((B,), L, dtype=torch.int64, device="cuda")
    eb = torch.full((B,), e0, dtype=torch.int64, device="cuda")
    v.compress(desc, m=m, overlap=overlap, c=c, Ca=dev_arrs["Ca"], Za=dev_arrs["Za"],
               Cb=dev_arrs["Cb"] if overlap else None, Zb=dev_arrs["Zb"] if overlap else None,
               in_rows=rows_in, in_seq_stride=rows_in * c, in_row_stride=c, bias=dev(bias),
               seq_len=lens, entry_begin=eb, n_entries=n_e, out_dtype=fmt_id, out=out,
               out_scale=sc, out_rows=out_rows, apply_rmsnorm=norm_rope, apply_rope=norm_rope)
    torch.cuda.synchronize()
    ii = np.arange(e0, e0 + n_e)
    g = out.cpu().numpy()
    scn = None if sc is None else sc.cpu().numpy()
    for b in range(B):
        a64 = {k: a[b].astype(np.float64) for k, a in arrs.items()}
        e = ocomp.pool(ii, m, overlap, L, a64["Ca"], a64["Za"], bias, a64["Cb"], a64["Zb"])
        if norm_rope:
            e = ocomp.finish_main(e, ii, m, d_rope, 160000.0)
        # stored codes: the oracle's codes of its pooled values, except where
        # a float32 rounding decision may legitimately go the other way
        if fmt == "mxfp4":
            check_stored_keys(g[b, ii], scn[b, ii], fmt_id, e, ("entries", b))
        else:
            check_stored_kv(g[b, ii], None if scn is None else scn[b, ii], fmt_id, e, c, d_rope,
                            ("entries", b))
    # rows outside the computed range are untouched
    assert not g[:, n_ent:].any()


# ------------------------------------------------------------------ indexer + top-k

@pytest.mark.parametrize("fp4,d_I,H_I", [(True, 128, 64), (False, 32, 4), (False, 64, 16),
                                          (True, 128, 128), (True, 128, 32)])
def test_index_topk_parity(fp4, d_I, H_I):
    v = v4()
    rng = np.random.default_rng(d_I + H_I)
    B, N, k = 3, 3000, 64
    keys = rng.standard_normal((B, N, d_I)).astype(np.float32)
    positions = np.array([4 * N - 1, 4 * 700 + 2, 4 * 10 + 1, 2, 4 * N - 5, 4 * 2999 + 3])
    q_seq = np.array([0, 1, 2, 0, 2, 1], dtype=np.int32)
    nq = len(positions)
    qI = rng.standard_normal((nq, H_I, d_I)).astype(np.float32)
    w = rng.uniform(0, 1, (nq, H_I)).astype(np.float32)
    ly = synth.Layer("csa", 4, 16, 512, 64, 128, H_I, d_I, k, idx_fp4=fp4)
    desc = desc_for(ly)
    kfmt = v.MXFP4 if fp4 else v.F32
    krows, ksf = code_rows(desc, dev(keys), kfmt)
    qrows, qsf = code_rows(desc, dev(qI.reshape(1, nq * H_I, d_I)), kfmt)
    qrows = qrows.reshape(nq, H_I, -1)
    qsf = None if qsf is None else qsf.reshape(nq, H_I, -1)
    idx = torch.full((nq, k), -9, dtype=torch.int32, device="cuda")
    scores = torch.zeros(nq, N, dtype=torch.float32, device="cuda")
    ws = v.workspace(desc, nq, N)
    v.index_topk(desc, qI=qrows, qI_sf=qsf, w=dev(w), q_pos=dev(positions, torch.int64),
                 q_seq=dev(q_seq, torch.int32), B=B, keys=krows, keys_sf=ksf, key_rows=N,
                 max_vis=N, idx_out=idx, scores_out=scores, ws=ws)
    torch.cuda.synchronize()
    assert v.device_status(ws) == 0
    # stage-wise: the oracle scores the keys and queries as the GPU stored them
    # (the coding itself is checked bit-exact in test_coding_is_bit_exact)
    kd = read_keys(krows, ksf, kfmt)
    qd = read_keys(qrows, qsf, kfmt)
    g_idx, g_s = idx.cpu().numpy(), scores.cpu().numpy()
    for q in range(nq):
        nv = int(ocomp.n_visible(positions[q], 4))
        s = oidx.scores(qd[q], w[q], kd[q_seq[q], :nv])
        scale = max(1.0, float(np.max(np.abs(s)))) if nv else 1.0
        assert np.max(np.abs(g_s[q, :nv] - s), initial=0.0) <= 1e-5 * scale
        assert np.all(np.isneginf(g_s[q, nv:]))
        check_topk(g_idx[q], s, nv, k)


@pytest.mark.parametrize("H_I,nq", [(64, 8), (32, 6), (64, 7), (128, 6)])
def test_index_topk_one_sequence_pairs(H_I, nq):
    """Queries of one sequence (B = 1): the tensor-core indexer scores two
    consecutive queries per key tile when their count is even (7: every
    query alone; H_I = 128: alone, N = 128).  Positions differ inside a pair,
    down to one key.  16384 keys give every CTA several tiles, so that its
    stages fill up to their tile limit (the accumulator count at N = 128)."""
    v = v4()
    rng = np.random.default_rng(H_I + nq)
    N, k, d_I = 16384, 64, 128
    keys = rng.standard_normal((1, N, d_I)).astype(np.float32)
    positions = np.array([4 * N - 1, 4 * N - 5, 4 * 700 + 3, 4 * 700 + 4, 9, 4 * 129,
                          4 * 1000 + 1, 4 * 1000 + 2])[:nq]
    qI = rng.standard_normal((nq, H_I, d_I)).astype(np.float32)
    w = rng.uniform(-0.2, 1, (nq, H_I)).astype(np.float32)
    ly = synth.Layer("csa", 4, 16, 512, 64, 128, H_I, d_I, k, idx_fp4=True)
    desc = desc_for(ly)
    krows, ksf = code_rows(desc, dev(keys), v.MXFP4)
    qrows, qsf = code_rows(desc, dev(qI.reshape(1, nq * H_I, d_I)), v.MXFP4)
    qrows, qsf = qrows.reshape(nq, H_I, -1), qsf.reshape(nq, H_I, -1)
    idx = torch.full((nq, k), -9, dtype=torch.int32, device="cuda")
    scores = torch.zeros(nq, N, dtype=torch.float32, device="cuda")
    ws = v.workspace(desc, nq, N)
    v.index_topk(desc, qI=qrows, qI_sf=qsf, w=dev(w), q_pos=dev(positions, torch.int64),
                 q_seq=dev(np.zeros(nq), torch.int32), B=1, keys=krows, keys_sf=ksf,
                 key_rows=N, max_vis=N, idx_out=idx, scores_out=scores, ws=ws)
    torch.cuda.synchronize()
    assert v.device_status(ws) == 0
    kd = read_keys(krows, ksf, v.MXFP4)
    qd = read_keys(qrows, qsf, v.MXFP4)
    g_idx, g_s = idx.cpu().numpy(), scores.cpu().numpy()
    for q in range(nq):
        nv = int(ocomp.n_visible(positions[q], 4))
        s = oidx.scores(qd[q], w[q], kd[0, :nv])
        scale = max(1.0, float(np.max(np.abs(s)))) if nv else 1.0
        assert np.max(np.abs(g_s[q, :nv] - s), initial=0.0) <= 1e-5 * scale
        assert np.all(np.isneginf(g_s[q, nv:]))
        check_topk(g_idx[q], s, nv, k)


@pytest.mark.parametrize("one_seq", [False, True])
def test_index_topk_bf16_scores(one_seq):
    """score_dtype BF16: every score rounded to bf16 (checked against the
    oracle's scores of the GPU's stored keys within bf16 rounding), the
    selection exact among those bf16 values (ties to the lower index), and
    its recall of the fp32 selection reported (the bf16 grid makes near-ties
    of the fp32 scores exact ties)."""
    v = v4()
    rng = np.random.default_rng(11 + one_seq)
    H_I, d_I, k = 64, 128, 256
    B, N = (1, 16384) if one_seq else (3, 20000)
    keys = rng.standard_normal((B, N, d_I)).astype(np.float32)
    positions = (np.array([4 * N - 1, 4 * N - 5, 4 * 700 + 3, 4 * 700 + 4, 9, 4 * 129])
                 if one_seq else np.array([4 * N - 1, 4 * 7000 + 2, 4 * 100, 4 * N - 9]))
    nq = len(positions)
    q_seq = np.zeros(nq, np.int32) if one_seq else np.array([0, 1, 2, 1], np.int32)
    qI = rng.standard_normal((nq, H_I, d_I)).astype(np.float32)
    w = rng.uniform(0, 1, (nq, H_I)).astype(np.float32)
    ly = synth.Layer("csa", 4, 16, 512, 64, 128, H_I, d_I, k, idx_fp4=True)
    desc = desc_for(ly)
    krows, ksf = code_rows(desc, dev(keys), v.MXFP4)
    qrows, qsf = code_rows(desc, dev(qI.reshape(1, nq * H_I, d_I)), v.MXFP4)
    qrows, qsf = qrows.reshape(nq, H_I, -1), qsf.reshape(nq, H_I, -1)
    idx = torch.full((nq, k), -9, dtype=torch.int32, device="cuda")
    scores = torch.zeros(nq, N, dtype=torch.bfloat16, device="cuda")
    ws = v.workspace(desc, nq, N)
    v.index_topk(desc, qI=qrows, qI_sf=qsf, w=dev(w), q_pos=dev(positions, torch.int64),
                 q_seq=dev(q_seq, torch.int32), B=B, keys=krows, keys_sf=ksf, key_rows=N,
                 max_vis=N, idx_out=idx, scores_out=scores, ws=ws, score_dtype=v.BF16)
    torch.cuda.synchronize()
    assert v.device_status(ws) == 0
    kd = read_keys(krows, ksf, v.MXFP4)
    qd = read_keys(qrows, qsf, v.MXFP4)
    g_idx, g_s = idx.cpu().numpy(), scores.float().cpu().numpy()
    recall = []
    for q in range(nq):
        nv = int(ocomp.n_visible(positions[q], 4))
        s = oidx.scores(qd[q], w[q], kd[q_seq[q], :nv])
        scale = max(1.0, float(np.max(np.abs(s)))) if nv else 1.0
        # bf16 round to nearest of an fp32 sum within 1e-5 of the oracle's
        assert np.all(np.abs(g_s[q, :nv] - s) <= 2.0 ** -8 * np.abs(s) + 1e-5 * scale)
        assert np.all(np.isneginf(g_s[q, nv:]))
        assert np.array_equal(g_idx[q], oidx.topk(g_s[q], nv, k))       # exact among bf16 values
        ref = oidx.topk(s, nv, k)
        kk = min(k, nv)
        recall.append(len(np.intersect1d(g_idx[q][:kk], ref[:kk])) / kk)
    assert np.mean(recall) >= 0.9, recall


def test_topk_ties_go_to_lower_index():
    """Many exactly equal scores: the selection must be the lowest indices."""
    v = v4()
    B, N, k = 1, 5000, 100
    keys = np.zeros((B, N, 32), dtype=np.float32)
    keys[0, :, 0] = 1.0                      # every key scores w * q0
    keys[0, 4000:4010, 0] = 2.0              # ten larger ones
    ly = synth.Layer("csa", 4, 16, 512, 64, 128, 1, 32, k, idx_fp4=False)
    desc = desc_for(ly)
    krows, _ = code_rows(desc, dev(keys), v.F32)
    qI = np.zeros((1, 1, 32), dtype=np.float32)
    qI[0, 0, 0] = 1.0
    idx = torch.zeros(1, k, dtype=torch.int32, device="cuda")
    ws = v.workspace(desc, 1, N)
    v.index_topk(desc, qI=dev(qI), w=dev(np.ones((1, 1), np.float32)),
                 q_pos=dev(np.array([4 * N - 1]), torch.int64), keys=krows, key_rows=N, max_vis=N,
                 idx_out=idx, ws=ws, B=1)
    got = idx.cpu().numpy()[0]
    assert list(got) == list(range(90)) + list(range(4000, 4010))


@pytest.mark.parametrize("n_vis,k,mode", [(300000, 1024, "ties"), (300000, 777, "random"),
                                          (262144, 1024, "random"), (70000, 512, "ties"),
                                          (9, 64, "random"), (4096, 2048, "random")])
def test_topk_selection_exact(n_vis, k, mode):
    """The selection alone, fed exact scores through index_topk's F32 path:
    ties spanning the cluster's slices, more keys than the CTAs keep in shared
    memory, k equal to the number of keys, fewer keys than k."""
    v = v4()
    rng = np.random.default_rng(n_vis + k)
    d_I = 32
    keys = np.zeros((1, n_vis, d_I), dtype=np.float32)
    if mode == "ties":
        keys[0, :, 0] = rng.integers(0, 3, n_vis).astype(np.float32)    # massive ties
    else:
        keys[0, :, 0] = rng.standard_normal(n_vis).astype(np.float32) ** 2
    ly = synth.Layer("csa", 4, 16, 512, 64, 128, 1, d_I, min(k, 2048), idx_fp4=False)
    desc = desc_for(ly)
    krows, _ = code_rows(desc, dev(keys), v.F32)
    qI = np.zeros((1, 1, d_I), dtype=np.float32)
    qI[0, 0, 0] = 1.0
    idx = torch.full((1, k), -3, dtype=torch.int32, device="cuda")
    ws = v.workspace(desc, 1, n_vis)
    v.index_topk(desc, qI=dev(qI), w=dev(np.ones((1, 1), np.float32)),
                 q_pos=dev(np.array([4 * n_vis - 1]), torch.int64), keys=krows, key_rows=n_vis,
                 max_vis=n_vis, idx_out=idx, ws=ws, B=1)
    torch.cuda.synchronize()
    s = keys[0, :, 0].astype(np.float64)
    want = oidx.topk(s, n_vis, k)
    assert np.array_equal(idx.cpu().numpy()[0], want)


# ------------------------------------------------------------------ MQA

@pytest.mark.parametrize("sparse", [True, False])
@pytest.mark.parametrize("fp8,H,d,d_rope,q_rmsnorm", [(True, 64, 512, 64, False),
                                                      (True, 128, 512, 64, False),
                                                      (True, 128, 512, 64, True),
                                                      (False, 16, 128, 32, False)])
def test_mqa_parity(sparse, fp8, H, d, d_rope, q_rmsnorm):
    v = v4()
    rng = np.random.default_rng(H + d + sparse)
    m, B, N, n_win, k = (4 if sparse else 128), 3, 700, 128, 96
    ly = synth.Layer("csa" if sparse else "hca", m, H, d, d_rope, n_win, 4, 32, k, kv_fp8=fp8,
                     idx_fp4=False)
    desc = desc_for(ly)
    fmt = v.E4M3_BF16ROPE if fp8 else v.F32
    ents = rng.standard_normal((B, N, d)).astype(np.float32)
    T = m * N + 50
    swa_rows = 256
    swa_vals = rng.standard_normal((B, swa_rows, d)).astype(np.float32)
    kv, kv_sc = code_rows(desc, dev(ents), fmt, d_rope=d_rope)
    swa, swa_sc = code_rows(desc, dev(swa_vals), fmt, d_rope=d_rope)
    positions = np.array([m * N - 1, m * 300 + 1, 5, m * 10, m * N - 2, 200])
    q_seq = np.array([0, 1, 2, 2, 1, 0], dtype=np.int32)
    nq = len(positions)
    Q = synth.bf16_values(rng.standard_normal((nq, H, d)).astype(np.float32))
    if q_rmsnorm:                   # rows far from unit RMS: the normalisation matters
        Q = synth.bf16_values(Q * rng.uniform(0.1, 10.0, (nq, H, 1)).astype(np.float32))
    sink = rng.standard_normal(H).astype(np.float32)
    idx = np.full((nq, k), -1, dtype=np.int32)
    for q in range(nq):
        nv = int(ocomp.n_visible(positions[q], m))
        sel = np.sort(rng.choice(nv, size=min(k, nv), replace=False)) if nv else np.zeros(0, int)
        idx[q, : len(sel)] = sel
    # parity on the fp32 output; the bf16 output is checked to be its rounding
    out = torch.zeros(nq, H, d, dtype=torch.float32, device="cuda")
    lse = torch.zeros(nq, H, dtype=torch.float32, device="cuda")
    ws = v.workspace(desc, nq, N)
    kw = dict(Q=dev(Q, torch.bfloat16), q_pos=dev(positions, torch.int64),
              q_seq=dev(q_seq, torch.int32), B=B, kv=kv, kv_scale=kv_sc, kv_rows=N, swa=swa,
              swa_scale=swa_sc, swa_rows=swa_rows, out=out, ws=ws, sink=dev(sink), lse=lse,
              q_rmsnorm=q_rmsnorm)
    def run(**extra):
        if sparse:
            v.sparse_mqa(desc, idx=dev(idx, torch.int32), **{**kw, **extra})
        else:
            v.dense_mqa(desc, max_vis=N, **{**kw, **extra})
    run()
    torch.cuda.synchronize()
    assert v.device_status(ws) == 0
    if fp8:
        ob = torch.zeros(nq, H, d, dtype=torch.bfloat16, device="cuda")
        run(out=ob)
        torch.cuda.synchronize()
        assert torch.equal(ob, out.to(torch.bfloat16))
    g_out, g_lse = out.float().cpu().numpy(), lse.cpu().numpy()
    e_val = read_kv(kv, kv_sc, fmt, d, d_rope)
    s_val = read_kv(swa, swa_sc, fmt, d, d_rope)
    for q in range(nq):
        p, b = int(positions[q]), int(q_seq[q])
        nv = int(ocomp.n_visible(p, m))
        rows = idx[q][idx[q] >= 0] if sparse else np.arange(nv)
        toks = omqa.window_tokens(p, n_win)
        keys = np.concatenate([e_val[b, rows], s_val[b, toks % swa_rows]], 0)
        o, l = oracle_attention(Q[q], p, keys, sink, ly, fp8, q_rmsnorm=q_rmsnorm)
        check_output(g_out[q], o, g_lse[q], l, not fp8, ("query", q))


@pytest.mark.parametrize("H", [64, 48])
def test_dense_mqa_one_sequence_pairs(H):
    """Dense MQA over many queries of one sequence (the prefill form): the
    tensor-core kernel runs two consecutive queries per CTA (rows 0..63 /
    64..127), each row masked to its own query's entries and window.
    Positions: consecutive runs crossing block boundaries, gaps inside a pair,
    a pair of equal positions, position 0."""
    v = v4()
    rng = np.random.default_rng(H)
    m, N, n_win, d, d_rope = 128, 40, 128, 512, 64
    ly = synth.Layer("hca", m, H, d, d_rope, n_win)
    desc = desc_for(ly)
    fmt = v.E4M3_BF16ROPE
    L = m * N
    ents = rng.standard_normal((1, N, d)).astype(np.float32)
    swa_vals = rng.standard_normal((1, L, d)).astype(np.float32)
    kv, kv_sc = code_rows(desc, dev(ents), fmt, d_rope=d_rope)
    swa, swa_sc = code_rows(desc, dev(swa_vals), fmt, d_rope=d_rope)
    pos = list(range(2 * m - 100, 2 * m + 100)) + [0, 1, 3000, 3000, 4000, 4900, 127, 128]
    pos += sorted(rng.integers(0, L, 256 - len(pos)).tolist())
    positions = np.array(pos[:256])
    nq = len(positions)
    Q = synth.bf16_values(rng.standard_normal((nq, H, d)).astype(np.float32))
    sink = rng.standard_normal(H).astype(np.float32)
    out = torch.zeros(nq, H, d, dtype=torch.float32, device="cuda")
    lse = torch.zeros(nq, H, dtype=torch.float32, device="cuda")
    ws = v.workspace(desc, nq, N)
    v.dense_mqa(desc, Q=dev(Q, torch.bfloat16), q_pos=dev(positions, torch.int64),
                q_seq=dev(np.zeros(nq), torch.int32), B=1, kv=kv, kv_scale=kv_sc, kv_rows=N,
                swa=swa, swa_scale=swa_sc, swa_rows=L, max_vis=N, out=out, ws=ws,
                sink=dev(sink), lse=lse)
    torch.cuda.synchronize()
    assert v.device_status(ws) == 0
    g_out, g_lse = out.cpu().numpy(), lse.cpu().numpy()
    e_val = read_kv(kv, kv_sc, fmt, d, d_rope)
    s_val = read_kv(swa, swa_sc, fmt, d, d_rope)
    for q in range(nq):
        p = int(positions[q])
        nv = int(ocomp.n_visible(p, m))
        toks = omqa.window_tokens(p, n_win)
        keys = np.concatenate([e_val[0, :nv], s_val[0, toks]], 0)
        o, l = oracle_attention(Q[q], p, keys, sink, ly, True)
        check_output(g_out[q], o, g_lse[q], l, False, ("query", q))


def test_mqa_no_sink_and_empty_selection():
    v = v4()
    rng = np.random.default_rng(5)
    ly = synth.Layer("csa", 4, 64, 512, 64, 128, 4, 32, 32)
    desc = desc_for(ly)
    ents = rng.standard_normal((1, 50, 512)).astype(np.float32)
    kv, kv_sc = code_rows(desc, dev(ents), v.E4M3_BF16ROPE)
    swa, swa_sc = code_rows(desc, dev(ents[:, :128 if 50 > 128 else 50]), v.E4M3_BF16ROPE,
                            rows=128)
    Q = synth.bf16_values(rng.standard_normal((1, 64, 512)).astype(np.float32))
    idx = torch.full((1, 32), -1, dtype=torch.int32, device="cuda")     # nothing selected
    out = torch.zeros(1, 64, 512, dtype=torch.float32, device="cuda")
    ws = v.workspace(desc, 1, 50)
    v.sparse_mqa(desc, Q=dev(Q, torch.bfloat16), q_pos=dev(np.array([40]), torch.int64), kv=kv,
                 kv_scale=kv_sc, kv_rows=50, swa=swa, swa_scale=swa_sc, swa_rows=128, idx=idx,
                 out=out, ws=ws, B=1)
    torch.cuda.synchronize()
    ev = read_kv(swa[0], swa_sc[0], v.E4M3_BF16ROPE)
    o, _ = oracle_attention(Q[0], 40, ev[:41], None, ly, True)      # window = tokens 0..40
    check_output(out.float().cpu().numpy()[0], o, None, None, False)


# ------------------------------------------------------------------ decode steps

def _small(kind, L, B):
    base = synth.WORKLOADS["csa_flash_128k" if kind == "csa" else "hca_flash_128k"]
    return synth.scaled(base, B=B, L=L, top_k=64, name=f"small_{kind}")


@pytest.mark.parametrize("kind,L", [("csa", 4 * 3000), ("hca", 128 * 40), ("csa", 4 * 1000 + 2),
                                    ("hca", 128 * 9 + 50)])
def test_decode_step_small(kind, L):
    w = _small(kind, L, 3)
    inp = synth.decode_layer_inputs(w, 0)
    st = DecodeState(w, 0, inp)
    st.step()
    compare_decode(st, [0, 1, 2])
    check_bf16_output_is_rounded_fp32(st)


def test_decode_is_deterministic_and_batch_invariant():
    w = _small("csa", 4 * 2000, 3)
    inp = synth.decode_layer_inputs(w, 0)
    st = DecodeState(w, 0, inp)
    st.step()
    out1, idx1 = st.out.clone(), st.idx.clone()
    st.step()                       # same step again: the appends rewrite the same rows
    assert torch.equal(out1, st.out) and torch.equal(idx1, st.idx)
    # changing another sequence's query leaves sequence 1 bit-identical
    st.Q[0].neg_()
    st.qI[2] = st.qI[0]
    st.step()
    assert torch.equal(out1[1], st.out[1]) and torch.equal(idx1[1], st.idx[1])


# ------------------------------------------------------------------ full-size workloads

def test_tiny_csa_fp32_full():
    """The fp32 CSA layer (L = 8192, 32 queries): projections, pooling of all
    entries and keys, window KV, indexer + top-k, sparse MQA, all in fp32."""
    v = v4()
    w = synth.WORKLOADS["tiny_csa_fp32"]
    ly = w.layers[0]
    inp = synth.tiny_inputs(w)
    ref = pipeline.tiny_layer(inp, w)
    desc = desc_for(ly)
    L, c, cI = w.L, ly.d, ly.d_I
    x = dev(inp["x"])
    Wcat = dev(np.concatenate([inp["W_kv"], inp["W_z"], inp["W_kvI"], inp["W_zI"]], 1))
    CZ = torch.empty(L, Wcat.shape[1], dtype=torch.float32, device="cuda")
    v.project(x, Wcat, CZ)
    ld = CZ.shape[1]
    n_ent = L // 4
    one = lambda val: torch.full((1,), val, dtype=torch.int64, device="cuda")
    ents = torch.zeros(1, n_ent, 4 * c, dtype=torch.uint8, device="cuda")
    v.compress(desc, m=4, overlap=True, c=c, Ca=CZ[:, :c], Za=CZ[:, c:2 * c], Cb=CZ[:, :c],
               Zb=CZ[:, c:2 * c], in_rows=L, in_seq_stride=L * ld, in_row_stride=ld,
               bias=dev(inp["bias"]), seq_len=one(L), entry_begin=one(0), n_entries=n_ent,
               out_dtype=v.F32, out=ents, out_rows=n_ent)
    keys = torch.zeros(1, n_ent, 4 * cI, dtype=torch.uint8, device="cuda")
    v.compress(desc, m=4, overlap=True, c=cI, Ca=CZ[:, 2 * c:2 * c + cI],
               Za=CZ[:, 2 * c + cI:2 * c + 2 * cI], Cb=CZ[:, 2 * c:2 * c + cI],
               Zb=CZ[:, 2 * c + cI:2 * c + 2 * cI], in_rows=L, in_seq_stride=L * ld,
               in_row_stride=ld, bias=dev(inp["ibias"]), seq_len=one(L), entry_begin=one(0),
               n_entries=n_ent, out_dtype=v.F32, out=keys, out_rows=n_ent, apply_rmsnorm=False,
               apply_rope=False)
    swa = torch.zeros(1, L, 4 * c, dtype=torch.uint8, device="cuda")
    v.compress(desc, m=1, overlap=False, c=c, Ca=CZ[:, :c], Za=None, in_rows=L,
               in_seq_stride=L * ld, in_row_stride=ld, seq_len=one(L), entry_begin=one(0),
               n_entries=L, out_dtype=v.F32, out=swa, out_rows=L)
    pos = inp["positions"]
    nq = len(pos)
    xq = x[torch.from_numpy(pos).cuda()]
    Wq = dev(np.concatenate([inp["W_dq"], inp["W_w"], inp["W_q"]], 1))
    QQ = torch.empty(nq, Wq.shape[1], dtype=torch.float32, device="cuda")
    v.project(xq, Wq, QQ)
    r = w.low_rank
    qI = torch.empty(nq, ly.H_I * cI, dtype=torch.float32, device="cuda")
    v.project(QQ[:, :r], dev(inp["W_uq"]), qI)
    wh = QQ[:, r:r + ly.H_I].contiguous()
    Q = QQ[:, r + ly.H_I:].contiguous().reshape(nq, ly.H, c)
    q_pos = dev(pos, torch.int64)
    q_seq = torch.zeros(nq, dtype=torch.int32, device="cuda")
    idx = torch.zeros(nq, ly.top_k, dtype=torch.int32, device="cuda")
    scores = torch.zeros(nq, n_ent, dtype=torch.float32, device="cuda")
    ws = v.workspace(desc, nq, n_ent)
    v.index_topk(desc, qI=qI.reshape(nq, ly.H_I, cI), w=wh, q_pos=q_pos, q_seq=q_seq, B=1,
                 keys=keys, key_rows=n_ent, max_vis=n_ent, idx_out=idx, scores_out=scores, ws=ws)
    out = torch.zeros(nq, ly.H, c, dtype=torch.float32, device="cuda")
    lse = torch.zeros(nq, ly.H, dtype=torch.float32, device="cuda")
    v.sparse_mqa(desc, Q=Q, q_pos=q_pos, q_seq=q_seq, B=1, kv=ents, kv_rows=n_ent, swa=swa,
                 swa_rows=L, idx=idx, out=out, ws=ws, sink=dev(inp["sink"]), lse=lse,
                 q_rmsnorm=True)
    torch.cuda.synchronize()
    assert v.device_status(ws) == 0
    assert np.max(np.abs(ents.cpu().numpy()[0].view(np.float32) - ref["entries"])) <= F32_ABS_TOL
    assert np.max(np.abs(keys.cpu().numpy()[0].view(np.float32) - ref["keys"])) <= F32_ABS_TOL
    assert np.max(np.abs(swa.cpu().numpy()[0].view(np.float32) - ref["swa"])) <= F32_ABS_TOL
    g_idx, g_s, g_o, g_l = (idx.cpu().numpy(), scores.cpu().numpy(), out.cpu().numpy(),
                            lse.cpu().numpy())
    for q in range(nq):
        nv = len(ref["scores"][q])
        s = ref["scores"][q]
        assert np.max(np.abs(g_s[q, :nv] - s)) <= 1e-4 * max(1.0, np.max(np.abs(s)))
        check_topk(g_idx[q], s, nv, ly.top_k)
        # the oracle's attention over the GPU's selection (the same as the
        # oracle's own selection unless the GPU took a legal tie swap)
        p = int(pos[q])
        sel = g_idx[q][g_idx[q] >= 0]
        keys_q = np.concatenate([ref["entries"][sel],
                                 ref["swa"][omqa.window_tokens(p, ly.n_win)]], 0)
        o, l = omqa.attend(ref["q"][q], keys_q, 1 / np.sqrt(ly.d), inp["sink"])
        o = omqa.finish_output(o, p, ly.d_rope, ly.rope_theta)
        check_output(g_o[q], o, g_l[q], l, True, ("query", q))


def _full_decode(name, seqs):
    w = synth.WORKLOADS[name]
    for li in range(len(w.layers)):
        inp = synth.decode_layer_inputs(w, li)
        st = DecodeState(w, li, inp)
        st.step()
        rep = compare_decode(st, seqs)
        check_bf16_output_is_rounded_fp32(st)
        print(name, li, rep)
        del st
        torch.cuda.empty_cache()


def test_full_hca_flash_128k():
    _full_decode("hca_flash_128k", [0, 15])


def test_full_csa_flash_128k():
    _full_decode("csa_flash_128k", [0, 31])


def test_full_pro_pair_1m():
    _full_decode("pro_pair_1m", [0, 3])


# ------------------------------------------------------------------ projection (a0)

@pytest.mark.parametrize("M,N,K,y_bf16", [(300, 700, 200, False), (1024, 3584, 4096, False),
                                          (129, 257, 64, True), (5, 40, 1000, False)])
def test_projection_tensor_core(M, N, K, y_bf16):
    """bf16 x bf16 -> fp32 / bf16 on the tcgen05 GEMM, ragged in every dim
    (partial 128 x 256 tiles, a k tail that the loads zero-fill), against the
    float64 product of the same bf16 values."""
    v = v4()
    rng = np.random.default_rng(M + N + K)
    X = synth.bf16_values(rng.standard_normal((M, K)).astype(np.float32))
    W = synth.bf16_values((rng.standard_normal((K, N)) / np.sqrt(K)).astype(np.float32))
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16 if y_bf16 else torch.float32,
                   device="cuda")
    # row strides of X and W must be multiples of 16 bytes: views of padded buffers
    ldx, ldw = (K + 7) // 8 * 8, (N + 7) // 8 * 8
    Xd = torch.zeros(M, ldx, dtype=torch.bfloat16, device="cuda")
    Wd = torch.zeros(K, ldw, dtype=torch.bfloat16, device="cuda")
    Xd[:, :K] = dev(X, torch.bfloat16)
    Wd[:, :N] = dev(W, torch.bfloat16)
    v.project(Xd[:, :K], Wd[:, :N], Y)
    torch.cuda.synchronize()
    want = X.astype(np.float64) @ W.astype(np.float64)
    got = Y.float().cpu().numpy().astype(np.float64)
    # fp32 accumulation of exact bf16 products over K terms; bf16 output rounding
    tol = (2.0 ** -8 if y_bf16 else 1e-4) * np.maximum(np.abs(want), 1.0)
    assert np.all(np.abs(got - want) <= tol)
