"""Helpers shared by the GPU parity tests: moving seeded inputs to the
device, building decode state through the C-ABI, reading stored rows back and
the tolerance checks (from the stated parity bar: top-k sets exact except
swaps within 1e-3 relative of the k-th oracle score; entries and outputs
within max-abs 1e-4 for the fp32 layer and 2e-2 relative-to-RMS for the
FP8/BF16/FP4 layers)."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import codecs

TOPK_REL_TOL = 1e-3
R16_TOL = 2e-2
F32_ABS_TOL = 1e-4


def v4():
    import long_context_compressed_kv_b200 as m
    return m


def dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype).cuda()


def r16(gpu, ref):
    """max-abs error over the RMS of the reference."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(gpu - ref)) / np.sqrt(np.mean(ref * ref)))


def desc_for(ly, kv_fp8=None):
    v = v4()
    fp8 = ly.kv_fp8 if kv_fp8 is None else kv_fp8
    return v.layer_desc(v.CSA if ly.kind == "csa" else v.HCA, ly.m, ly.H, ly.d, ly.d_rope,
                        n_win=ly.n_win, rope_theta=ly.rope_theta, H_I=ly.H_I, d_I=ly.d_I,
                        top_k=ly.top_k, kv_dtype=v.E4M3_BF16ROPE if fp8 else v.F32,
                        idx_dtype=v.MXFP4 if ly.idx_fp4 else v.F32)


def code_rows(desc, vals, fmt, rows=None, first_row=0, d_rope=64):
    """Store fp32 rows [B, n, c] (cuda) in ``fmt`` through compress with m = 1
    (no norm, no RoPE).  Returns (rows [B, out_rows, rb] uint8, scale)."""
    v = v4()
    B, n, c = vals.shape
    out_rows = rows if rows is not None else n
    rb = v.row_bytes(fmt, c, d_rope)
    out = torch.zeros(B, out_rows, rb, dtype=torch.uint8, device="cuda")
    if fmt == v.E4M3_BF16ROPE:
        sc = torch.zeros(B, out_rows, dtype=torch.float32, device="cuda")
    elif fmt == v.MXFP4:
        sc = torch.zeros(B, out_rows, c // 32, dtype=torch.uint8, device="cuda")
    else:
        sc = None
    if n == 0:
        return out, sc
    lens = torch.full((B,), first_row + n, dtype=torch.int64, device="cuda")
    eb = torch.full((B,), first_row, dtype=torch.int64, device="cuda")
    v.compress(desc, m=1, overlap=False, c=c, Ca=vals, Za=None, in_rows=n, in_seq_stride=n * c,
               in_row_stride=c, seq_len=lens, entry_begin=eb, n_entries=n, out_dtype=fmt, out=out,
               out_scale=sc, out_rows=out_rows, apply_rmsnorm=False, apply_rope=False)
    return out, sc


def read_kv(rows, scale, fmt, d=512, d_rope=64):
    """Stored KV rows (numpy uint8 [..., rb]) -> float64 values [..., d]."""
    rows = np.asarray(rows)
    v = v4()
    if fmt == v.F32:
        return rows.view(np.float32).astype(np.float64)
    dn = d - d_rope
    codes = rows[..., :dn]
    rbits = rows[..., dn:].copy().view(np.uint16)
    return codecs.dequantize_kv(codes, rbits, np.asarray(scale))


def read_keys(rows, sf, fmt):
    v = v4()
    rows = np.asarray(rows)
    if fmt == v.F32:
        return rows.view(np.float32).astype(np.float64)
    return codecs.dequantize_mxfp4(codecs.unpack_e2m1(rows), np.asarray(sf))


def check_topk(gpu_idx, oracle_scores, n_vis, k, extra_tol=None):
    """GPU selection vs the oracle: ascending, -1 padded, and the same set up
    to swaps among entries whose oracle score is within 1e-3 relative of the
    k-th oracle score (plus ``extra_tol[i]`` where the two sides' stored keys
    differ by a coding decision).  Returns the number of swaps."""
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    s = np.asarray(oracle_scores, dtype=np.float64)[:n_vis]
    kk = min(k, n_vis)
    sel = gpu_idx[:kk]
    assert np.all(gpu_idx[kk:] == -1), "padding"
    assert np.all(sel >= 0) and np.all(sel < n_vis), "range"
    assert np.all(np.diff(sel) > 0), "ascending, distinct"
    if kk == 0:
        return 0
    order = np.lexsort((np.arange(n_vis), -s))
    want = set(order[:kk].tolist())
    got = set(sel.tolist())
    kth = s[order[kk - 1]]
    diff = want ^ got
    for i in diff:
        tol = TOPK_REL_TOL * abs(kth) + (0.0 if extra_tol is None else extra_tol[i])
        assert abs(s[i] - kth) <= tol, (i, s[i], kth)
    return len(diff) // 2


def check_coded_row(got, ref, ref_raw, d_rope=64, what=""):
    """One stored E4M3 + bf16 row against the oracle's coded row.  Codes may
    differ only where the two sides took a rounding decision differently: the
    oracle's value before coding lies within 1e-4 relative of the midpoint of
    the two decoded values (fp32 pooling against fp64 pooling), and such
    flips are rare; a changed power-of-two scale is allowed only when the
    oracle's amax / 448 lies within 1e-4 (log2) of a power of two."""
    got, ref, raw = (np.asarray(a, dtype=np.float64) for a in (got, ref, ref_raw))
    if r16(got, ref) <= R16_TOL:
        return
    dn = len(raw) - d_rope
    t = np.max(np.abs(raw[:dn])) / codecs.E4M3_MAX
    if t > 0 and abs(np.log2(t) - np.round(np.log2(t))) < 1e-4:
        assert r16(got, ref) <= 8 * R16_TOL, (what, "scale boundary", r16(got, ref))
        return
    d = got != ref
    mid = 0.5 * (got + ref)
    near = np.abs(raw - mid) <= 1e-4 * np.maximum(np.abs(raw), 1e-6)
    assert np.all(near[d]), (what, "code differs away from a rounding midpoint",
                             np.flatnonzero(d & ~near)[:8])
    assert d.mean() < 0.01, (what, "too many flipped codes", int(d.sum()))


def coding_bound(keys_ref, keys_gpu, a, q, o, scale, d_rope=64):
    """First-order bound on how much the MQA output of one query moves when
    its key rows change from the oracle's codes (keys_ref [n, d]) to the
    codes the GPU stored (keys_gpu), both valid roundings of nearly equal
    values: |do_h| <= sum_j a_hj |dk_j| + sum_j a_hj |k_j - o_h| scale |q_h . dk_j|
    (V = K), with a [H, n] the oracle's attention weights and o [H, d] its
    output before the inverse RoPE.  The RoPE dims are rotated afterwards, so
    a pair gets the larger bound of its two dims times sqrt(2).  [H, d]."""
    dk = np.asarray(keys_gpu, np.float64) - np.asarray(keys_ref, np.float64)
    rows = np.flatnonzero(np.any(dk != 0, axis=1))
    b = np.zeros_like(np.asarray(o, np.float64))
    if len(rows) == 0:
        return b
    dk, kr, ar = dk[rows], np.asarray(keys_ref, np.float64)[rows], np.asarray(a)[:, rows]
    ds = scale * np.abs(np.asarray(q, np.float64) @ dk.T)                 # [H, m]
    b = ar @ np.abs(dk) + np.einsum("hm,hmd->hd", ar * ds, np.abs(kr[None] - o[:, None, :]))
    dn = b.shape[1] - d_rope
    pair = np.maximum(b[:, dn::2], b[:, dn + 1::2]) * np.sqrt(2.0)
    b[:, dn::2] = pair
    b[:, dn + 1::2] = pair
    return b


def r16_excess(got, ref, bound):
    """max(|got - ref| - bound, 0) over the RMS of ref."""
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.maximum(np.abs(got - ref) - bound, 0.0)) / np.sqrt(np.mean(ref * ref)))


class DecodeState:
    """The decode layer exactly as bench.py builds and times it (coded synthetic
    history, window ring, tail rings, queries), plus what the checks need."""

    def __init__(self, w, li, inp, in_dtype=torch.float32):
        from bench import build_decode_layer
        self.ly, self.inp, self.B = w.layers[li], inp, w.B
        self.lay = build_decode_layer(w, li, inp, in_dtype)
        lay = self.lay
        self.desc, self.fmt, self.csa = lay.desc, lay.fmt, lay.csa
        self.kv, self.kv_scale, self.swa, self.swa_scale = lay.kv, lay.kv_scale, lay.swa, lay.swa_scale
        self.swa_rows, self.out, self.lse, self.ws, self.Q = lay.swa_rows, lay.out, lay.lse, lay.ws, lay.Q
        self.max_vis = lay.max_vis
        if self.csa:
            self.kfmt, self.keys, self.keys_sf = lay.kfmt, lay.keys, lay.keys_sf
            self.idx, self.qI = lay.idx, lay.qI

    def step(self, stream=None):
        self.lay.step(self.max_vis, stream=stream)


def compare_decode(st: DecodeState, ref: dict, seqs, strict_keys=True):
    """Check one decode step of ``seqs`` against ``oracle.pipeline.decode_layer``."""
    v = v4()
    ly, p = st.ly, st.inp["p"]
    torch.cuda.synchronize()
    assert v.device_status(st.ws) == 0
    i_new = (p + 1) // ly.m - 1
    complete = (p + 1) % ly.m == 0
    report = {}
    for n, b in enumerate(seqs):
        if complete:
            row = st.kv[b, i_new].cpu().numpy()
            sc = None if st.kv_scale is None else st.kv_scale[b, i_new].cpu().numpy()
            got = read_kv(row, sc, st.fmt, ly.d, ly.d_rope)
            err = r16(got, ref["entry_new_val"][n])
            assert err <= R16_TOL, ("new entry", b, err)
        srow = st.swa[b, p % st.swa_rows].cpu().numpy()
        ssc = None if st.swa_scale is None else st.swa_scale[b, p % st.swa_rows].cpu().numpy()
        assert r16(read_kv(srow, ssc, st.fmt, ly.d, ly.d_rope), ref["swa_new_val"][n]) <= R16_TOL
        extra = None
        if st.csa:
            if complete:
                krow = st.keys[b, i_new].cpu().numpy()
                ksf = None if st.keys_sf is None else st.keys_sf[b, i_new].cpu().numpy()
                kgot = read_keys(krow, ksf, st.kfmt)
                kref = ref["key_new_val"][n]
                assert r16(kgot, kref) <= R16_TOL
                if not np.array_equal(kgot, kref):
                    # a coding decision taken differently on the two sides (values
                    # within fp32 rounding of a grid midpoint): bound its effect
                    from oracle import codecs as C
                    qv = C.dequantize_mxfp4(*C.quantize_mxfp4(st.inp["qI"][b])) \
                        if ly.idx_fp4 else st.inp["qI"][b]
                    bound = float(np.abs(qv) @ np.abs(kgot - kref) @ st.inp["w"][b])
                    extra = np.zeros(len(ref["scores"][n]))
                    extra[i_new] = bound
            nsw = check_topk(st.idx[b].cpu().numpy(), ref["scores"][n], (p + 1) // ly.m,
                             ly.top_k, extra)
            report.setdefault("swaps", []).append(nsw)
        got = st.out[b].float().cpu().numpy()
        err = r16(got, ref["out"][n])
        report.setdefault("out_r16", []).append(err)
        assert err <= R16_TOL, ("out", b, err)
        lse_err = np.max(np.abs(st.lse[b].cpu().numpy() - ref["lse"][n]))
        assert lse_err <= 5e-2, ("lse", b, lse_err)
    return report
