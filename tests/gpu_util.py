"""Helpers shared by the GPU parity tests: moving seeded inputs to the
device, building decode state through the C-ABI, reading stored rows back,
and the stage-wise checks (tests/parity.py states the tolerances and why).

Stage-wise: every stage is checked on the GPU's own checked output of the
stage before.  Stored rows (entries, indexer keys, window KV) are checked as
valid codings of the oracle's values; then the oracle's indexer scores the
keys the GPU stored, and the oracle's attention runs over the rows the GPU
stored and the entries the GPU selected."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import codecs, indexer as oidx, mqa as omqa, pipeline
from tests.parity import (F32_ABS_TOL, LSE_ABS_TOL, R16_TOL, TOPK_REL_TOL, check_e4m3_rows,
                          check_mxfp4_rows, check_topk, r16)

__all__ = ["F32_ABS_TOL", "LSE_ABS_TOL", "R16_TOL", "TOPK_REL_TOL", "check_topk", "r16", "v4",
           "dev", "desc_for", "code_rows", "read_kv", "read_keys", "check_stored_kv",
           "check_stored_keys", "oracle_attention", "check_output", "DecodeState",
           "compare_decode", "check_bf16_output_is_rounded_fp32"]


def v4():
    import long_context_compressed_kv_b200 as m
    return m


def dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype).cuda()


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


def _np(x):
    return x.cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x)


def read_kv(rows, scale, fmt, d=512, d_rope=64):
    """Stored KV rows (uint8 [..., rb]) -> float64 values [..., d]."""
    rows = _np(rows)
    v = v4()
    if fmt == v.F32:
        return rows.view(np.float32).astype(np.float64)
    dn = d - d_rope
    codes = rows[..., :dn]
    rbits = rows[..., dn:].copy().view(np.uint16)
    return codecs.dequantize_kv(codes, rbits, _np(scale))


def read_keys(rows, sf, fmt):
    v = v4()
    rows = _np(rows)
    if fmt == v.F32:
        return rows.view(np.float32).astype(np.float64)
    return codecs.dequantize_mxfp4(codecs.unpack_e2m1(rows), _np(sf))


def check_stored_kv(rows, scale, fmt, raw, d=512, d_rope=64, what=""):
    """Stored KV rows [n, rb] (+ scales [n]) against the oracle's values before
    coding raw [n, d]: valid codings (E4M3 + bf16), or within F32_ABS_TOL (fp32)."""
    v = v4()
    rows = _np(rows).reshape(-1, _np(rows).shape[-1])
    raw = np.asarray(raw, dtype=np.float64).reshape(len(rows), -1)
    if fmt == v.F32:
        got = rows.view(np.float32).astype(np.float64)
        assert np.max(np.abs(got - raw)) <= F32_ABS_TOL, (what, np.max(np.abs(got - raw)))
        return 0
    dn = d - d_rope
    return check_e4m3_rows(rows[:, :dn], rows[:, dn:].copy().view(np.uint16),
                           _np(scale).reshape(-1), raw, d_rope, what)


def check_stored_keys(rows, sf, fmt, raw, what=""):
    """Stored indexer keys [n, rb] (+ E8M0 [n, c/32]) against raw [n, c]."""
    v = v4()
    rows = _np(rows).reshape(-1, _np(rows).shape[-1])
    raw = np.asarray(raw, dtype=np.float64).reshape(len(rows), -1)
    if fmt == v.F32:
        got = rows.view(np.float32).astype(np.float64)
        assert np.max(np.abs(got - raw)) <= F32_ABS_TOL, (what, np.max(np.abs(got - raw)))
        return 0
    return check_mxfp4_rows(rows, _np(sf), raw, what)


def oracle_attention(Q_h, p, keys, sink, ly, fp8, q_rmsnorm=False):
    """The oracle's attention of one query (raw Q [H, d]) at position p over
    the given key rows (the GPU's stored rows, decoded): (out [H, d], lse [H])."""
    q = omqa.prepare_query(Q_h, p, ly.d_rope, ly.rope_theta, fp8, apply_rmsnorm=q_rmsnorm)
    o, lse = omqa.attend(q, keys, 1.0 / np.sqrt(ly.d), sink)
    return omqa.finish_output(o, p, ly.d_rope, ly.rope_theta), lse


def check_output(got, want, lse_got, lse_want, fp32, what=""):
    if fp32:
        err = float(np.max(np.abs(np.asarray(got, np.float64) - want)))
        assert err <= F32_ABS_TOL, (what, "out", err)
    else:
        err = r16(got, want)
        assert err <= R16_TOL, (what, "out", err)
    if lse_got is not None:
        le = float(np.max(np.abs(np.asarray(lse_got, np.float64) - lse_want)))
        assert le <= LSE_ABS_TOL, (what, "lse", le)
    return err


class DecodeState:
    """The decode layer as bench.py builds and times it (coded synthetic
    history, window ring, tail rings, queries), plus what the checks need.
    Parity is checked on the kernels' fp32 output (out_dtype float32): the
    bf16 output bench.py times is that value rounded to nearest even, which
    ``check_bf16_output_is_rounded_fp32`` checks bit-exactly.  (Rounding the
    output to bf16 alone moves max-abs / RMS by up to 2^-9 max|o| / rms(o),
    0.014 on N(0,1) rows where heads differ in peakiness.)"""

    def __init__(self, w, li, inp, in_dtype=torch.float32, out_dtype=torch.float32):
        from bench import build_decode_layer
        self.ly, self.inp, self.B = w.layers[li], inp, w.B
        self.lay = build_decode_layer(w, li, inp, in_dtype, out_dtype)
        lay = self.lay
        self.desc, self.fmt, self.csa = lay.desc, lay.fmt, lay.csa
        self.kv, self.kv_scale, self.swa, self.swa_scale = lay.kv, lay.kv_scale, lay.swa, lay.swa_scale
        self.swa_rows, self.out, self.lse, self.ws, self.Q = lay.swa_rows, lay.out, lay.lse, lay.ws, lay.Q
        self.max_vis = lay.max_vis
        if self.csa:
            self.kfmt, self.keys, self.keys_sf = lay.kfmt, lay.keys, lay.keys_sf
            self.idx, self.qI, self.qI_sf, self.w = lay.idx, lay.qI, lay.qI_sf, lay.w

    def step(self, stream=None):
        self.lay.step(self.max_vis, stream=stream)


def check_bf16_output_is_rounded_fp32(st: DecodeState):
    """The same step with a bf16 output tensor gives exactly the bf16 rounding
    (to nearest even) of the fp32 output (the step is idempotent: its appends
    rewrite the same rows)."""
    f32 = st.lay.out.clone()
    st.lay.out = torch.zeros(f32.shape, dtype=torch.bfloat16, device=f32.device)
    st.step()
    torch.cuda.synchronize()
    got = st.lay.out
    st.lay.out = f32
    assert torch.equal(got, f32.to(torch.bfloat16))


def compare_decode(st: DecodeState, seqs):
    """Stage-wise check of one decode step of sequences ``seqs``:
      a1  the new window row, and on a block boundary the new entry (and the
          new indexer key), are valid codings of the oracle's values
          (``oracle.pipeline.decode_layer``);
      a3  the oracle's scores of the keys the GPU stored, with the indexer
          query the GPU stored, select what the GPU selected (a4);
      a6  the oracle's attention over the rows the GPU stored (the selected /
          visible entries and the window tokens) gives the GPU's output and LSE."""
    v = v4()
    ly, inp = st.ly, st.inp
    p = inp["p"]
    torch.cuda.synchronize()
    assert v.device_status(st.ws) == 0
    ref = pipeline.decode_layer(inp, ly, seqs)
    n_vis = (p + 1) // ly.m
    i_new = n_vis - 1
    complete = (p + 1) % ly.m == 0
    fp32 = st.fmt == v.F32
    report = {"out_err": [], "swaps": []}
    for n, b in enumerate(seqs):
        sr = p % st.swa_rows
        check_stored_kv(st.swa[b, sr:sr + 1], None if fp32 else st.swa_scale[b, sr:sr + 1],
                        st.fmt, ref["swa_new_raw"][n][None], ly.d, ly.d_rope, ("window row", b))
        if complete:
            check_stored_kv(st.kv[b, i_new:i_new + 1],
                            None if fp32 else st.kv_scale[b, i_new:i_new + 1], st.fmt,
                            ref["entry_new_raw"][n][None], ly.d, ly.d_rope, ("new entry", b))
        if st.csa:
            if complete:
                check_stored_keys(st.keys[b, i_new:i_new + 1],
                                  None if st.keys_sf is None else st.keys_sf[b, i_new:i_new + 1],
                                  st.kfmt, ref["key_new_raw"][n][None], ("new key", b))
            kv = read_keys(st.keys[b, :n_vis], None if st.keys_sf is None
                           else st.keys_sf[b, :n_vis], st.kfmt)
            qv = read_keys(st.qI[b], None if st.qI_sf is None else st.qI_sf[b], st.kfmt)
            s = oidx.scores(qv, _np(st.w[b]), kv)
            gidx = _np(st.idx[b])
            report["swaps"].append(check_topk(gidx, s, n_vis, ly.top_k))
            sel = gidx[gidx >= 0]
        else:
            sel = np.arange(n_vis)
        ent = read_kv(st.kv[b][torch.from_numpy(sel).long().cuda()],
                      None if fp32 else st.kv_scale[b][torch.from_numpy(sel).long().cuda()],
                      st.fmt, ly.d, ly.d_rope)
        toks = omqa.window_tokens(p, ly.n_win)
        rr = torch.from_numpy(toks % st.swa_rows).long().cuda()
        win = read_kv(st.swa[b][rr], None if fp32 else st.swa_scale[b][rr], st.fmt, ly.d,
                      ly.d_rope)
        o, lse = oracle_attention(inp["Q"][b], p, np.concatenate([ent, win], 0), inp["sink"], ly,
                                  ly.kv_fp8)
        report["out_err"].append(check_output(_np(st.out[b].float()), o, _np(st.lse[b]), lse,
                                              fp32, ("output", b)))
    return report
