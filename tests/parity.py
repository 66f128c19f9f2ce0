"""Parity checks of stored codes and of the stages built on them (numpy only,
no GPU needed).

Stored codes.  Both sides quantise with the same rule (E4M3 with a per-row
power-of-two scale and bf16 RoPE dims; MXFP4 with an E8M0 exponent per 32
elements; OCP OFP8 rev 1.0 and OCP MX v1.0 formats), but the kernel pools and
normalises in float32 while the oracle does so in float64, so the value each
side quantises differs by float32 rounding.  A GPU code is therefore *valid*
when it is the round-to-nearest-even code of some value within ``REL`` of the
oracle's value before coding (relative to the larger of the element and the
row's RMS), under a scale that is itself the rule's scale of some amax within
``REL`` of the oracle's.  Away from rounding midpoints and scale boundaries
this is the oracle's code exactly; nothing wider is allowed.

``REL`` = 1e-4 bounds the float32 error of the kernel's pooling: up to 256
window terms summed in float32 (256 * 2^-24 = 1.5e-5 of the weighted sum),
the fast exponentials of the softmax weights (a few ulp), the RMSNorm sum of
squares over 512 channels and its square root, and the RoPE rotation; with
margin for the softmax normalisation, 1e-4.

Stages.  Every later stage is checked on the GPU's own checked output of the
stage before (stage-wise parity): the oracle's indexer scores the keys the GPU
stored, and the oracle's attention runs over the rows the GPU stored and the
entries the GPU selected.  Then the selection must equal the oracle's up to
swaps among keys whose oracle score lies within ``TOPK_REL_TOL`` of the k-th
score, and outputs must be within ``R16_TOL`` (max-abs error over the RMS of
the oracle's output) or ``F32_ABS_TOL`` (fp32 layer), with nothing subtracted.
"""
from __future__ import annotations

import numpy as np

from oracle import codecs

TOPK_REL_TOL = 1e-3
R16_TOL = 2e-2
F32_ABS_TOL = 1e-4
REL = 1e-4
# LSE: the scores are fp32 sums of exact E4M3 x E4M3 (and bf16 x bf16)
# products over 512 dims; on N(0,1)-like rows their rounding error is a few
# 1e-6, and the log-sum-exp moves by at most the largest score error
LSE_ABS_TOL = 1e-3
MAX_FLIP_FRACTION = 0.01


def r16(gpu, ref) -> float:
    """max-abs error over the RMS of the reference."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(gpu - ref)) / np.sqrt(np.mean(ref * ref)))


def _interval(raw, rel=REL):
    """Per-element interval [lo, hi] of values within rel of raw (relative
    to max(|raw|, rms of the row))."""
    raw = np.asarray(raw, dtype=np.float64)
    rms = np.sqrt(np.mean(raw * raw, axis=-1, keepdims=True))
    tol = rel * np.maximum(np.abs(raw), rms)
    return raw - tol, raw + tol


def _between(g, a, b):
    lo, hi = np.minimum(a, b), np.maximum(a, b)
    return (g >= lo) & (g <= hi)


def e4m3_row_violations(codes, rope_bits, scale, raw, d_rope: int, rel: float = REL):
    """Indices of the stored elements of one E4M3 + bf16 row (codes [dn],
    rope_bits [d_rope], scale) that are not a valid coding of ``raw`` [d]
    (the oracle's value before coding), plus whether the scale is valid.
    Returns (scale_ok, bad_element_indices, n_differing_from_oracle)."""
    raw = np.asarray(raw, dtype=np.float64)
    dn = raw.shape[-1] - d_rope
    lo, hi = _interval(raw, rel)
    amax = np.max(np.abs(raw[:dn]))
    tol_a = rel * max(amax, float(np.sqrt(np.mean(raw * raw))))
    s = float(scale)
    s_lo = float(codecs.pow2_scale(max(amax - tol_a, 0.0)))
    s_hi = float(codecs.pow2_scale(amax + tol_a))
    scale_ok = s_lo <= s <= s_hi
    g = codecs.e4m3_decode(codes)
    c_lo = codecs.e4m3_decode(codecs.e4m3_encode(lo[:dn] / s))
    c_hi = codecs.e4m3_decode(codecs.e4m3_encode(hi[:dn] / s))
    ok = _between(g, c_lo, c_hi)
    gr = codecs.bf16_decode(rope_bits)
    r_lo = codecs.bf16_decode(codecs.bf16_encode(lo[dn:]))
    r_hi = codecs.bf16_decode(codecs.bf16_encode(hi[dn:]))
    ok_r = _between(gr, r_lo, r_hi)
    bad = np.concatenate([np.flatnonzero(~ok), dn + np.flatnonzero(~ok_r)])
    oc, orb, osc = codecs.quantize_kv(raw[None], d_rope)
    ndiff = int(np.sum(codecs.e4m3_decode(oc[0]) * float(osc[0]) != g * s) +
                np.sum(orb[0] != np.asarray(rope_bits)))
    return scale_ok, bad, ndiff


def check_e4m3_rows(codes, rope_bits, scales, raw, d_rope: int = 64, what=""):
    """Every row of a stored E4M3 + bf16 block ([n, dn], [n, d_rope], [n])
    is a valid coding of the oracle's rows ``raw`` [n, d], and at most 1 % of
    all elements differ from the oracle's own codes.  (A decoded-value
    tolerance would add nothing: equal codes decode equally, and one valid
    flip at a row's largest element moves it by one E4M3 step, up to 1/8 of
    that element.)"""
    codes = np.asarray(codes).reshape(-1, np.shape(codes)[-1])
    rope_bits = np.asarray(rope_bits).reshape(-1, np.shape(rope_bits)[-1])
    scales = np.asarray(scales, dtype=np.float64).reshape(-1)
    raw = np.asarray(raw, dtype=np.float64).reshape(len(scales), -1)
    nd = 0
    for j in range(len(scales)):
        sok, bad, ndiff = e4m3_row_violations(codes[j], rope_bits[j], scales[j], raw[j], d_rope)
        assert sok, (what, j, "scale", float(scales[j]))
        assert len(bad) == 0, (what, j, "invalid codes at", bad[:8])
        nd += ndiff
    assert nd <= MAX_FLIP_FRACTION * raw.size, (what, "flipped codes", nd, raw.size)
    return nd


def check_mxfp4_rows(packed, sf, raw, what=""):
    """Every row of a stored MXFP4 block (packed E2M1 [n, c/2], E8M0 [n, c/32])
    is a valid coding of ``raw`` [n, c]: each block's exponent is the rule's
    exponent of an amax within REL of the oracle's, each element the RNE E2M1
    code (saturating at 6) of a value within REL of the oracle's.  At most 1 %
    of the elements differ from the oracle's codes."""
    packed = np.asarray(packed)
    c = packed.shape[-1] * 2
    packed = packed.reshape(-1, c // 2)
    sf = np.asarray(sf).reshape(-1, c // 32).astype(np.int64)
    raw = np.asarray(raw, dtype=np.float64).reshape(-1, c)
    lo, hi = _interval(raw)
    g = codecs.e2m1_decode(codecs.unpack_e2m1(packed)).reshape(-1, c // 32, 32)
    X = sf - 127
    rb = raw.reshape(-1, c // 32, 32)
    amax = np.max(np.abs(rb), axis=-1)
    rms = np.sqrt(np.mean(raw * raw, axis=-1, keepdims=True))
    tol_a = REL * np.maximum(amax, rms)
    x_lo = codecs.mx_exponent(np.maximum(amax - tol_a, 0.0))
    x_hi = codecs.mx_exponent(amax + tol_a)
    sok = (X >= x_lo) & (X <= x_hi)
    assert np.all(sok), (what, "block exponents", np.argwhere(~sok)[:8])
    f = np.ldexp(1.0, X)[..., None]
    c_lo = codecs.e2m1_decode(codecs.e2m1_encode(lo.reshape(rb.shape) / f))
    c_hi = codecs.e2m1_decode(codecs.e2m1_encode(hi.reshape(rb.shape) / f))
    ok = _between(g, c_lo, c_hi)
    assert np.all(ok), (what, "invalid codes at", np.argwhere(~ok)[:8])
    oc, osf = codecs.quantize_mxfp4(raw)
    ref = codecs.dequantize_mxfp4(oc, osf)
    nd = int(np.sum(ref != (g * f).reshape(raw.shape)))
    assert nd <= MAX_FLIP_FRACTION * raw.size, (what, "flipped codes", nd, raw.size)
    return nd


def check_topk(gpu_idx, oracle_scores, n_vis, k):
    """GPU selection vs the oracle's scores: ascending, -1 padded, in range,
    and the same set up to swaps among entries whose oracle score is within
    TOPK_REL_TOL relative of the k-th oracle score.  Returns the number of
    swaps."""
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
        assert abs(s[i] - kth) <= TOPK_REL_TOL * abs(kth), (i, s[i], kth)
    return len(diff) // 2
