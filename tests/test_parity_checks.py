"""The stage-wise parity checks themselves (tests/parity.py), on the CPU: the
oracle's own codes pass; a code that no value within the float32 error
bound of the oracle's value rounds to, a scale off by a factor of two away
from a scale boundary, or a swap outside the tie tolerance fails; and the
codes a float32 computation may legitimately produce at a rounding midpoint
or at a scale boundary pass."""
import numpy as np
import pytest

from oracle import codecs
from tests import parity


def _rows(n=6, d=512, seed=3):
    return np.random.default_rng(seed).standard_normal((n, d))


def test_oracle_codes_are_valid_e4m3():
    raw = _rows()
    codes, rbits, s = codecs.quantize_kv(raw, 64)
    assert parity.check_e4m3_rows(codes, rbits, s, raw) == 0


def test_a_code_away_from_a_midpoint_is_rejected():
    raw = _rows()
    codes, rbits, s = codecs.quantize_kv(raw, 64)
    # the row's largest element: its neighbour code is far from any valid rounding
    j = int(np.argmax(np.abs(raw[0, :448])))
    bad = codes.copy()
    bad[0, j] = bad[0, j] - 1
    with pytest.raises(AssertionError):
        parity.check_e4m3_rows(bad, rbits, s, raw)
    badr = rbits.copy()
    badr[1, 5] ^= 0x4
    with pytest.raises(AssertionError):
        parity.check_e4m3_rows(codes, badr, s, raw)


def test_a_flip_at_a_rounding_midpoint_is_valid():
    raw = _rows(n=1)
    codes, rbits, s = codecs.quantize_kv(raw, 64)
    sc = float(s[0])
    # place element 3 exactly between two E4M3 grid values (times the scale),
    # nudged by 1e-7: float32 may round it either way
    lo_code = int(codes[0, 3]) & 0x7F
    lo_code = min(lo_code, 0x7D)
    a, b = codecs.E4M3_TABLE[lo_code], codecs.E4M3_TABLE[lo_code + 1]
    raw2 = raw.copy()
    raw2[0, 3] = (0.5 * (a + b)) * sc * (1 + 1e-7)
    c2, r2, s2 = codecs.quantize_kv(raw2, 64)
    assert float(s2[0]) == sc
    other = c2.copy()
    other[0, 3] = lo_code if c2[0, 3] == lo_code + 1 else lo_code + 1
    parity.check_e4m3_rows(other, r2, s2, raw2)          # valid: a midpoint flip
    far = c2.copy()
    far[0, 3] = lo_code + 2
    with pytest.raises(AssertionError):
        parity.check_e4m3_rows(far, r2, s2, raw2)


def test_scale_must_be_the_rule_scale_except_at_a_boundary():
    raw = _rows(n=1)
    codes, rbits, s = codecs.quantize_kv(raw, 64)
    twice = codecs.quantize_kv(raw / 2, 64)[0]           # codes under scale 2 s
    with pytest.raises(AssertionError):
        parity.check_e4m3_rows(twice, rbits, s * 2, raw)
    # amax just above 448 * 2^-5: the rule's scale is 2^-4, but float32 pooling
    # may have seen an amax just below it and chosen 2^-5
    raw_b = raw.copy()
    j = int(np.argmax(np.abs(raw_b[0, :448])))
    raw_b[0, :448] *= (448 * 2.0 ** -5) * (1 + 3e-6) / abs(raw_b[0, j])
    c_rule, r_rule, s_rule = codecs.quantize_kv(raw_b, 64)
    assert float(s_rule[0]) == 2.0 ** -4
    s_alt = np.float32(2.0 ** -5)
    c_alt = codecs.e4m3_encode(np.clip(raw_b[0, :448] / s_alt, -448, 448))[None]
    parity.check_e4m3_rows(c_alt, r_rule, np.array([s_alt]), raw_b)


def test_mxfp4_validity():
    raw = np.random.default_rng(9).standard_normal((5, 128))
    c, sf = codecs.quantize_mxfp4(raw)
    packed = codecs.pack_e2m1(c)
    assert parity.check_mxfp4_rows(packed, sf, raw) == 0
    bad = c.copy()
    j = int(np.argmax(np.abs(raw[2, :32])))
    bad[2, j] = (bad[2, j] & 0x8) | max(0, (bad[2, j] & 7) - 2)
    with pytest.raises(AssertionError):
        parity.check_mxfp4_rows(codecs.pack_e2m1(bad), sf, raw)
    sf2 = sf.copy()
    sf2[1, 2] += 1
    with pytest.raises(AssertionError):
        parity.check_mxfp4_rows(packed, sf2, raw)


def test_topk_check_tie_tolerance():
    s = np.array([5.0, 4.0, 3.0, 2.0, 1.0, 2.0 * (1 - 5e-4)])
    want = np.array([0, 1, 2, 3])
    assert parity.check_topk(want, s, 6, 4) == 0
    # 5 for 3: 5's score is within 1e-3 of the 4th score (2.0)
    assert parity.check_topk(np.array([0, 1, 2, 5]), s, 6, 4) == 1
    with pytest.raises(AssertionError):                 # 4 (score 1.0) is not a tie
        parity.check_topk(np.array([0, 1, 2, 4]), s, 6, 4)
    with pytest.raises(AssertionError):                 # not ascending
        parity.check_topk(np.array([1, 0, 2, 3]), s, 6, 4)
    assert parity.check_topk(np.array([0, 1, -1, -1]), s[:2], 2, 4) == 0
