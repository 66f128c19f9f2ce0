"""Pins of the oracle's number formats against the format definitions (golden
tables from the OCP specifications), an independent library (torch's
float8_e4m3fn and bfloat16 casts on the CPU) and exact brute force."""
import os

import numpy as np
import pytest
import torch

from oracle import codecs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    rows = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append(line.split())
    return rows


def test_e2m1_table_matches_ocp():
    for code, val in _read("e2m1_values.txt"):
        got = codecs.e2m1_decode(np.uint8(int(code)))
        assert got == float(val) and np.signbit(got) == np.signbit(float(val)), (code, got, val)


def test_e2m1_rounding_ties_and_saturation():
    for x, want in _read("e2m1_rne_ties.txt"):
        code = codecs.e2m1_encode(np.float64(float(x)))
        got = codecs.e2m1_decode(code)
        assert got == float(want) and np.signbit(got) == np.signbit(float(want)), (x, got, want)


def test_e4m3_special_values():
    for code, val in _read("e4m3_special.txt"):
        got = codecs.e4m3_decode(np.uint8(int(code, 16)))
        if val == "nan":
            assert np.isnan(got)
        else:
            assert got == float(val) and np.signbit(got) == np.signbit(float(val))


def test_e4m3_decode_matches_torch_exhaustively():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = codecs.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000) * 30,
        rng.uniform(-448, 448, 20000),
        rng.standard_normal(5000) * 1e-2,
        # every midpoint between neighbouring finite codes (the tie cases)
        (codecs.E4M3_TABLE[:126] + codecs.E4M3_TABLE[1:127]) / 2,
        -(codecs.E4M3_TABLE[:126] + codecs.E4M3_TABLE[1:127]) / 2,
        codecs.E4M3_TABLE[:127],
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = codecs.e4m3_encode(x.astype(np.float64))
    # torch gives +0 for negative values that round to zero only if the input is +0
    assert np.array_equal(codecs.e4m3_decode(ref), codecs.e4m3_decode(got))
    assert np.array_equal(ref, got)


def test_e4m3_saturates():
    got = codecs.e4m3_decode(codecs.e4m3_encode(np.array([449.0, 464.0, 1e6, -1e6])))
    assert np.array_equal(got, [448.0, 448.0, 448.0, -448.0])


def test_bf16_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(50000) * 10, rng.standard_normal(1000) * 1e-30,
                        rng.uniform(-1e30, 1e30, 1000)]).astype(np.float32)
    # exact ties: low 16 bits 0x8000
    u = rng.integers(0, 2 ** 31, 2000, dtype=np.uint32) & 0xFFFF0000 | 0x8000
    u = u & 0x7F7FFFFF
    x = np.concatenate([x, u.view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(codecs.bf16_encode(x), ref)
    assert np.array_equal(codecs.bf16_decode(ref),
                          torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy())


def test_pow2_scale_definition():
    rng = np.random.default_rng(2)
    amax = np.concatenate([np.exp(rng.uniform(-30, 30, 5000)), 448.0 * 2.0 ** np.arange(-20, 20),
                           448.0 * 2.0 ** np.arange(-20, 20) * (1 + 2 ** -40)])
    s = codecs.pow2_scale(amax)
    m, e = np.frexp(s)
    assert np.all(m == 0.5)                     # a power of two
    assert np.all(amax / s <= 448.0)            # fits
    assert np.all(amax / (s / 2) > 448.0)       # smallest such
    assert codecs.pow2_scale(0.0) == 1.0


def test_mx_exponent_definition():
    rng = np.random.default_rng(3)
    amax = np.exp(rng.uniform(-40, 40, 5000))
    X = codecs.mx_exponent(amax)
    # floor(log2 amax) = X + 2 exactly: 2^(X+2) <= amax < 2^(X+3)
    assert np.all(np.ldexp(1.0, X + 2) <= amax) and np.all(amax < np.ldexp(1.0, X + 3))
    assert codecs.mx_exponent(0.0) == -127
    assert codecs.mx_exponent(2.0 ** -200) == -127
    assert codecs.mx_exponent(2.0 ** 200) == 127


def test_mxfp4_roundtrip_of_representable_values():
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 16, (64, 128)).astype(np.uint8)
    codes[:, 0] = 7                      # each block's amax is 6 * 2^X exactly
    codes[:, 32] = 7
    codes[:, 64] = 15
    codes[:, 96] = 7
    X = rng.integers(-10, 10, (64, 4))
    vals = codecs.e2m1_decode(codes).reshape(64, 4, 32) * np.ldexp(1.0, X)[..., None]
    vals = vals.reshape(64, 128)
    c2, sf = codecs.quantize_mxfp4(vals)
    assert np.array_equal(codecs.dequantize_mxfp4(c2, sf), vals)
    assert np.array_equal(sf.astype(np.int64) - 127, X)


def test_mxfp4_error_bound():
    """Within the grid an element is off by at most half the widest gap (the
    4 -> 6 gap, 2 * 2^X); above 6 * 2^X it saturates to exactly +-6 * 2^X."""
    rng = np.random.default_rng(5)
    v = codecs.f32(rng.standard_normal((200, 128)))
    codes, sf = codecs.quantize_mxfp4(v)
    dq = codecs.dequantize_mxfp4(codes, sf)
    unit = np.repeat(np.ldexp(1.0, sf.astype(np.int64) - 127), 32, axis=-1)
    sat = np.abs(v) > 6 * unit
    assert np.all(np.abs(dq - v)[~sat] <= unit[~sat])
    assert np.array_equal(dq[sat], np.sign(v[sat]) * 6 * unit[sat])
    assert sat.any()


def test_pack_unpack():
    rng = np.random.default_rng(6)
    codes = rng.integers(0, 16, (7, 128)).astype(np.uint8)
    packed = codecs.pack_e2m1(codes)
    assert packed.shape == (7, 64)
    assert np.array_equal(codecs.unpack_e2m1(packed), codes)
    assert packed[0, 0] == (codes[0, 0] | (codes[0, 1] << 4))


def test_quantize_kv_layout():
    rng = np.random.default_rng(7)
    v = rng.standard_normal((50, 512)) * 3
    codes, rbits, s = codecs.quantize_kv(v, 64)
    assert codes.shape == (50, 448) and rbits.shape == (50, 64) and s.shape == (50,)
    dq = codecs.dequantize_kv(codes, rbits, s)
    # rope dims are exactly the bf16 rounding; nope dims within e4m3 relative step
    assert np.array_equal(dq[:, 448:], codecs.bf16_decode(codecs.bf16_encode(v[:, 448:])))
    rel = np.abs(dq[:, :448] - v[:, :448]) / np.maximum(np.abs(v[:, :448]), 2 ** -6 * s[:, None])
    assert np.max(rel) <= 2 ** -4 + 1e-9
    assert np.all(np.max(np.abs(codecs.e4m3_decode(codes)), axis=1) <= 448)
