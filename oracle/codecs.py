"""Number formats of the stored KV, indexer keys and queries (oracle side).

Written from the public format definitions, not from any library:
  * E4M3 (OCP OFP8 rev 1.0): 1 sign, 4 exponent bits (bias 7), 3 mantissa
    bits; subnormals at exponent field 0; S.1111.111 is NaN; max 448; no inf.
  * BF16: the top 16 bits of an IEEE binary32.
  * E2M1 (OCP MX v1.0, FP4): 1 sign, 2 exponent bits (bias 1), 1 mantissa
    bit; magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
  * E8M0 (OCP MX v1.0 scale): 2^(code-127), code 255 is NaN.

Rounding is round-to-nearest-even onto the finite grid with saturation
("satfinite").  Decisions are taken on float32 values (the precision the
kernel holds them in); the power-of-two scalings are exact.

Scale readings (the pages give the formats, not the scale rules):
  R8  FP8 KV / R10 FP8 query: one power-of-two scale per entry (per query
      head), s = 2^ceil(log2(amax / 448)) over the 448 non-RoPE dims;
      amax = 0 gives s = 1.  The RoPE dims are stored as bf16, unscaled.
  R9  MXFP4: per block of 32 elements the shared exponent is
      X = floor(log2(amax)) - 2 (E2M1's largest exponent is 2), clamped to the
      E8M0 range [-127, 127]; amax = 0 gives X = -127.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0


def _e4m3_table() -> np.ndarray:
    t = np.empty(256, dtype=np.float64)
    for c in range(256):
        sign = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        mant = c & 0x7
        if e == 0xF and mant == 0x7:
            t[c] = np.nan
        elif e == 0:
            t[c] = sign * (mant / 8.0) * 2.0 ** -6
        else:
            t[c] = sign * (1.0 + mant / 8.0) * 2.0 ** (e - 7)
    return t


def _e2m1_table() -> np.ndarray:
    t = np.empty(16, dtype=np.float64)
    for c in range(16):
        sign = -1.0 if c & 0x8 else 1.0
        e = (c >> 1) & 0x3
        mant = c & 0x1
        t[c] = sign * ((mant / 2.0) if e == 0 else (1.0 + mant / 2.0) * 2.0 ** (e - 1))
    return t


E4M3_TABLE = _e4m3_table()
E2M1_TABLE = _e2m1_table()


def _rne_to_grid(mag: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index into ascending non-negative ``grid`` nearest to ``mag`` (ties to the
    even index, i.e. the even mantissa); magnitudes above the top saturate."""
    mag = np.minimum(mag, grid[-1])
    hi = np.searchsorted(grid, mag, side="left")          # grid[hi] >= mag
    hi = np.clip(hi, 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    dlo = mag - grid[lo]
    dhi = grid[hi] - mag
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(grid[hi] == mag, hi, idx)
    return idx


def e4m3_decode(codes) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    """float32-valued x -> E4M3 codes (RNE, satfinite; NaN -> 0x7F)."""
    x = np.asarray(x, dtype=np.float64)
    grid = E4M3_TABLE[:127]                      # codes 0..126, ascending, 0..448
    idx = _rne_to_grid(np.abs(np.nan_to_num(x, nan=0.0)), grid).astype(np.uint8)
    # IEEE sign semantics: a negative input that rounds to zero gives -0 (0x80)
    codes = np.where(np.signbit(x), idx | 0x80, idx).astype(np.uint8)
    codes = np.where(np.isnan(x), np.uint8(0x7F), codes)
    return codes


def e2m1_decode(codes) -> np.ndarray:
    return E2M1_TABLE[np.asarray(codes, dtype=np.uint8) & 0xF]


def e2m1_encode(x) -> np.ndarray:
    """float32-valued x -> E2M1 codes (4-bit, one per uint8; RNE, satfinite)."""
    x = np.asarray(x, dtype=np.float64)
    grid = E2M1_TABLE[:8]
    idx = _rne_to_grid(np.abs(x), grid).astype(np.uint8)
    return np.where(np.signbit(x), idx | 0x8, idx).astype(np.uint8)


def e8m0_decode(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.int64)
    return np.where(c == 255, np.nan, np.ldexp(1.0, c - 127))


def bf16_encode(x) -> np.ndarray:
    """float32-valued x -> bf16 bit patterns (uint16), round-to-nearest-even."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    out = np.where(nan, (u >> 16) | 0x40, rounded)
    return out.astype(np.uint16)


def bf16_decode(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f32(x) -> np.ndarray:
    """The float32 value the kernel holds (decision precision)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def pow2_scale(amax, fmax=E4M3_MAX) -> np.ndarray:
    """Smallest power of two s with amax / s <= fmax (s = 1 where amax == 0)."""
    amax = np.asarray(amax, dtype=np.float64)
    safe = np.where(amax > 0, amax, 1.0)
    e = np.ceil(np.log2(safe / fmax))
    # exact fix-up of the log2 guess by direct comparison (powers of two are exact)
    e = np.where(safe / np.ldexp(1.0, e.astype(np.int64)) > fmax, e + 1, e)
    e = np.where(safe / np.ldexp(1.0, (e - 1).astype(np.int64)) <= fmax, e - 1, e)
    s = np.ldexp(1.0, e.astype(np.int64))
    return np.where(amax > 0, s, 1.0)


def quantize_kv(v, d_rope: int):
    """R8: entry vectors [..., d] -> (e4m3 codes [..., d-d_rope] uint8,
    bf16 bits [..., d_rope] uint16, scale [...] float32)."""
    v = f32(v)
    d = v.shape[-1]
    nope, rope = v[..., : d - d_rope], v[..., d - d_rope:]
    amax = np.max(np.abs(nope), axis=-1)
    s = pow2_scale(amax)
    codes = e4m3_encode(nope / s[..., None])
    return codes, bf16_encode(rope), s.astype(np.float32)


def dequantize_kv(codes, rope_bits, scale) -> np.ndarray:
    nope = e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[..., None]
    return np.concatenate([nope, bf16_decode(rope_bits)], axis=-1)


def mx_exponent(amax) -> np.ndarray:
    """R9: shared exponent X = floor(log2 amax) - 2, clamped to [-127, 127]."""
    amax = np.asarray(amax, dtype=np.float64)
    safe = np.where(amax > 0, amax, 1.0)
    _, E = np.frexp(safe)                     # safe = f * 2^E, f in [0.5, 1)
    X = (E - 1) - 2
    X = np.clip(X, -127, 127)
    return np.where(amax > 0, X, -127).astype(np.int64)


def quantize_mxfp4(v):
    """R9: vectors [..., c] (c % 32 == 0) -> (e2m1 codes [..., c] one per
    uint8, e8m0 codes [..., c/32] uint8)."""
    v = f32(v)
    c = v.shape[-1]
    blocks = v.reshape(v.shape[:-1] + (c // 32, 32))
    X = mx_exponent(np.max(np.abs(blocks), axis=-1))
    codes = e2m1_encode(blocks / np.ldexp(1.0, X)[..., None])
    return codes.reshape(v.shape), (X + 127).astype(np.uint8)


def dequantize_mxfp4(codes, sf) -> np.ndarray:
    codes = np.asarray(codes)
    c = codes.shape[-1]
    vals = e2m1_decode(codes).reshape(codes.shape[:-1] + (c // 32, 32))
    return (vals * e8m0_decode(sf)[..., None]).reshape(codes.shape)


def pack_e2m1(codes) -> np.ndarray:
    """Two E2M1 codes per byte: element 2i in the low nibble, 2i+1 in the high."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[..., 0::2] & 0xF) | ((codes[..., 1::2] & 0xF) << 4)


def unpack_e2m1(packed) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out
