"""Pins for the oracle's MXFP4 format and quantiser (CPU only).

Each check reaches the expected value without the oracle function it tests:
hand-derived tables and worked blocks (tests/golden), exact rational brute
force over every bf16 bit pattern, closed forms at power-of-two boundaries,
idempotence and the rounding-error bound.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import mxfp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
MAGS = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
        Fraction(4), Fraction(6)]


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _bf16_bits(v: float) -> int:
    b = int(np.array([v], np.float32).view(np.uint32)[0])
    assert (b & 0xFFFF) == 0, f"{v} is not a bf16 value"
    return b >> 16


def test_e2m1_table_golden():
    rows = _rows("e2m1_codes.txt")
    assert len(rows) == 16
    for code, val in rows:
        got = mxfp4.decode_e2m1(int(code))
        want = float(val)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), (code, got, want)


def test_e8m0_table_golden():
    for byte, val in _rows("e8m0_bytes.txt"):
        got = float(mxfp4.decode_e8m0(int(byte)))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val), (byte, got, val)
            assert got == 2.0 ** (int(byte) - 127)


def test_worked_blocks_golden():
    blocks = {}
    for name, val, code, sbyte in _rows("quant_blocks.txt"):
        blocks.setdefault(name, []).append((float(val), int(code), int(sbyte)))
    for name, items in blocks.items():
        vals = [v for v, _, _ in items] + [0.0] * (32 - len(items))
        bits = np.array([[_bf16_bits(v) for v in vals]], dtype=np.uint16)
        codes, scales = mxfp4.quantize(bits)
        nib = mxfp4.unpack_codes(codes)[0]
        assert int(scales[0, 0]) == items[0][2], name
        for j, (_, c, _) in enumerate(items):
            assert int(nib[j]) == c, (name, j, items[j], int(nib[j]))
        assert all(int(n) == 0 for n in nib[len(items):])


def _floor_log2_from_bits(b: int) -> int:
    """floor(log2 |w|) of a finite nonzero bf16 pattern, from its exponent/mantissa fields."""
    e, m = (b >> 7) & 0xFF, b & 0x7F
    if e:
        return e - 127
    return m.bit_length() - 1 - 133  # subnormal: value = m * 2^-133


def _bf16_fraction(b: int) -> Fraction:
    e, m, s = (b >> 7) & 0xFF, b & 0x7F, -1 if b & 0x8000 else 1
    if e == 0:
        return s * Fraction(m, 2 ** 133)
    return s * Fraction(128 + m, 128) * Fraction(2) ** (e - 127)


def _brute_code(p: Fraction, s: int, negative: bool) -> int:
    v = abs(p) / Fraction(2) ** s
    dists = [abs(v - m) for m in MAGS]
    best = min(dists)
    cands = [i for i, d in enumerate(dists) if d == best]
    mag = cands[0] if len(cands) == 1 else [i for i in cands if i % 2 == 0][0]
    return (8 if negative else 0) | mag


def test_quantize_every_bf16_as_block_max():
    """Block [p, 0, ..., 0] for all 65,536 patterns: scale and code by exact brute force."""
    pats = np.arange(65536, dtype=np.uint32)
    bits = np.zeros((65536, 32), dtype=np.uint16)
    bits[:, 0] = pats
    codes, scales = mxfp4.quantize(bits)
    nib0 = codes[:, 0] & 0x0F
    for b in range(65536):
        e = (b >> 7) & 0xFF
        if e == 0xFF:  # inf / nan
            assert scales[b, 0] == 255 and codes[b].max() == 0, hex(b)
            continue
        frac = _bf16_fraction(b)
        if frac == 0:
            assert scales[b, 0] == 0 and nib0[b] == (8 if b & 0x8000 else 0), hex(b)
            continue
        s = max(_floor_log2_from_bits(b) - 2, -127)
        assert scales[b, 0] == s + 127, hex(b)
        assert nib0[b] == _brute_code(frac, s, bool(b & 0x8000)), hex(b)


@pytest.mark.parametrize("amax", [1.0, 6.0 * 2.0 ** 10, 1.5 * 2.0 ** -120, 2.0 ** -125])
def test_quantize_every_smaller_bf16_under_fixed_max(amax):
    """Block [amax, p, 0...] for every finite p with |p| <= amax (exact brute force)."""
    abits = _bf16_bits(amax)
    pats = [b for b in range(65536) if ((b >> 7) & 0xFF) != 0xFF
            and abs(_bf16_fraction(b)) <= Fraction(amax)]
    bits = np.zeros((len(pats), 32), dtype=np.uint16)
    bits[:, 0] = abits
    bits[:, 1] = pats
    codes, scales = mxfp4.quantize(bits)
    s = max(_floor_log2_from_bits(abits) - 2, -127)
    assert (scales[:, 0] == s + 127).all()
    got = codes[:, 0] >> 4  # element 1 sits in the high nibble of byte 0
    for i, b in enumerate(pats):
        assert got[i] == _brute_code(_bf16_fraction(b), s, bool(b & 0x8000)), (amax, hex(b))


@pytest.mark.parametrize("n", [-133, -126, -100, -7, -1, 0, 1, 5, 20, 127])
def test_scale_at_power_of_two_boundaries(n):
    """amax = 2^n gives s = n-2; the largest bf16 below 2^n gives s = n-3 (clamped at -127)."""
    def one(v):
        b = np.zeros((1, 32), np.uint16)
        b[0, 0] = _bf16_bits(v)
        return int(mxfp4.quantize(b)[1][0, 0]) - 127
    assert one(2.0 ** n) == max(n - 2, -127)
    below = float(np.nextafter(np.float32(2.0 ** n), np.float32(0)))
    below = float(mxfp4.bf16_to_f64(np.array([_bf16_bits_trunc(below)], np.uint16))[0])
    assert below < 2.0 ** n
    assert one(below) == max(n - 3, -127)


def _bf16_bits_trunc(v: float) -> int:
    return int(np.array([v], np.float32).view(np.uint32)[0]) >> 16


def test_idempotent_on_random_blocks():
    rng = np.random.default_rng(1)
    w = rng.standard_normal((64, 256)).astype(np.float32) * np.float32(0.02)
    w[3] *= np.float32(2.0 ** -120)  # tiny blocks: scale clamps
    bits = (w.view(np.uint32) >> 16).astype(np.uint16)
    codes, scales = mxfp4.quantize(bits)
    deq = mxfp4.dequantize(codes, scales)
    back = (deq.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert (mxfp4.bf16_to_f64(back) == deq).all()  # decoded values are bf16-exact
    c2, s2 = mxfp4.quantize(back)
    assert (c2 == codes).all() and (s2 == scales).all()


def test_rounding_error_bound():
    rng = np.random.default_rng(2)
    w = (rng.standard_normal((128, 512)) * 0.02).astype(np.float32)
    bits = (w.view(np.uint32) >> 16).astype(np.uint16)
    wv = mxfp4.bf16_to_f64(bits)
    codes, scales = mxfp4.quantize(bits)
    err = np.abs(mxfp4.dequantize(codes, scales) - wv).reshape(128, 16, 32)
    s = (scales.astype(np.float64) - 127)[..., None]
    v = np.abs(wv.reshape(128, 16, 32)) / 2.0 ** s
    half_gap = np.select([v < 2, v < 4, v < 6], [0.25, 0.5, 1.0], 2.0) * 2.0 ** s
    assert (err <= half_gap).all()
    assert (v.max(axis=-1) >= 4).all() and (v.max(axis=-1) < 8).all()


def test_pack_roundtrip_and_nibble_order():
    codes = np.array([[0x21, 0xF8]], np.uint8)
    nib = mxfp4.unpack_codes(codes)
    assert nib.tolist() == [[1, 2, 8, 15]]
    assert (mxfp4.pack_codes(nib) == codes).all()
