"""MXFP4 in fp64: E2M1 element codes, E8M0 block scales, reference quantiser.

Format (OCP Microscaling v1.0, MXFP4; named by the MiMo/TileRT pages, bjdmk.com.cn
news, section "极致协同，通向千速之路": 4 bits per expert parameter):

* a block is 32 consecutive elements along the contraction dimension K;
* each element is an E2M1 code: bit 3 sign, bits 2..0 magnitude index into
  {0, 0.5, 1, 1.5, 2, 3, 4, 6};
* the block shares one E8M0 scale byte e, worth 2^(e - 127); e = 255 is NaN;
* storage: codes ``[rows][K/2]`` bytes, element 2j in the low nibble and 2j+1
  in the high nibble; scales ``[rows][K/32]`` bytes.

Quantiser (per block): s = max(floor(log2 amax) - 2, -127), with floor(log2)
taken exactly via frexp; each element v = w / 2^s (exact) is rounded to the
nearest E2M1 magnitude, ties to the even code, saturating at 6; the sign bit is
the input's sign bit (so -0.0 and small negatives give code 8).  A block that
holds a NaN or an infinity gets scale byte 255 and all-zero codes.
"""
from __future__ import annotations

import numpy as np

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
BLOCK = 32
SCALE_NAN = 255

# Midpoints between consecutive magnitudes, and whether a value exactly on the
# midpoint rounds up (the upper neighbour has the even code) or down.
_MIDPOINTS = (E2M1_MAGNITUDES[:-1] + E2M1_MAGNITUDES[1:]) / 2.0  # .25 .75 1.25 1.75 2.5 3.5 5
_TIE_UP = np.array([(i + 1) % 2 == 0 for i in range(7)])


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (uint16) as float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def decode_e2m1(code) -> np.ndarray:
    """Value of 4-bit E2M1 codes (sign bit 3, magnitude bits 2..0)."""
    c = np.asarray(code, dtype=np.int64)
    mag = E2M1_MAGNITUDES[c & 7]
    return np.where((c & 8) != 0, -mag, mag)


def decode_e8m0(byte) -> np.ndarray:
    """Value 2^(e-127) of E8M0 scale bytes; 255 decodes to NaN."""
    e = np.asarray(byte, dtype=np.int64)
    v = np.ldexp(1.0, (e - 127).astype(np.int32) if isinstance(e, np.ndarray) else int(e) - 127)
    return np.where(e == SCALE_NAN, np.nan, v)


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """``[rows][K/2]`` packed bytes -> ``[rows][K]`` 4-bit codes (low nibble first)."""
    c = np.asarray(codes, dtype=np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = c & 0x0F
    out[..., 1::2] = c >> 4
    return out


def pack_codes(nib: np.ndarray) -> np.ndarray:
    """``[rows][K]`` 4-bit codes -> ``[rows][K/2]`` bytes (element 2j in the low nibble)."""
    n = np.asarray(nib, dtype=np.uint8)
    return (n[..., 0::2] | (n[..., 1::2] << 4)).astype(np.uint8)


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Exact fp64 weights ``[rows][K]`` from MXFP4 codes and scales."""
    vals = decode_e2m1(unpack_codes(codes))
    rows, K = vals.shape[-2], vals.shape[-1]
    sc = decode_e8m0(scales)
    return (vals.reshape(vals.shape[:-1] + (K // BLOCK, BLOCK)) * sc[..., None]).reshape(
        vals.shape[:-2] + (rows, K))


def shared_exponent(amax: np.ndarray) -> np.ndarray:
    """s = max(floor(log2 amax) - 2, -127) per block; amax = 0 gives -127.

    floor(log2 amax) is read exactly from frexp (amax = m * 2^p, m in [0.5, 1),
    so floor(log2 amax) = p - 1), never from a floating log2.
    """
    _, p = np.frexp(amax)
    s = np.where(amax > 0, p.astype(np.int64) - 1 - 2, -127)
    return np.maximum(s, -127)


def round_e2m1_magnitude(a: np.ndarray) -> np.ndarray:
    """Nearest E2M1 magnitude index of |v| (ties to the even index; >= 6 -> 7)."""
    a = np.asarray(a, dtype=np.float64)
    idx = np.zeros(a.shape, dtype=np.uint8)
    for m, up in zip(_MIDPOINTS, _TIE_UP):
        idx += (a > m) | ((a == m) & up)
    return idx


def quantize(w_bits: np.ndarray):
    """Reference MXFP4 quantiser of bf16 weights ``[rows][K]`` (uint16 bits), K % 32 == 0.

    Returns (codes ``[rows][K/2]`` uint8, scales ``[rows][K/32]`` uint8).
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    rows, K = w_bits.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    w = bf16_to_f64(w_bits).reshape(rows, K // BLOCK, BLOCK)
    finite = np.isfinite(w).all(axis=-1)
    wz = np.where(np.isfinite(w), w, 0.0)
    amax = np.abs(wz).max(axis=-1)
    s = shared_exponent(amax)
    v = np.ldexp(wz, (-s)[..., None].astype(np.int32))  # exact: scaling by a power of two
    mag = round_e2m1_magnitude(np.abs(v))
    sign = np.signbit(w).astype(np.uint8) << 3
    nib = np.where(finite[..., None], sign | mag, 0).astype(np.uint8)
    scales = np.where(finite, s + 127, SCALE_NAN).astype(np.uint8)
    return pack_codes(nib.reshape(rows, K)), scales
