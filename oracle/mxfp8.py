"""MXFP8 (OCP Microscaling v1.0, E4M3 elements, E8M0 shared scale) -- bit-level, fp64.

The article names MXFP8 as the activation format carried through dispatch, the grouped
GEMM and SwiGLU (§02, last technical paragraph) but does not define it; the definition
used here is the OCP MX v1.0 one the layer's configuration spells out: blocks of 32
contiguous elements along the GEMM's K axis, one E8M0 scale per block, E4M3 elements,
round-to-nearest-even, saturating conversion.

Scale rule (OCP MX v1.0 conversion): s = floor(log2(amax)) - emax_elem, with emax_elem = 8
for E4M3 (largest normal 448 = 1.75 * 2**8), clamped to the E8M0 range [-127, 127]; the
stored byte is s + 127.  With this "floor" rule amax * 2**-s lies in [256, 512), so
values in (448, 512) saturate to 448 -- the "saturate" of the configuration.

Readings where the definition is silent (listed in the design notes):
* all-zero block: floor(log2(0)) is -inf; we take s = -127 (byte 0x00), elements 0.
* a negative value that rounds to zero keeps its sign: code 0x80 (IEEE behaviour).
* NaN / Inf inputs are out of scope (the generators never produce them).
"""
from __future__ import annotations

import numpy as np

BLOCK = 32
E4M3_MAX = 448.0
E4M3_EMAX = 8
SCALE_MIN, SCALE_MAX = -127, 127


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 (fn variant: bias 7, no infinities, NaN = S.1111.111) bytes -> float64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    exp = (c >> 3) & 0xF
    man = c & 0x7
    sub = man.astype(np.float64) * 2.0 ** -9
    norm = (1.0 + man / 8.0) * np.ldexp(1.0, exp - 7)
    v = np.where(exp == 0, sub, norm)
    v = np.where((exp == 15) & (man == 7), np.nan, v)
    return sign * v


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """float64 -> E4M3 bytes: round to nearest (ties to even), saturate to +-448.

    The rounding is done on the magnitude with the quantum of its binade: 2**(e-3) for
    normal values (e = floor(log2|v|) >= -6) and 2**-9 in the subnormal range.
    """
    v = np.asarray(v, dtype=np.float64)
    neg = np.signbit(v)
    a = np.abs(v)
    _, e2 = np.frexp(a)               # a = m * 2**e2, m in [0.5, 1)
    e = np.maximum(e2.astype(np.int64) - 1, -6)    # binade exponent, subnormals share -6
    q = np.ldexp(1.0, e - 3)          # quantum of the binade
    r = np.rint(a / q) * q            # np.rint rounds half to even; a / q is exact
    r = np.minimum(r, E4M3_MAX)       # saturating conversion
    # encode the (now representable) magnitude r
    _, re2 = np.frexp(r)
    re = re2.astype(np.int64) - 1
    is_norm = r >= 2.0 ** -6
    exp_field = np.where(is_norm, re + 7, 0)
    man_norm = np.rint((np.ldexp(r, -np.where(is_norm, re, 0)) - 1.0) * 8.0)
    man_sub = np.rint(r / 2.0 ** -9)
    man = np.where(is_norm, man_norm, man_sub).astype(np.int64)
    code = (exp_field << 3) | man
    code = np.where(r == 0, 0, code)
    code = code | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


def e8m0_decode(scale_bytes: np.ndarray) -> np.ndarray:
    """E8M0 byte -> its power of two as float64 (byte 0xFF, NaN, is never produced)."""
    return np.ldexp(1.0, np.asarray(scale_bytes, dtype=np.int64) - 127)


def block_scale_exponent(amax: np.ndarray) -> np.ndarray:
    """s = floor(log2(amax)) - 8, clamped to [-127, 127]; s = -127 for amax == 0.

    floor(log2) comes from the binary exponent (np.frexp), never from a float log2.
    """
    amax = np.asarray(amax, dtype=np.float64)
    _, e2 = np.frexp(amax)
    s = e2.astype(np.int64) - 1 - E4M3_EMAX
    s = np.where(amax > 0, s, SCALE_MIN)
    return np.clip(s, SCALE_MIN, SCALE_MAX)


def quantize_mx(x: np.ndarray):
    """Quantise along the last axis in blocks of 32.

    Returns (codes uint8 [..., K], scale bytes uint8 [..., K/32]).
    """
    x = np.asarray(x, dtype=np.float64)
    K = x.shape[-1]
    if K % BLOCK:
        raise ValueError("last axis must be a multiple of 32")
    xb = x.reshape(x.shape[:-1] + (K // BLOCK, BLOCK))
    s = block_scale_exponent(np.max(np.abs(xb), axis=-1))
    v = np.ldexp(xb, -s[..., None])   # exact: scaling by a power of two
    codes = e4m3_encode(v).reshape(x.shape)
    return codes, (s + 127).astype(np.uint8)


def dequantize_mx(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """codes [..., K] and scale bytes [..., K/32] -> float64 values code * 2**s."""
    K = codes.shape[-1]
    v = e4m3_decode(codes).reshape(codes.shape[:-1] + (K // BLOCK, BLOCK))
    return (v * e8m0_decode(scales)[..., None]).reshape(codes.shape)


def fake_quantize_mx(x: np.ndarray) -> np.ndarray:
    """Quantise then dequantise along the last axis."""
    return dequantize_mx(*quantize_mx(x))


def quantize_mx_axis0_segment(x: np.ndarray):
    """Quantise a [n, C] block along axis 0 (tokens) in blocks of 32 rows.

    The segment is zero-padded to a multiple of 32 rows first.  Returns
    (codes [n_pad, C], scale bytes [n_pad/32, C]) with n_pad = ceil(n/32)*32.
    """
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[0]
    n_pad = -(-n // BLOCK) * BLOCK
    xp = np.zeros((n_pad,) + x.shape[1:], np.float64)
    xp[:n] = x
    codes_t, scales_t = quantize_mx(xp.T)        # along tokens
    return codes_t.T.copy(), scales_t.T.copy()
