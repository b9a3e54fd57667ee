"""Number formats used by the layer, written from their definitions (oracle).

* bf16: IEEE-754 binary32 with the low 16 fraction bits dropped -- 8
  significant bits, same exponent range as fp32; rounding is to nearest, ties
  to even.
* OCP FP8 E4M3 (OCP "8-bit Floating Point Specification (OFP8)" and OCP
  "Microscaling Formats (MX) Specification v1.0"): 1 sign, 4 exponent (bias 7),
  3 mantissa bits; no infinities; S.1111.111 is NaN; largest finite 448;
  smallest normal 2^-6; subnormals m/8 * 2^-6.
* E8M0 scale (MX v1.0): an unsigned biased exponent, value 2^(byte-127),
  byte 255 is NaN.

MX block scaling (the MXFP8 format of "Ai2 rebuilds Olmo's training stack for
trillion-parameter MoEs", section "MXFP8 reduces compute and memory costs":
separate scaling for small blocks of values) follows MX v1.0: a block of 32
values shares X = floor(log2(amax)) - emax_elem with emax_elem = 8 for E4M3,
each value is stored as E4M3(v / 2^X) rounded to nearest-even and clamped to
+-448.  X is clamped to [-127, 127]; an all-zero block gets X = 0.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_EMAX = 8


def round_bf16(x) -> np.ndarray:
    """Nearest bf16 value (ties to even) of fp64 ``x``, returned as fp64."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                 # |x| = m 2^e with m in [0.5, 1)
    e = np.maximum(e, -125)            # below 2^-126 the spacing stays 2^-133
    q = np.ldexp(1.0, e - 8)           # 8 significant bits
    r = np.rint(x / q) * q             # x / q is exact; rint ties to even
    big = np.abs(r) >= 2.0 ** 128
    if np.any(big):
        r = np.where(big, np.copysign(np.inf, x), r)
    return r


def round_f32(x) -> np.ndarray:
    """Nearest fp32 value of fp64 ``x`` (numpy's cast rounds to nearest-even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def e4m3_round(v) -> np.ndarray:
    """Nearest E4M3 value of ``v`` (ties to even), clamped to +-448 ("satfinite")."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, e = np.frexp(a)
    e = np.maximum(e, -5)              # subnormal spacing 2^-9 below 2^-6
    q = np.ldexp(1.0, e - 4)           # 4 significant bits
    r = np.minimum(np.rint(a / q) * q, E4M3_MAX)
    return np.copysign(r, v)


def e4m3_encode(v) -> np.ndarray:
    """E4M3 code (uint8) of ``v`` after ``e4m3_round``; the sign of zero is kept."""
    r = e4m3_round(v)
    a = np.abs(r)
    sign = np.signbit(r).astype(np.int64) << 7
    _, e = np.frexp(a)
    normal = a >= 2.0 ** -6
    E = np.where(normal, e - 1, -6)                       # unbiased exponent
    mant_normal = np.rint((a / np.ldexp(1.0, E) - 1.0) * 8.0)
    mant_sub = np.rint(a / 2.0 ** -9)
    field_e = np.where(normal, E + 7, 0)
    field_m = np.where(normal, mant_normal, mant_sub).astype(np.int64)
    return (sign | (field_e.astype(np.int64) << 3) | field_m).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    """Value (fp64) of E4M3 codes; 0x7F / 0xFF decode to NaN."""
    c = np.asarray(codes).astype(np.int64)
    s = np.where((c >> 7) & 1, -1.0, 1.0)
    E = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    val = np.where(E == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.ldexp(1.0, E - 7))
    val = np.where((E == 15) & ((c & 7) == 7), np.nan, val)
    return s * val


def mx_scale_exponent(amax) -> np.ndarray:
    """Shared block exponent X = floor(log2(amax)) - 8, clamped to [-127, 127];
    0 for an all-zero block."""
    a = np.asarray(amax, dtype=np.float64)
    _, e = np.frexp(a)
    X = np.clip(e - 1 - E4M3_EMAX, -127, 127)
    return np.where(a == 0.0, 0, X).astype(np.int64)


def mx_quantize_blocks(blocks) -> tuple[np.ndarray, np.ndarray]:
    """Quantise ``blocks`` [..., n] (n <= 32 values sharing one scale).

    Returns (codes uint8 [..., n], scale bytes uint8 [...]) with
    scale byte = X + 127."""
    b = np.asarray(blocks, dtype=np.float64)
    amax = np.max(np.abs(b), axis=-1) if b.shape[-1] else np.zeros(b.shape[:-1])
    X = mx_scale_exponent(amax)
    codes = e4m3_encode(b * np.ldexp(1.0, -X)[..., None])
    return codes, (X + 127).astype(np.uint8)


def mx_dequantize(codes, scale_bytes) -> np.ndarray:
    """code value * 2^(scale byte - 127), scale broadcast over the last axis."""
    return e4m3_decode(codes) * np.ldexp(1.0, np.asarray(scale_bytes).astype(np.int64) - 127)[..., None]
