"""Storage-format codecs of the oracle (test infrastructure; see package doc).

The KV cache keeps most dims in FP8 and the 64 RoPE dims in BF16
(«DeepSeek-V4: 1 Million Token Context endlich nutzbar», section "Hybrid
Attention: CSA und HCA"; «Chinas KI-Unabhaengigkeit?: Bei Deepseek V4 haben
kleine Aenderungen grosse Wirkung», section "Komprimierte Erinnerung fuer
laengere Kontexte").  The FP8 flavour is E4M3 with a finite-only encoding
(the F8_E4M3 weight format listed in «DeepSeek-V4 Pro und Flash: 1,6
Billionen Parameter ...», section "Modelldetails").

E4M3 as used here: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
exponent field 0 is subnormal (value m/8 * 2^-6); no infinities; the only NaN
pattern is S.1111.111; the largest finite magnitude is 1.75 * 2^8 = 448.
BF16: the upper 16 bits of an IEEE binary32.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_value_table() -> np.ndarray:
    """Value of each of the 256 E4M3 codes, from the bit-field definition."""
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * (m / 8.0) * 2.0 ** -6
        else:
            vals[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_TABLE = e4m3_value_table()
# positive finite codes 0x00..0x7E have strictly increasing values
_POS = _TABLE[:0x7F].copy()


def e4m3_decode(codes) -> np.ndarray:
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    """Round to the nearest E4M3 value, ties to the even code, saturating to
    +-448; the sign is kept (so -0.0 and negative underflow give 0x80)."""
    x = np.asarray(x, dtype=np.float64)
    mag = np.abs(x)
    out = np.empty(x.shape, dtype=np.uint8)
    nan = np.isnan(x)
    m = np.where(nan, 0.0, np.minimum(mag, E4M3_MAX))
    hi = np.searchsorted(_POS, m, side="left")          # first grid value >= m
    hi = np.clip(hi, 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    d_lo = m - _POS[lo]
    d_hi = _POS[hi] - m
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(m == _POS[hi], hi, code)             # exact grid values
    sign = np.signbit(x).astype(np.uint8) << 7
    out[...] = (code.astype(np.uint8) | sign)
    out[nan] = 0x7F
    return out


def bf16_decode(bits) -> np.ndarray:
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_encode(x) -> np.ndarray:
    """Round a float64 value to the nearest BF16 value (ties to even) and
    return its 16-bit pattern.  BF16 keeps 8 significant bits, its smallest
    normal exponent is -126 and its subnormal spacing 2^-133."""
    x = np.asarray(x, dtype=np.float64)
    mant, ex = np.frexp(x)                 # x = mant * 2^ex, |mant| in [0.5, 1)
    ex = np.maximum(ex, -125)              # below the normal range the spacing stays 2^-133
    ulp = np.ldexp(1.0, ex - 8)
    q = np.rint(x / ulp) * ulp             # np.rint rounds halves to even
    bf16_max = (2.0 - 2.0 ** -7) * 2.0 ** 127
    q = np.where(np.abs(q) > bf16_max, np.copysign(np.inf, x), q)
    q = np.where(np.isnan(x), np.nan, q)
    return (q.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


# ------------------------------------------------------------------- MXFP4 ---
#
# The lightning indexer runs in FP4 («DeepSeek-V4: 1 Million Token Context
# endlich nutzbar», section "Hybrid Attention: CSA und HCA"); the 4-bit
# format named for DeepSeek-V4's attention is MXFP4 («Chinas
# KI-Unabhaengigkeit?: Bei Deepseek V4 haben kleine Aenderungen grosse
# Wirkung», introduction) and F8_E8M0 is among its stored types («DeepSeek-V4
# Pro und Flash ...», "Modelldetails").  MXFP4 as defined by the OCP
# Microscaling Formats (MX) Specification v1.0: blocks of 32 elements share
# one E8M0 scale; each element is FP4 E2M1.
#   E2M1: 1 sign bit, 2 exponent bits with bias 1, 1 mantissa bit; exponent
#         field 0 is subnormal (value m/2); no infinities or NaN; magnitudes
#         0, 0.5, 1, 1.5, 2, 3, 4, 6.
#   E8M0: an unsigned 8-bit exponent, value 2^(e - 127); e = 255 is NaN.
# Storage here: two E2M1 codes per byte, the even element in the low nibble.

E2M1_MAX = 6.0
MX_BLOCK = 32


def e2m1_value_table() -> np.ndarray:
    """Value of each of the 16 E2M1 codes, from the bit-field definition."""
    vals = np.empty(16, dtype=np.float64)
    for code in range(16):
        sign = -1.0 if code & 0x8 else 1.0
        e = (code >> 1) & 0x3
        m = code & 0x1
        vals[code] = sign * ((m / 2.0) if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1))
    return vals


_E2M1 = e2m1_value_table()
_E2M1_POS = _E2M1[:8].copy()            # codes 0..7, strictly increasing


def e2m1_decode(codes) -> np.ndarray:
    return _E2M1[np.asarray(codes, dtype=np.uint8) & 0xF]


def e2m1_encode(x) -> np.ndarray:
    """Round to the nearest E2M1 value, ties to the even code, saturating to
    +-6; the sign is kept (negative values that round to zero give 0x8)."""
    x = np.asarray(x, dtype=np.float64)
    m = np.minimum(np.abs(x), E2M1_MAX)
    hi = np.clip(np.searchsorted(_E2M1_POS, m, side="left"), 0, 7)
    lo = np.clip(hi - 1, 0, 7)
    d_lo = m - _E2M1_POS[lo]
    d_hi = _E2M1_POS[hi] - m
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(m == _E2M1_POS[hi], hi, code)
    return (code.astype(np.uint8) | (np.signbit(x).astype(np.uint8) << 3)).astype(np.uint8)


def e8m0_decode(e) -> np.ndarray:
    e = np.asarray(e, dtype=np.int64)
    return np.where(e == 255, np.nan, np.ldexp(1.0, (e - 127).astype(np.int64)))


def mxfp4_pack(codes) -> np.ndarray:
    """[..., d] E2M1 codes -> [..., d/2] bytes, element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def mxfp4_unpack(packed) -> np.ndarray:
    """[..., d/2] bytes -> [..., d] E2M1 codes."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def mxfp4_decode(packed, exps) -> np.ndarray:
    """Values of MXFP4 vectors: [..., d/2] packed codes, [..., d/32] E8M0
    exponents -> float64 [..., d]."""
    v = e2m1_decode(mxfp4_unpack(packed))
    s = e8m0_decode(exps)
    return v * np.repeat(s, MX_BLOCK, axis=-1)[..., : v.shape[-1]]


def mxfp4_quantize(x):
    """MXFP4 encoding of float64 vectors [..., d] (d a multiple of 32), the
    OCP MX conversion: per block, the shared exponent is
    X = floor(log2(amax)) - 2 (2 = the largest E2M1 exponent), clamped to the
    E8M0 range, and every element is E2M1(x / 2^X) rounded to nearest even
    and saturated.  READING: an all-zero block takes exponent 0 (byte 127).
    Returns (packed codes [..., d/2] uint8, E8M0 bytes [..., d/32] uint8)."""
    x = np.asarray(x, dtype=np.float64)
    blocks = x.reshape(x.shape[:-1] + (x.shape[-1] // MX_BLOCK, MX_BLOCK))
    amax = np.max(np.abs(blocks), axis=-1)
    with np.errstate(divide="ignore"):
        X = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 2, 0.0)
    X = np.clip(X, -127, 127)
    codes = e2m1_encode(blocks / np.ldexp(1.0, X.astype(np.int64))[..., None])
    return mxfp4_pack(codes.reshape(x.shape)), (X + 127).astype(np.uint8)
