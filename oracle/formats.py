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
