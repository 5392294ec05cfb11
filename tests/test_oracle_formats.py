"""Pins of the oracle's storage codecs against the format definition (golden
table) and against torch's own float8/bfloat16 casts (independent library
routines).  CPU only."""
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_e4m3():
    rows = []
    for line in open(os.path.join(GOLDEN, "e4m3_values.txt")):
        line = line.split("#")[0].strip()
        if line:
            c, v = line.split()
            rows.append((int(c, 16), float(v)))
    return rows


def test_e4m3_golden_values():
    for code, val in _golden_e4m3():
        got = O.e4m3_decode(np.array([code], dtype=np.uint8))[0]
        if np.isnan(val):
            assert np.isnan(got), hex(code)
        else:
            assert got == val and np.signbit(got) == np.signbit(val), (hex(code), got, val)


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_e4m3_encode_roundtrips_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(O.e4m3_encode(O.e4m3_decode(codes)), codes)


def test_e4m3_encode_matches_torch_cast():
    g = torch.Generator().manual_seed(1)
    x = torch.cat([torch.randn(200000, generator=g) * s for s in (0.003, 0.1, 1.0, 30.0, 150.0)])
    x = x.clamp(-448, 448)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_encode(x.double().numpy())
    assert np.array_equal(ref, got)


def test_e4m3_encode_ties_saturation_sign():
    # midpoint of 1.0 (0x38, even) and 1.125 (0x39) -> 0x38; of 1.125 and 1.25 (0x3A) -> 0x3A
    assert O.e4m3_encode([1.0625])[0] == 0x38
    assert O.e4m3_encode([1.1875])[0] == 0x3A
    # half the smallest subnormal ties to zero; 1.5 subnormal steps tie to 2 steps
    assert O.e4m3_encode([2.0 ** -10])[0] == 0x00
    assert O.e4m3_encode([3 * 2.0 ** -10])[0] == 0x02
    # saturation (finite-only encoding): beyond 448 stays 448
    assert O.e4m3_encode([1000.0, -1e9, 464.0])[0] == 0x7E
    assert O.e4m3_encode([-1e9])[0] == 0xFE
    assert O.e4m3_encode([-0.0])[0] == 0x80
    assert O.e4m3_encode([-1e-6])[0] == 0x80
    assert O.e4m3_encode([np.nan])[0] == 0x7F


def test_bf16_codec_matches_torch():
    g = torch.Generator().manual_seed(2)
    x = torch.cat([torch.randn(100000, generator=g) * s for s in (1e-30, 1e-3, 1.0, 1e5)])
    x = torch.cat([x, torch.tensor([0.0, -0.0, 1e-40, -3e-39, 3.3e38])])
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.bf16_encode(x.double().numpy())
    assert np.array_equal(ref, got)
    back = torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(O.bf16_decode(ref), back)
