"""Pins of the oracle's MXFP4 codecs (the FP4 lightning-indexer layout)
against the OCP MX definition (golden table, closed forms) and torch's own
float8_e8m0fnu decoding; and of the MXFP4 indexer score against a brute-force
block-by-block sum.  CPU only."""
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_e2m1_golden_values():
    rows = []
    for line in open(os.path.join(GOLDEN, "e2m1_values.txt")):
        line = line.split("#")[0].strip()
        if line:
            c, v = line.split()
            rows.append((int(c, 16), float(v)))
    assert len(rows) == 16
    tab = O.e2m1_value_table()
    for c, v in rows:
        assert tab[c] == v and np.signbit(tab[c]) == np.signbit(v), hex(c)


def test_e8m0_decode_matches_torch_and_closed_form():
    codes = np.arange(256, dtype=np.uint8)
    got = O.e8m0_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).double().numpy()
    assert np.isnan(got[255]) and np.isnan(ref[255])
    assert np.array_equal(got[:255], ref[:255])
    assert got[127] == 1.0 and got[128] == 2.0 and got[0] == 2.0 ** -127


def test_e2m1_encode_roundtrip_ties_saturation_sign():
    tab = O.e2m1_value_table()
    for c in range(16):
        if c == 8:
            continue                                  # -0.0 encodes as 0x8 too
        assert O.e2m1_encode(tab[c])[()] == c
    assert O.e2m1_encode(-0.0)[()] == 8
    # ties go to the even code: 0.25 -> 0 (code 0), 0.75 -> 1.0 (code 2),
    # 1.25 -> 1.0 (code 2), 1.75 -> 2.0 (code 4), 2.5 -> 2.0, 3.5 -> 4.0, 5 -> 4.0
    for x, want in ((0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0),
                    (3.5, 4.0), (5.0, 4.0), (-5.0, -4.0)):
        assert tab[O.e2m1_encode(x)[()]] == want, x
    # nearest otherwise, saturation beyond 6
    for x, want in ((0.26, 0.5), (2.6, 3.0), (5.1, 6.0), (6.0, 6.0), (7.0, 6.0), (1e9, 6.0),
                    (-1e9, -6.0)):
        assert tab[O.e2m1_encode(x)[()]] == want, x


def test_pack_order_and_roundtrip():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, size=(5, 64)).astype(np.uint8)
    packed = O.mxfp4_pack(codes)
    assert packed.shape == (5, 32)
    assert packed[0, 0] == (codes[0, 0] | (codes[0, 1] << 4))   # even element in the low nibble
    assert np.array_equal(O.mxfp4_unpack(packed), codes)


def test_mxfp4_quantize_follows_the_shared_exponent_rule():
    # blocks already on the grid of their shared exponent round-trip exactly
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 16, size=(6, 128)).astype(np.uint8)
    codes[:, ::32] = 0x7                               # each block's amax is 6 * 2^X
    X = rng.integers(-5, 6, size=(6, 4))
    vals = O.e2m1_decode(codes) * np.repeat(np.ldexp(1.0, X), 32, axis=1)
    packed, exps = O.mxfp4_quantize(vals)
    assert np.array_equal(exps.astype(np.int64), X + 127)
    assert np.array_equal(O.mxfp4_unpack(packed), np.where(codes == 8, 0, codes) | (codes & 8))
    assert np.array_equal(O.mxfp4_decode(packed, exps), vals)
    # X = floor(log2 amax) - 2: amax 1 -> X = -2 (1 becomes 4), amax 7 -> X = 0
    # (7 saturates to 6), amax 0.3 -> X = -4 (0.3 / 2^-4 = 4.8 -> 4)
    for amax, x_want, v_want in ((1.0, -2, 1.0), (7.0, 0, 6.0), (0.3, -4, 0.25)):
        v = np.zeros((1, 32))
        v[0, 5] = amax
        p, e = O.mxfp4_quantize(v)
        assert int(e[0, 0]) - 127 == x_want
        assert O.mxfp4_decode(p, e)[0, 5] == v_want
    # an all-zero block keeps exponent 0 and zero codes
    p, e = O.mxfp4_quantize(np.zeros((1, 32)))
    assert e[0, 0] == 127 and not p.any()


def test_mxfp4_score_is_the_blockwise_sum():
    # s = sum_h w_h max(0, q_h . k) with q, k MXFP4: brute force per element,
    # element value = E2M1(code) * 2^(e_block - 127)
    rng = np.random.default_rng(5)
    H, d, n = 4, 128, 9
    qp = rng.integers(0, 256, size=(H, d // 2)).astype(np.uint8)
    qe = rng.integers(120, 134, size=(H, d // 32)).astype(np.uint8)
    kp = rng.integers(0, 256, size=(n, d // 2)).astype(np.uint8)
    ke = rng.integers(120, 134, size=(n, d // 32)).astype(np.uint8)
    w = rng.normal(size=H)
    tab = O.e2m1_value_table()
    cache = {"fmt": "mxfp4", "d_nope": d, "d_rope": 0, "data": kp[None], "scale": ke[None],
             "rope": None}
    k = O.dequant_slots(cache, 0, np.arange(n))
    s = O.indexer_scores(O.mxfp4_decode(qp, qe), w, k)
    for j in range(n):
        want = 0.0
        for h in range(H):
            dot = 0.0
            for i in range(d):
                qc = (int(qp[h, i // 2]) >> (4 * (i % 2))) & 15
                kc = (int(kp[j, i // 2]) >> (4 * (i % 2))) & 15
                dot += tab[qc] * 2.0 ** (int(qe[h, i // 32]) - 127) * tab[kc] * \
                    2.0 ** (int(ke[j, i // 32]) - 127)
            want += w[h] * max(0.0, dot)
        assert s[j] == pytest.approx(want, rel=1e-12, abs=1e-300)
    # a planted mistake: the exponents of blocks 0 and 1 swapped
    wrong = dict(cache)
    wrong["scale"] = ke[None][:, :, [1, 0, 2, 3]]
    assert not np.allclose(O.dequant_slots(wrong, 0, np.arange(n)), k)
