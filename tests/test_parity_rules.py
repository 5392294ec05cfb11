"""The comparison rules of parity.py, on the CPU: each accepts what the
definitions allow (exact results, near-tie swaps, rounding-boundary flips)
and rejects planted mistakes, so that a GPU parity test cannot pass by a
checker that is too lenient."""
import numpy as np
import pytest

import oracle as O
from parity import (ATTN_REL, LSE_TOL, POOL_EPS, check_attention, check_codes,
                    check_pooled_f32, check_topk)


def _scores(n=200, seed=0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(n)


def _sel(s, k):
    # the oracle's top-k in selection order (score descending, index ascending)
    return O.topk(np.asarray(s), len(s), k)


def _gpu_order(sel):
    # the CUDA path's order: ascending entry index, then -1 padding
    live = np.sort(sel[sel >= 0])
    return np.concatenate([live, np.full(sel.size - live.size, -1, dtype=np.int64)])


def test_topk_exact_and_near_tie_pass():
    s = _scores()
    k = 20
    ref = _sel(s, k)
    assert check_topk(_gpu_order(ref), ref, s) == 0
    # the best entry outside the selection made a near tie (within 1e-3
    # relative) of the k-th score: swapping the two is allowed
    kth = int(ref[k - 1])
    outside = int(_sel(s, k + 1)[k])
    s2 = s.copy()
    s2[outside] = s2[kth] * (1 - 0.5e-3) if s2[kth] > 0 else s2[kth] * (1 + 0.5e-3)
    ref2 = _sel(s2, k)
    swapped = np.array(sorted((set(ref2.tolist()) - {int(ref2[k - 1])}) | {outside}))
    assert check_topk(swapped, ref2, s2) == 1


def test_topk_rejects_far_swap_order_padding_and_range():
    s = _scores()
    k = 20
    ref = _sel(s, k)
    gpu = _gpu_order(ref)
    low = int(np.argmin(s))                      # far below the k-th score
    bad = np.array(sorted((set(ref.tolist()) - {int(ref[0])}) | {low}))
    with pytest.raises(AssertionError):
        check_topk(bad, ref, s)
    with pytest.raises(AssertionError):          # not ascending
        check_topk(gpu[::-1].copy(), ref, s)
    with pytest.raises(AssertionError):          # one entry short
        check_topk(np.concatenate([gpu[:-1], [-1]]), ref, s)
    short = _sel(s[:10], k)                      # fewer visible than k: -1 padding
    g_short = _gpu_order(short)
    assert check_topk(g_short, short, s[:10]) == 0
    with pytest.raises(AssertionError):          # padding before real entries
        check_topk(np.concatenate([[-1], g_short[:-1]]), short, s[:10])
    with pytest.raises(AssertionError):          # entry beyond the visible range
        check_topk(np.concatenate([g_short[:9], [12], g_short[10:]]), short, s[:10])


def test_attention_tolerance():
    rng = np.random.default_rng(1)
    ref_o = rng.standard_normal((4, 64))
    ref_l = rng.standard_normal(4)
    rms = np.sqrt(np.mean(ref_o ** 2))
    ok = ref_o.copy()
    ok[1, 3] += 0.9 * ATTN_REL * rms
    check_attention(ok, ref_l + 0.5 * LSE_TOL, ref_o, ref_l)
    bad = ref_o.copy()
    bad[2, 5] += 1.5 * ATTN_REL * rms
    with pytest.raises(AssertionError):
        check_attention(bad, ref_l, ref_o, ref_l)
    with pytest.raises(AssertionError):
        check_attention(ref_o, ref_l + 2 * LSE_TOL, ref_o, ref_l)
    nan = ref_o.copy()
    nan[0, 0] = np.nan
    with pytest.raises(AssertionError):
        check_attention(nan, ref_l, ref_o, ref_l)


def test_codes_band():
    rng = np.random.default_rng(2)
    y = rng.uniform(-300, 300, 4000)
    codes = O.e4m3_encode(y)
    assert check_codes(codes, y, O.e4m3_encode, O.e4m3_decode, np.zeros_like(y)) == 1.0
    # a value right at a rounding boundary may round either way within the band
    lo = float(O.e4m3_decode(np.array([0x38], dtype=np.uint8))[0])   # 1.0
    hi = float(O.e4m3_decode(np.array([0x39], dtype=np.uint8))[0])   # 1.125
    mid = np.array([(lo + hi) / 2])
    other = np.array([0x39 if O.e4m3_encode(mid)[0] == 0x38 else 0x38], dtype=np.uint8)
    check_codes(other, mid, O.e4m3_encode, O.e4m3_decode, np.array([1e-3]), min_exact=0.0)
    # two steps away is outside any band of that width
    far = codes.copy()
    far[7] = np.uint8((int(far[7]) + 2) & 0xFF) if (int(far[7]) & 0x7F) < 0x7C else far[7] - 2
    with pytest.raises(AssertionError):
        check_codes(far, y, O.e4m3_encode, O.e4m3_decode, np.full_like(y, 1e-6))


def test_pooled_bound():
    ref = np.array([1.0, -2.0, 3.0])
    mag = np.array([1.0, 2.0, 3.0])
    check_pooled_f32(ref + 0.5 * POOL_EPS * mag, ref, mag)
    with pytest.raises(AssertionError):
        check_pooled_f32(ref + 2 * POOL_EPS * mag, ref, mag)
