"""Pins of the oracle's softmax-gated pooling and requantisation: printed
entry counts, identity at pool = stride = 1, closed forms for uniform gates,
the bias-to-slot mapping, the gate's source vector, convexity.  CPU only."""
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_entry_counts_match_stated_workloads():
    n = 0
    for line in open(os.path.join(GOLDEN, "entry_counts.txt")):
        line = line.split("#")[0].strip()
        if line:
            t, s, e = map(int, line.split())
            assert O.n_entries(t, s) == e
            n += 1
    assert n >= 4


def test_pool_positions_overlap_previous_group():
    # CSA: window 8, stride 4 -> previous group + own group
    assert list(O.pool_positions(0, 8, 4)) == [-4, -3, -2, -1, 0, 1, 2, 3]
    assert list(O.pool_positions(5, 8, 4)) == list(range(16, 24))
    # HCA: window = stride = 128 -> disjoint blocks
    assert list(O.pool_positions(2, 128, 128)) == list(range(256, 384))


def _scalar_tokens(D=3):
    # token p carries the value p in every dim
    return lambda p: np.full(D, float(p))


def test_identity_when_pool_equals_stride_equals_one():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((37, 6))
    src = lambda p: X[p]
    (out,), w = O.pool_entries(src, [src], rng.standard_normal(6), rng.standard_normal(1), 1, 1,
                               range(37))
    assert np.array_equal(out, X)
    assert np.all(w == 1.0)


def test_uniform_gates_give_window_mean_csa():
    src = _scalar_tokens()
    (out,), w = O.pool_entries(src, [src], np.zeros(3), np.zeros(8), 8, 4, range(6))
    # entry 0 sees positions 0..3 only (left edge), entry j>=1 sees 4j-4..4j+3
    assert np.allclose(out[0], 1.5, rtol=0, atol=1e-15)
    for j in range(1, 6):
        assert np.allclose(out[j], 4 * j - 0.5, rtol=0, atol=1e-13)
    assert np.allclose(w[0], [0, 0, 0, 0, 0.25, 0.25, 0.25, 0.25])


def test_uniform_gates_give_window_mean_hca():
    src = _scalar_tokens()
    (out,), _ = O.pool_entries(src, [src], np.zeros(3), np.zeros(128), 128, 128, range(3))
    for j in range(3):
        assert np.allclose(out[j], 128 * j + 63.5, rtol=0, atol=1e-12)


@pytest.mark.parametrize("slot", [0, 3, 4, 7])
def test_positional_bias_selects_slot(slot):
    src = _scalar_tokens()
    b = np.zeros(8)
    b[slot] = 60.0       # e^60 dominates every other slot
    (out,), _ = O.pool_entries(src, [src], np.zeros(3), b, 8, 4, [3])
    assert np.allclose(out[0], 4 * 3 - 4 + slot, rtol=1e-12)


def test_gate_reads_the_key_not_the_value():
    rng = np.random.default_rng(1)
    K = rng.standard_normal((16, 4)) * 0.01
    V = rng.standard_normal((16, 4))
    K[9, 2] = 40.0                      # token 9 has a large key component on dim 2
    w = np.zeros(4); w[2] = 1.0         # the gate looks at key dim 2 only
    (ok, ov), _ = O.pool_entries(lambda p: K[p], [lambda p: K[p], lambda p: V[p]], w,
                                 np.zeros(8), 8, 4, [2, 3])
    # token 9 lies in the windows of entries 2 (4..11) and 3 (8..15)
    for row in (0, 1):
        assert np.allclose(ov[row], V[9], rtol=1e-12, atol=1e-12)


def test_weights_sum_to_one_and_convexity():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((64, 5))
    src = lambda p: X[p]
    (out,), w = O.pool_entries(src, [src], rng.standard_normal(5), rng.standard_normal(8),
                               8, 4, range(16))
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    for j in range(16):
        pos = O.pool_positions(j, 8, 4)
        pos = pos[pos >= 0]
        assert np.all(out[j] <= X[pos].max(axis=0) + 1e-14)
        assert np.all(out[j] >= X[pos].min(axis=0) - 1e-14)


def test_requantize_roundtrip_and_amax():
    rng = np.random.default_rng(3)
    # values already on the E4M3 grid at scale s = amax/448 quantise to themselves
    codes = rng.integers(0, 0x7E, size=(10, 128)).astype(np.uint8)
    codes[:, 0] = 0x7E                      # force the block amax to 448 * s
    codes[:, 64] = 0xFE
    s = rng.uniform(0.5, 2.0, size=(10, 2))
    c = O.e4m3_decode(codes) * np.repeat(s, 64, axis=1)
    c = np.concatenate([c, rng.standard_normal((10, 64))], axis=1)
    qc, qs, qr = O.requantize(c, 128)
    assert np.array_equal(qc, codes)
    assert np.allclose(qs, s, rtol=1e-15, atol=0)
    assert np.array_equal(qr, O.bf16_encode(c[:, 128:]))


def test_requantize_zero_block_and_codes_match_torch():
    rng = np.random.default_rng(4)
    c = rng.standard_normal((50, 448 + 64)) * 3
    c[7, 64:128] = 0.0
    qc, qs, _ = O.requantize(c, 448)
    assert qs[7, 1] == 1.0 and np.all(qc[7, 64:128] == 0)
    assert np.all(np.abs(O.e4m3_decode(qc)) <= 448)
    # every block's largest magnitude lands on 448 exactly
    for b in range(7):
        blk = np.abs(O.e4m3_decode(qc[:, 64 * b:64 * (b + 1)])).max(axis=1)
        assert np.all((blk == 448) | (qs[:, b] == 1.0))
    ref = torch.from_numpy(c[:, :448] / np.repeat(qs, 64, axis=1)).clamp(-448, 448)
    ref = ref.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ref, qc)


def test_requantize_one_scale_per_vector():
    # the indexer layout: one scale over all 128 dims, no BF16 part
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 0x7E, size=(12, 128)).astype(np.uint8)
    codes[:, 77] = 0xFE                     # amax = 448 * s, sign negative
    s = rng.uniform(0.01, 3.0, size=(12, 1))
    c = O.e4m3_decode(codes) * s
    qc, qs, qr = O.requantize(c, 128, O.scale_block("e4m3vec", 128))
    assert qs.shape == (12, 1) and qr.shape[1] == 0
    assert np.array_equal(qc, codes)
    assert np.allclose(qs, s, rtol=1e-15, atol=0)
    # a block-64 quantisation of the same rows keeps two scales, and differs
    # wherever the two halves' maxima differ
    qc64, qs64, _ = O.requantize(c, 128)
    assert qs64.shape == (12, 2)
    half = np.abs(O.e4m3_decode(codes)).reshape(12, 2, 64).max(axis=2) * s
    assert np.allclose(qs64, half / 448.0, rtol=1e-15)
    # the zero vector takes scale 1 and zero codes
    z, zs, _ = O.requantize(np.zeros((1, 128)), 128, 128)
    assert zs[0, 0] == 1.0 and not z.any()


def test_dequant_slots_per_vector_brute_force():
    rng = np.random.default_rng(6)
    codes = rng.integers(0, 256, size=(2, 9, 32)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0      # no NaN codes
    sc = rng.uniform(0.1, 2.0, size=(2, 9, 1))
    cache = {"fmt": "e4m3vec", "d_nope": 32, "d_rope": 0, "data": codes, "scale": sc,
             "rope": None}
    tab = O.e4m3_value_table()
    got = O.dequant_slots(cache, 1, [4, 0, 8])
    for r, j in enumerate([4, 0, 8]):
        for d in range(32):
            assert got[r, d] == tab[codes[1, j, d]] * sc[1, j, 0]


def test_layer_compress_tiny_uniform_gate_equals_mean():
    wl = W.get("tiny")
    L = W.make_csa_layer(wl)
    L["gate_w"] = torch.zeros_like(L["gate_w"])
    L["gate_b"] = torch.zeros_like(L["gate_b"])
    res = O.layer_compress(L, [wl.T - 12], [wl.T])[0]
    ring = L["ring_k"]["data"][0].double().numpy()
    for j, row in zip(res["j"], res["k"]):
        pos = O.pool_positions(int(j), 8, 4)
        assert np.allclose(row, ring[pos % ring.shape[0]].mean(axis=0), rtol=1e-13, atol=1e-13)


def _bf16_bits_to_float(bits: int) -> float:
    # a BF16 value is the upper half of an IEEE binary32 word
    import struct
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def _kv_entry_brute_force(codes, scales, rope, b, j):
    """One cache entry of the FP8 + BF16 KV layout read value by value: dims
    0 .. 447 are E4M3 codes times the scale of their 64-dim block, dims
    448 .. 511 the BF16 RoPE part."""
    tab = O.e4m3_value_table()
    d_nope, d_rope = codes.shape[2], rope.shape[2]
    out = []
    for d in range(d_nope):
        out.append(tab[int(codes[b, j, d])] * float(scales[b, j, d // 64]))
    for r in range(d_rope):
        out.append(_bf16_bits_to_float(rope[b, j, r]))
    return np.array(out)


def test_dequant_slots_kv_layout_brute_force():
    # the compressed KV cache entry of the measured workloads: 448 E4M3 dims
    # with seven fp32 block scales (scale plane padded to eight columns), then
    # 64 BF16 RoPE dims.  Planted mistakes (RoPE part first, scale columns
    # shifted by one block, the pad column used) must all disagree.
    rng = np.random.default_rng(11)
    B, n, d_nope, d_rope = 2, 5, 448, 64
    codes = rng.integers(0, 256, size=(B, n, d_nope)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x01     # no NaN codes
    scales = rng.uniform(0.25, 4.0, size=(B, n, 8))
    scales[:, :, 7] = np.nan                 # the pad column is never read
    rope_vals = rng.normal(size=(B, n, d_rope))
    rope = torch.tensor(rope_vals, dtype=torch.float32).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)
    cache = {"fmt": "e4m3", "d_nope": d_nope, "d_rope": d_rope, "data": codes, "scale": scales,
             "rope": rope}
    slots = [3, 0, 4]
    got = O.dequant_slots(cache, 1, slots)
    assert got.shape == (3, d_nope + d_rope)
    for r, j in enumerate(slots):
        want = _kv_entry_brute_force(codes, scales, rope, 1, j)
        assert np.array_equal(got[r], want), f"slot {j}"
        # planted mistakes that a wrong oracle could make
        rope_first = np.concatenate([want[d_nope:], want[:d_nope]])
        assert not np.array_equal(got[r], rope_first)
        tab = O.e4m3_value_table()
        shifted = np.array([tab[codes[1, j, d]] * scales[1, j, min(d // 64 + 1, 6)]
                            for d in range(d_nope)])
        assert not np.array_equal(got[r, :d_nope], shifted)
        assert np.all(np.isfinite(got[r]))    # the NaN pad scale is not used
    # the BF16 part is exactly torch's bfloat16 value of the stored bits
    ref_rope = torch.tensor(rope.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(got[:, d_nope:], ref_rope[1, slots])
