"""Pins of the oracle's hybrid attention: window-only equals exact causal
attention (torch SDPA in float64 as the library cross-check), Q = 0 closed
form, k >= n equals dense, LSE-merge identity, probabilities sum to one.
CPU only."""
import math

import numpy as np
import torch

import oracle as O
import workloads as W


def test_window_positions():
    assert list(O.window_positions(200, 128)) == list(range(73, 201))
    assert list(O.window_positions(5, 128)) == list(range(0, 6))


def test_window_only_short_sequence_equals_causal_sdpa():
    # with no compressed entries and T <= window, every query sees exactly
    # the tokens 0..pos: plain causal attention
    rng = np.random.default_rng(0)
    T, H, D = 100, 4, 16
    q = rng.standard_normal((T, H, D))
    K = rng.standard_normal((T, D))
    V = rng.standard_normal((T, D))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).permute(1, 0, 2),
        torch.from_numpy(K)[None].expand(H, T, D),
        torch.from_numpy(V)[None].expand(H, T, D),
        is_causal=True, scale=1 / math.sqrt(D)).permute(1, 0, 2).numpy()
    for pos in (0, 1, 37, 99):
        wp = O.window_positions(pos, 128)
        o, _ = O.hybrid_attention(q[pos], K[:0], V[:0], K[wp], V[wp], 1 / math.sqrt(D))
        assert np.allclose(o, ref[pos], rtol=1e-12, atol=1e-12)


def test_zero_query_gives_mean_value_and_log_count():
    rng = np.random.default_rng(1)
    K = rng.standard_normal((70, 8))
    V = rng.standard_normal((70, 8))
    o, lse = O.attend(np.zeros((3, 8)), K, V, 0.3)
    assert np.allclose(o, V.mean(axis=0), rtol=1e-13, atol=1e-14)
    assert np.allclose(lse, math.log(70), rtol=1e-14)


def test_probabilities_sum_to_one():
    rng = np.random.default_rng(2)
    K = rng.standard_normal((50, 8)) * 3
    o, _ = O.attend(rng.standard_normal((5, 8)), K, np.ones((50, 2)), 1.0)
    assert np.allclose(o, 1.0, rtol=0, atol=1e-13)


def test_lse_merge_of_parts_equals_single_pass():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((6, 16))
    K = rng.standard_normal((90, 16))
    V = rng.standard_normal((90, 16))
    o, lse = O.attend(q, K, V, 0.25)
    parts = [O.attend(q, K[a:b], V[a:b], 0.25) for a, b in ((0, 7), (7, 64), (64, 90))]
    L = np.log(sum(np.exp(l) for _, l in parts))
    om = sum(np.exp(l - L)[:, None] * oo for oo, l in parts)
    assert np.allclose(L, lse, rtol=1e-13)
    assert np.allclose(om, o, rtol=1e-12, atol=1e-13)


def test_topk_at_least_entry_count_equals_dense():
    wl = W.get("tiny").with_(T=700)          # 175 CSA entries, k below and above
    L = W.make_csa_layer(wl)
    dense = O.layer_attention(L, sel=None)
    r = O.layer_indexer_topk(L, 400)
    (idx, _), = r.values()
    sparse = O.layer_attention(L, sel=idx[None, None, :])
    (od, ld), = dense.values()
    (os_, ls), = sparse.values()
    assert np.allclose(od, os_, rtol=1e-12, atol=1e-12)
    assert np.allclose(ld, ls, rtol=1e-13)


def test_window_only_layer_tiny_equals_sdpa_over_ring():
    # T <= 128: the ring holds every token; no compressed entries visible for HCA
    wl = W.get("tiny").with_(T=100)
    L = W.make_hca_layer(wl)
    (o, lse), = O.layer_attention(L, sel=None).values()
    ring_k = L["ring_k"]["data"][0, :100].double()
    ring_v = L["ring_v"]["data"][0, :100].double()
    q = L["q"][0, 0].double()
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[:, None, :], ring_k[None].expand(8, 100, 128), ring_v[None].expand(8, 100, 128),
        scale=1.0)[:, 0].numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)
