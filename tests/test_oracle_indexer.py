"""Pins of the oracle's lightning-indexer score and top-k selection: closed
forms of the weighted-ReLU score, brute-force sorting on tiny inputs,
tie-breaking, k >= n, visibility and padding.  CPU only."""
import numpy as np

import oracle as O


def test_score_single_head_is_relu_dot():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, 16))
    k = rng.standard_normal((40, 16))
    s = O.indexer_scores(q, np.array([1.0]), k)
    for j in range(40):
        d = sum(q[0, i] * k[j, i] for i in range(16))
        assert abs(s[j] - max(d, 0.0)) < 1e-12


def test_score_relu_is_per_head_before_the_weighted_sum():
    # heads q and -q with unit weights: the per-head ReLU gives |q.k|;
    # a ReLU after the sum would give 0, no ReLU would give 0 too.
    rng = np.random.default_rng(1)
    q0 = rng.standard_normal(8)
    k = rng.standard_normal((30, 8))
    s = O.indexer_scores(np.stack([q0, -q0]), np.array([1.0, 1.0]), k)
    assert np.allclose(s, np.abs(k @ q0), rtol=1e-14, atol=1e-14)


def test_score_weight_sign_and_linearity():
    rng = np.random.default_rng(2)
    q = np.abs(rng.standard_normal((3, 8)))
    k = np.abs(rng.standard_normal((20, 8)))       # every dot positive -> ReLU inactive
    w = np.array([0.5, -2.0, 1.0])
    assert np.allclose(O.indexer_scores(q, w, k), k @ (w @ q), rtol=1e-13)
    assert np.all(O.indexer_scores(q, np.array([-1.0, -1.0, -1.0]), k) < 0)


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(3)
    for trial in range(50):
        n = int(rng.integers(1, 60))
        s = np.round(rng.standard_normal(n) * 2) / 2          # many exact ties
        k = int(rng.integers(1, 70))
        got = O.topk(s, n, k)
        ref = sorted(range(n), key=lambda j: (-s[j], j))[:k]
        assert list(got[:len(ref)]) == ref
        assert np.all(got[len(ref):] == -1)


def test_topk_k_at_least_n_takes_every_visible_entry():
    s = np.array([3.0, -1.0, 2.0, 7.0, 0.0, 9.0])
    got = O.topk(s, 4, 10)        # entries 4, 5 are not yet visible
    assert sorted(got[got >= 0]) == [0, 1, 2, 3]
    assert np.sum(got == -1) == 6


def test_topk_respects_visibility_and_prefers_lower_index():
    s = np.array([5.0, 5.0, 5.0, 9.0])
    assert list(O.topk(s, 3, 2)) == [0, 1]
    assert list(O.topk(s, 0, 2)) == [-1, -1]


def _layer_scores_brute_force(L, b, n):
    """Score of entries 0..n-1 for query row (b, 0) from the stored codes,
    decoded through the E4M3 value table, with every scale applied to its
    own dims: sum_h w_h max(0, sum_d q[h,d] sq[h, blk(d)] k[j,d] sk[j, blk(d)])."""
    tab = O.e4m3_value_table()
    blk = O.scale_block(L["comp_ik"]["fmt"], L["wl"].d_I)
    q = L["q_ik"][b, 0].numpy()
    sq = L["q_ik_scale"][b, 0].double().numpy()
    kc = L["comp_ik"]["data"][b].numpy()
    sk = L["comp_ik"]["scale"][b].double().numpy()
    w = L["head_w"][b, 0].double().numpy()
    H, d_I = q.shape
    out = np.zeros(n)
    for j in range(n):
        tot = 0.0
        for h in range(H):
            dot = 0.0
            for d in range(d_I):
                dot += tab[q[h, d]] * sq[h, d // blk] * tab[kc[j, d]] * sk[j, d // blk]
            tot += w[h] * max(dot, 0.0)
        out[j] = tot
    return out


def test_layer_scores_follow_each_indexer_scale_layout():
    # tiny FP8 layer, both indexer layouts: the query scales follow the keys'
    import workloads as W
    base = W.get("parity_decode").with_(B=1, T=163, H_I=3, d_I=64, k=8, needles=0)
    for ik_fmt in ("e4m3vec", "e4m3"):
        wl = base.with_(ik_fmt=ik_fmt)
        L = W.make_csa_layer(wl)
        (idx, s), = O.layer_indexer_topk(L, wl.k).values()
        ref = _layer_scores_brute_force(L, 0, len(s))
        assert np.allclose(s, ref, rtol=1e-12, atol=1e-12)
    # the same codes under two scale layouts give different scores
    wl = base.with_(ik_fmt="e4m3", d_I=128)
    L = W.make_csa_layer(wl)
    (idx, s), = O.layer_indexer_topk(L, wl.k).values()
    assert np.allclose(s, _layer_scores_brute_force(L, 0, len(s)), rtol=1e-12, atol=1e-12)
    L["comp_ik"]["fmt"] = "e4m3vec"
    (idx2, s2), = O.layer_indexer_topk(L, wl.k).values()
    assert np.allclose(s2, _layer_scores_brute_force(L, 0, len(s2)), rtol=1e-12, atol=1e-12)
    assert not np.allclose(s, s2)
