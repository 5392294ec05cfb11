"""The paged storage of compressed caches (block tables), as the inputs
generator builds it and as the oracle reads it back: every logical slot of
every plane lands in pool row table[b][s // block_size] * block_size +
s % block_size and reads back unchanged; slots of unmapped blocks read NaN;
a swapped table entry is caught.  CPU only."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from oracle.layer import as_numpy_cache


def _same(x, y):
    if x.dtype.kind == "f":
        return np.array_equal(np.nan_to_num(x, nan=7.0), np.nan_to_num(y, nan=7.0))
    return np.array_equal(x, y)


@pytest.mark.parametrize("ik_fmt", ["e4m3vec", "e4m3", "mxfp4"])
@pytest.mark.parametrize("bs", [1, 16, 128])
def test_paged_planes_hold_every_slot_where_the_table_says(ik_fmt, bs):
    wl = W.get("parity_decode").with_(ik_fmt=ik_fmt, T=3001)
    L = W.make_csa_layer(wl)
    for key in ("comp_k", "comp_ik"):
        c = L[key]
        P = W.page_cache(c, bs, seed=bs + 1, unmapped_tail=1)
        bt = P["block_table"].numpy()
        assert bt.shape == (wl.B, P["cap"] // bs) and (bt[:, -1] == -1).all()
        mapped = bt[bt >= 0]
        assert len(np.unique(mapped)) == mapped.size and mapped.max() < P["num_blocks"]
        rng = np.random.default_rng(bs)
        for plane in ("data", "scale", "rope"):
            if c.get(plane) is None:
                continue
            def _np(t):
                return (t.view(torch.int16) if t.dtype == torch.bfloat16 else t).numpy()
            src, pool = _np(c[plane]), _np(P[plane])[0]
            for _ in range(50):                       # the row formula, slot by slot
                b, s = int(rng.integers(wl.B)), int(rng.integers(c["cap"]))
                assert _same(pool[bt[b, s // bs] * bs + s % bs], src[b, s])
        a, p = as_numpy_cache(c), as_numpy_cache(P)
        for plane in ("data", "scale", "rope"):
            if a[plane] is not None:
                assert _same(p[plane][:, : c["cap"]], a[plane])
        if p["scale"].dtype.kind == "f":
            assert np.isnan(p["scale"][:, -bs:]).all()   # the unmapped block


def test_a_swapped_table_entry_is_caught():
    wl = W.get("parity_decode")
    L = W.make_csa_layer(wl)
    P = W.page_cache(L["comp_ik"], 64, seed=9)
    good = as_numpy_cache(P)["data"]
    P["block_table"] = P["block_table"].clone()
    P["block_table"][1, [3, 4]] = P["block_table"][1, [4, 3]]
    bad = as_numpy_cache(P)["data"]
    assert not np.array_equal(good[1, 3 * 64: 5 * 64], bad[1, 3 * 64: 5 * 64])
    assert np.array_equal(good[0], bad[0]) and np.array_equal(good[2], bad[2])


def test_oracle_results_do_not_depend_on_the_storage():
    wl = W.get("parity_decode").with_(T=5000, k=64)
    L = W.make_csa_layer(wl)
    Lp = dict(L)
    Lp["comp_ik"] = W.page_cache(L["comp_ik"], 32, seed=2, unmapped_tail=2)
    Lp["comp_k"] = W.page_cache(L["comp_k"], 16, seed=3)
    r = O.layer_indexer_topk(L, wl.k, rows=[(0, 0), (2, 0)])
    rp = O.layer_indexer_topk(Lp, wl.k, rows=[(0, 0), (2, 0)])
    for row in r:
        assert np.array_equal(r[row][0], rp[row][0])
    sel = np.stack([r[(0, 0)][0], r[(0, 0)][0], r[(2, 0)][0]])[:, None, :]
    a = O.layer_attention(L, sel=sel, rows=[(0, 0)])
    ap = O.layer_attention(Lp, sel=sel, rows=[(0, 0)])
    assert np.array_equal(a[(0, 0)][0], ap[(0, 0)][0])
