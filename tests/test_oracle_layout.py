"""Pins of the oracle's key assembly for one query row: which compressed
entries and which raw window positions it attends, and where in the ring a
position lives.  Marker values planted at known positions (fp32 layout) make
an off-by-one in the visibility count, the window range or the ring slot
mapping show up directly."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W


@pytest.mark.parametrize("T,ring_cap", [(4096, 1024), (50, 128), (128, 128), (129, 128),
                                        (3000, 256)])
def test_row_keys_are_the_visible_entries_and_the_window(T, ring_cap):
    wl = W.get("tiny").with_(T=T)
    L = W.make_csa_layer(wl, ring_cap=ring_cap)
    pos = T - 1                                   # the decode query's own position
    # markers: raw position p in its ring slot (p mod cap), entry j in slot j
    rk, ck = L["ring_k"]["data"], L["comp_k"]["data"]
    for p in range(max(0, pos - ring_cap + 1), pos + 1):
        rk[0, p % ring_cap, 0] = float(p)
    ck[0, :, 0] = torch.arange(ck.shape[1], dtype=ck.dtype) + 1e5
    q, K, V, wk, wv = O.layer_attention_dense_keys(L, 0, 0)
    # every complete group of 4 tokens up to and including the query's is an entry
    n_vis = (pos + 1) // 4
    assert K.shape[0] == n_vis
    assert np.array_equal(K[:, 0], np.arange(n_vis) + 1e5)
    # the window: the last 128 positions, the query's own token included
    lo = max(0, pos - wl.window + 1)
    assert np.array_equal(wk[:, 0], np.arange(lo, pos + 1, dtype=np.float64))


def test_ring_slot_of_a_position():
    cap = 128
    pos = np.array([0, 1, 127, 128, 129, 1_048_575, 1_048_576])
    assert np.array_equal(O.ring_slots(pos, cap), np.array([0, 1, 127, 0, 1, 127, 0]))
