"""Device-side failure reporting, made to happen without a GPU fault: the
top-k meeting point is given a poll limit of zero (a CTA that arrives first
gives up at once), and a NaN head weight makes one query row unrankable.
The kernels must return, record the event in the device status word, and
leave either the exact result (the meeting point) or a row visibly marked
failed (NaN scores)."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_common import require_gpu, to_device
from parity import check_topk

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C():
    C = require_gpu()
    C.check_device_errors()          # start from a clear status word
    return C


def test_status_word_is_clear_after_normal_calls(C):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer, HCALayer
    wl = W.get("parity_decode")
    csa = CSALayer(to_device(W.make_csa_layer(wl)))
    csa.step()
    HCALayer(to_device(W.make_hca_layer(wl))).attend()
    assert C.check_device_errors() == 0
    assert C.check_device_errors() == 0


def test_topk_meeting_point_timeout_keeps_the_result_exact(C):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    # 25,000 visible entries per row: several selection CTAs share each row
    wl = W.get("parity_decode").with_(B=4, T=100_003, k=512)
    L = W.make_csa_layer(wl)
    layer = CSALayer(to_device(L))
    ref = O.layer_indexer_topk(L, wl.k)
    old = C.debug_topk_barrier_spins(0)
    try:
        seen = 0
        for _ in range(3):
            layer.select()
            torch.cuda.synchronize()
            idx = layer.idx.cpu().numpy()
            for (b, t), (ridx, rs) in ref.items():
                check_topk(idx[b, t], ridx, rs, where=f"row {(b, t)} after a timed-out meeting")
            ev = C.check_device_errors()
            assert ev & ~C.DEV_TOPK_BARRIER == 0, ev
            seen |= ev
        assert seen & C.DEV_TOPK_BARRIER
    finally:
        C.debug_topk_barrier_spins(old)
    # the default limit again: exact, and nothing recorded
    layer.select()
    torch.cuda.synchronize()
    idx = layer.idx.cpu().numpy()
    for (b, t), (ridx, rs) in ref.items():
        check_topk(idx[b, t], ridx, rs, where=f"row {(b, t)}")
    assert C.check_device_errors() == 0


@pytest.mark.parametrize("T", [9_999, 100_003, 1_000])
def test_nan_scores_mark_the_row_failed(C, T):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    # T = 1,000 has fewer visible entries than k: the all-visible path
    wl = W.get("parity_decode").with_(T=T)
    L = W.make_csa_layer(wl)
    Ld = to_device(L)
    Ld["head_w"][1, 0, 5] = float("nan")
    layer = CSALayer(Ld)
    layer.select()
    torch.cuda.synchronize()
    idx, sc = layer.idx.cpu().numpy(), layer.score.cpu().numpy()
    assert (idx[1, 0] == -1).all() and np.isnan(sc[1, 0]).all()
    ref = O.layer_indexer_topk(L, wl.k, rows=[(0, 0), (2, 0)])
    for (b, t), (ridx, rs) in ref.items():
        check_topk(idx[b, t], ridx, rs, where=f"healthy row {(b, t)}")
    assert C.check_device_errors() == C.DEV_ROW_FAILED
    assert C.check_device_errors() == 0
