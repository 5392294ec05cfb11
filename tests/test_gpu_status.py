"""Device-side failure reporting, made to happen without a GPU fault: the
top-k meeting point is given a poll limit of zero (a CTA that arrives first
gives up at once), a test hook makes the first scoring CTA miss one key tile
(nothing is left in flight) so that its bounded waits run out, and a NaN
head weight makes one query row unrankable.  The kernels must return, record the event in the
device status word, and leave the affected row visibly failed (-1 indices,
NaN scores) and every other row exact."""
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


@pytest.mark.parametrize("Tq,ik_fmt", [(1, "e4m3vec"), (4, "e4m3vec"), (1, "mxfp4")])
def test_scoring_wait_runs_out_and_the_row_is_reported(C, Tq, ik_fmt):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    # the hook makes the first scoring CTA miss its first key tile and bounds
    # its waits to a few thousand polls: the kernel returns, the CTA's scores
    # read NaN, its query rows are reported failed (row 0; with several rows
    # per sequence, the CTA's group: every row of sequence 0 here), the
    # other rows are exact
    wl = W.get("parity_decode").with_(Tq=Tq, prefill=Tq > 1, ik_fmt=ik_fmt)
    L = W.make_csa_layer(wl)
    layer = CSALayer(to_device(L))
    rows = [(b, t) for b in range(wl.B) for t in range(wl.Tq)]
    failed = [(0, t) for t in range(wl.Tq)]
    ref = O.layer_indexer_topk(L, wl.k, rows=[r for r in rows if r not in failed])
    old = C.debug_indexer_stall(4096)
    try:
        layer.select()
        torch.cuda.synchronize()
    finally:
        C.debug_indexer_stall(old)
    idx, sc = layer.idx.cpu().numpy(), layer.score.cpu().numpy()
    for b, t in failed:
        assert (idx[b, t] == -1).all() and np.isnan(sc[b, t]).all(), (b, t)
    for (b, t), (ridx, rs) in ref.items():
        check_topk(idx[b, t], ridx, rs, where=f"row {(b, t)} beside a stalled one")
    assert C.check_device_errors() == C.DEV_INDEXER_WAIT | C.DEV_ROW_FAILED
    # the hook off: every row exact, nothing recorded
    layer.select()
    torch.cuda.synchronize()
    idx = layer.idx.cpu().numpy()
    ref0 = O.layer_indexer_topk(L, wl.k, rows=failed)
    for (b, t), (ridx, rs) in ref0.items():
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
