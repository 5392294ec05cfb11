"""indexer_topk_noalloc: the indexer top-k for callers that cannot allocate a
workspace (a framework owning all device memory, an allocation-free real-time
loop, an op interface without scratch).  It must give the same selection as
indexer_topk with a caller workspace, call after call, although every call
reuses the library's one fixed scratch array.  This file is collected last so
that a failure here comes after every other test has run."""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
from gpu_common import require_gpu, to_device
from parity import check_topk

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice():
    C = require_gpu()
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    wl = W.get("parity_decode")
    Ld = to_device(W.make_csa_layer(wl))
    ref = CSALayer(Ld)                      # existing entry point, caller workspace
    ref.select()
    torch.cuda.synchronize()
    ref_idx = ref.idx.cpu().numpy()
    ref_sc = ref.score.cpu().numpy()
    for call in range(2):
        idx = torch.full_like(ref.idx, -7)
        sc = torch.full_like(ref.score, float("nan"))
        C.indexer_topk_noalloc(wl.B, wl.Tq, Ld["q_pos"], Ld["q_ik"], Ld["q_ik_scale"],
                               Ld["head_w"], wl.H_I, wl.d_I, Ld["comp_ik"], wl.csa_stride, wl.k,
                               ref.max_entries, idx, sc)
        torch.cuda.synchronize()
        got_idx, got_sc = idx.cpu().numpy(), sc.cpu().numpy()
        for b in range(wl.B):
            # same kernels on the same inputs: the selection must be identical,
            # which is inside the top-k tolerance the parity tests use
            n_vis = ref.max_entries
            dense = np.full(n_vis, -np.inf)
            sel = ref_idx[b, 0][ref_idx[b, 0] >= 0]
            dense[sel] = ref_sc[b, 0][: sel.size]
            check_topk(got_idx[b, 0], ref_idx[b, 0], dense, where=f"noalloc call {call}")
            assert np.array_equal(got_idx[b, 0], ref_idx[b, 0])
            assert np.allclose(got_sc[b, 0], ref_sc[b, 0], rtol=0, atol=0, equal_nan=True)


def test_noalloc_rejects_requests_beyond_its_scratch():
    C = require_gpu()
    wl = W.get("parity_decode")
    Ld = to_device(W.make_csa_layer(wl))
    limit = C.noalloc_scratch_bytes()
    rows = limit // (4 * Ld["comp_ik"]["cap"]) + 1       # one row more than fits
    big_pos = torch.zeros(rows, 1, dtype=torch.int64, device="cuda")
    with pytest.raises(C.CskvError) as e:
        C.indexer_topk_noalloc(rows, 1, big_pos, Ld["q_ik"], Ld["q_ik_scale"], Ld["head_w"],
                               wl.H_I, wl.d_I, Ld["comp_ik"], wl.csa_stride, wl.k,
                               Ld["comp_ik"]["cap"], torch.empty(1, device="cuda"), None)
    assert e.value.status == C.ERR_SCRATCH_LIMIT
