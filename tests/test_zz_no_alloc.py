"""indexer_topk_noalloc: the indexer top-k for callers that cannot allocate a
workspace (a framework owning all device memory, an allocation-free real-time
loop, an op interface without scratch).  It must give the same selection as
indexer_topk with a caller workspace, call after call, although every call
reuses the library's one fixed scratch array - also when a call of another
shape used the array in between.  This file is collected last so that a
failure here comes after every other test has run."""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_common import require_gpu, to_device

pytestmark = pytest.mark.gpu


def _noalloc(C, wl, Ld, max_entries, like):
    idx = torch.full_like(like.idx, -7)
    sc = torch.full_like(like.score, float("nan"))
    C.indexer_topk_noalloc(wl.B, wl.Tq, Ld["q_pos"], Ld["q_ik"], Ld["q_ik_scale"], Ld["head_w"],
                           wl.H_I, wl.d_I, Ld["comp_ik"], wl.csa_stride, wl.k, max_entries, idx,
                           sc)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), sc.cpu().numpy()


def _same(got, ref, where):
    # same kernels on the same inputs: the selection and its scores are
    # identical to the workspace entry point's (inside the parity tolerance)
    gi, gs = got
    ri, rs = ref
    assert np.array_equal(gi, ri), where
    assert np.array_equal(gs, rs, equal_nan=True), where


def test_noalloc_matches_workspace_entry_point_twice():
    C = require_gpu()
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    wl = W.get("parity_decode")
    Ld = to_device(W.make_csa_layer(wl))
    ref = CSALayer(Ld)                      # existing entry point, fresh workspace
    ref.select()
    torch.cuda.synchronize()
    want = (ref.idx.cpu().numpy(), ref.score.cpu().numpy())
    # a call of another shape (40 rows of one sequence, other entry count)
    wl2 = W.get("parity_prefill").with_(Tq=40)
    Ld2 = to_device(W.make_csa_layer(wl2))
    ref2 = CSALayer(Ld2)
    ref2.select()
    torch.cuda.synchronize()
    want2 = (ref2.idx.cpu().numpy(), ref2.score.cpu().numpy())
    _same(_noalloc(C, wl, Ld, ref.max_entries, ref), want, "noalloc call 1")
    _same(_noalloc(C, wl2, Ld2, ref2.max_entries, ref2), want2, "noalloc call of another shape")
    _same(_noalloc(C, wl, Ld, ref.max_entries, ref), want, "noalloc call 2")


@pytest.mark.parametrize("ik_fmt,bs", [("e4m3vec", 256), ("mxfp4", 128), ("e4m3vec", 32)])
def test_noalloc_on_paged_keys_matches_workspace_entry_point(ik_fmt, bs):
    # a paged indexer-key cache (block table, a tail block without a pool
    # block) through the fixed scratch: the same selection as with a
    # workspace (tensor-core scoring for blocks of 128 or more, the CUDA-core
    # kernel for smaller ones)
    C = require_gpu()
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    wl = W.get("parity_decode").with_(ik_fmt=ik_fmt)
    L = W.make_csa_layer(wl)
    L["comp_ik"] = W.page_cache(L["comp_ik"], bs, seed=bs, unmapped_tail=1)
    Ld = to_device(L)
    ref = CSALayer(Ld)
    ref.select()
    torch.cuda.synchronize()
    want = (ref.idx.cpu().numpy(), ref.score.cpu().numpy())
    _same(_noalloc(C, wl, Ld, ref.max_entries, ref), want, f"noalloc paged {ik_fmt} bs {bs}")


def test_noalloc_limit_is_the_workspace_size():
    C = require_gpu()
    wl = W.get("parity_decode")
    Ld = to_device(W.make_csa_layer(wl))
    limit = C.noalloc_scratch_bytes()
    cap = Ld["comp_ik"]["cap"]
    rows = 1
    while C.indexer_workspace_size(rows + 1, 1, cap, wl.k) <= limit:
        rows += 1
    # the largest request that fits is accepted (queries at position 0 see
    # no entry, so only the rows' padding is written) ...
    pos = torch.zeros(rows, 1, dtype=torch.int64, device="cuda")
    qik = torch.zeros(rows, 1, wl.H_I, wl.d_I, dtype=torch.uint8, device="cuda")
    qs = torch.ones(rows, 1, wl.H_I, dtype=torch.float32, device="cuda")
    hw = torch.ones(rows, 1, wl.H_I, dtype=torch.float32, device="cuda")
    ik = dict(Ld["comp_ik"])
    ik["data"] = torch.zeros(rows, cap, wl.d_I, dtype=torch.uint8, device="cuda")
    ik["scale"] = torch.ones(rows, cap, 1, dtype=torch.float32, device="cuda")
    idx = torch.full((rows, 1, wl.k), 7, dtype=torch.int32, device="cuda")
    C.indexer_topk_noalloc(rows, 1, pos, qik, qs, hw, wl.H_I, wl.d_I, ik, wl.csa_stride, wl.k,
                           cap, idx, None)
    torch.cuda.synchronize()
    assert (idx == -1).all()
    # ... one row more is refused before anything is enqueued
    with pytest.raises(C.CskvError) as e:
        C.indexer_topk_noalloc(rows + 1, 1, torch.zeros(rows + 1, 1, dtype=torch.int64,
                                                        device="cuda"),
                               qik, qs, hw, wl.H_I, wl.d_I, ik, wl.csa_stride, wl.k, cap, idx,
                               None)
    assert e.value.status == C.ERR_SCRATCH_LIMIT
