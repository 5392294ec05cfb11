"""Parity at the measured workloads' full sizes, in the launch configuration
the bench uses: every row of the decode workloads (8 x 65,536, 4 x 131,072,
1 x 1,048,576 tokens), and 64 sampled rows of the 8,192-token prefill chunk on
a 1,048,576-token context."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_common import require_gpu, sample_rows
from parity import check_attention, check_topk

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def C():
    return require_gpu()


@pytest.mark.parametrize("name", ["flash", "pro", "long", "prefill"])
def test_indexer_topk_full_size(C, name):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    wl = W.get(name)
    L = W.make_csa_layer(wl, device="cuda")
    layer = CSALayer(L)
    layer.select()
    torch.cuda.synchronize()
    rows = sample_rows(wl.B, wl.Tq)
    idx = layer.idx.cpu().numpy()
    swaps = 0
    for (b, t), (ridx, rs) in O.layer_indexer_topk(L, wl.k, rows=rows).items():
        swaps += check_topk(idx[b, t], ridx, rs, where=f"{name} row {(b, t)}")
    # sanity, not parity: most planted needles score high enough to be selected
    found = total = 0
    for b in range(wl.B if not wl.prefill else 0):
        sel = set(idx[b, 0].tolist())
        for p in L["needles"][b].tolist():
            total += 1
            found += (p // wl.csa_stride) in sel
    assert total == 0 or found >= total // 2, f"{found}/{total} needles selected"


@pytest.mark.parametrize("name", ["flash", "pro", "long"])
def test_decode_attention_full_size(C, name):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer, HCALayer
    wl = W.get(name)
    Lc = W.make_csa_layer(wl, device="cuda")
    ref_sel = O.layer_indexer_topk(Lc, wl.k)
    sel = np.full((wl.B, 1, wl.k), -1, dtype=np.int32)
    for (b, t), (ridx, _) in ref_sel.items():
        sel[b, t] = ridx
    csa = CSALayer(Lc)
    out, lse = csa.attend(torch.from_numpy(sel).cuda())
    torch.cuda.synchronize()
    ref = O.layer_attention(Lc, sel=sel)
    rows = sorted(ref)
    check_attention(np.stack([out[r].cpu().numpy() for r in rows]),
                    np.stack([lse[r].cpu().numpy() for r in rows]),
                    np.stack([ref[r][0] for r in rows]), np.stack([ref[r][1] for r in rows]),
                    where=f"{name} csa")
    Lh = W.make_hca_layer(wl, device="cuda")
    hca = HCALayer(Lh)
    out, lse = hca.attend()
    torch.cuda.synchronize()
    ref = O.layer_attention(Lh, sel=None)
    check_attention(np.stack([out[r].cpu().numpy() for r in rows]),
                    np.stack([lse[r].cpu().numpy() for r in rows]),
                    np.stack([ref[r][0] for r in rows]), np.stack([ref[r][1] for r in rows]),
                    where=f"{name} hca")


def test_prefill_sparse_attention_full_size(C):
    """8,192 query rows on a 1,048,576-token context, each with its own 1,024
    selected entries plus its causal window; 64 sampled rows checked."""
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    wl = W.get("prefill")
    L = W.make_csa_layer(wl, device="cuda")
    sel = W.random_selection(wl, wl.k, device="cuda")
    layer = CSALayer(L)
    out, lse = layer.attend(sel)
    torch.cuda.synchronize()
    rows = sample_rows(wl.B, wl.Tq)
    ref = O.layer_attention(L, sel=sel.cpu().numpy(), rows=rows)
    check_attention(np.stack([out[r].cpu().numpy() for r in rows]),
                    np.stack([lse[r].cpu().numpy() for r in rows]),
                    np.stack([ref[r][0] for r in rows]), np.stack([ref[r][1] for r in rows]),
                    where="prefill csa")


def test_prefill_dense_attention_full_size(C):
    """HCA over the same 8,192-token chunk: each row attends every compressed
    entry it can see (about 8,200) plus its causal window, so every row runs
    its whole key list through one CTA's online softmax; 64 sampled rows."""
    from compressed_sparse_kv_softmax_b200.layer import HCALayer
    wl = W.get("prefill")
    L = W.make_hca_layer(wl, device="cuda")
    layer = HCALayer(L)
    out, lse = layer.attend()
    torch.cuda.synchronize()
    rows = sample_rows(wl.B, wl.Tq)
    ref = O.layer_attention(L, sel=None, rows=rows)
    check_attention(np.stack([out[r].cpu().numpy() for r in rows]),
                    np.stack([lse[r].cpu().numpy() for r in rows]),
                    np.stack([ref[r][0] for r in rows]), np.stack([ref[r][1] for r in rows]),
                    where="prefill hca")
