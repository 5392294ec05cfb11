"""Paged compressed caches (block tables) on the GPU: every kernel that reads
or writes a compressed cache - the scoring kernels (FP8 per-vector and
per-64, MXFP4; one and several query rows), the CUDA-core scoring fall-back
(blocks under 128 entries), sparse and dense attention (bulk-copied runs for
blocks of 64 or more, gathered rows otherwise; decode and prefill), the
compressor - on a paged copy of a generated cache, against the oracle on the
contiguous original.  Every table ends in a block with no pool block (-1)."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_common import require_gpu, sample_rows, to_device
from parity import check_attention, check_compressed_e4m3, check_compressed_mxfp4, check_topk

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C():
    return require_gpu()


def _paged(L, keys, bs, tail=1):
    Lp = dict(L)
    for i, key in enumerate(keys):
        if L.get(key) is not None:
            Lp[key] = W.page_cache(L[key], bs, seed=17 * bs + i, unmapped_tail=tail)
    return Lp


@pytest.mark.parametrize("name,ik_fmt,bs", [
    ("parity_decode", "e4m3vec", 128), ("parity_decode", "e4m3vec", 256),
    ("parity_decode", "e4m3vec", 64), ("parity_decode", "e4m3", 128),
    ("parity_decode", "mxfp4", 128), ("parity_decode", "mxfp4", 32),
    ("parity_prefill", "e4m3vec", 128), ("parity_prefill", "mxfp4", 256)])
def test_indexer_on_paged_keys(C, name, ik_fmt, bs):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    wl = W.get(name).with_(ik_fmt=ik_fmt)
    L = W.make_csa_layer(wl)
    layer = CSALayer(to_device(_paged(L, ["comp_ik"], bs)))
    layer.select()
    torch.cuda.synchronize()
    idx, sc = layer.idx.cpu().numpy(), layer.score.cpu().numpy()
    ref = O.layer_indexer_topk(L, wl.k, rows=sample_rows(wl.B, wl.Tq))
    for (b, t), (ridx, rs) in ref.items():
        check_topk(idx[b, t], ridx, rs, where=f"{name} {ik_fmt} bs {bs} row {(b, t)}")
        sel = idx[b, t][idx[b, t] >= 0]
        assert np.allclose(sc[b, t][: sel.size], rs[sel], rtol=1e-4, atol=1e-4 * np.abs(rs).max())
    assert C.check_device_errors() == 0


def _oracle_sel(L, k):
    wl = L["wl"]
    ref = O.layer_indexer_topk(L, k)
    sel = np.full((wl.B, wl.Tq, k), -1, dtype=np.int32)
    for (b, t), (idx, _) in ref.items():
        sel[b, t] = idx
    return sel


@pytest.mark.parametrize("name,kind,bs", [
    ("parity_decode", "hca", 64), ("parity_decode", "hca", 16), ("parity_decode", "csa", 16),
    ("parity_decode", "csa", 128), ("parity_prefill", "hca", 64), ("parity_prefill", "csa", 32)])
def test_attention_on_paged_entries(C, name, kind, bs):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer, HCALayer
    wl = W.get(name)
    if kind == "hca":
        L = W.make_hca_layer(wl)
        out, lse = HCALayer(to_device(_paged(L, ["comp_k"], bs)),
                            max_entries=L["comp_k"]["cap"]).attend()
        sel = None
    else:
        L = W.make_csa_layer(wl)
        sel = _oracle_sel(L, wl.k)
        out, lse = CSALayer(to_device(_paged(L, ["comp_k"], bs))).attend(
            torch.from_numpy(sel).cuda())
    torch.cuda.synchronize()
    rows = sample_rows(wl.B, wl.Tq)
    ref = O.layer_attention(L, sel=sel, rows=rows)
    check_attention(np.stack([out[b, t].cpu().numpy() for b, t in rows]),
                    np.stack([lse[b, t].cpu().numpy() for b, t in rows]),
                    np.stack([ref[r][0] for r in rows]), np.stack([ref[r][1] for r in rows]),
                    where=f"{name} {kind} bs {bs}")
    assert C.check_device_errors() == 0


def _logical(c, key):
    """The planes of a paged GPU cache gathered back to [B][cap][...]."""
    bt = c["block_table"].long().cpu()
    bs = int(c["block_size"])
    rows = (bt.clamp(min=0)[:, :, None] * bs + torch.arange(bs)[None, None, :]).reshape(
        bt.shape[0], -1)
    out = dict(c)
    for plane in ("data", "scale", "rope"):
        if c.get(plane) is not None:
            out[plane] = c[plane][0].cpu()[rows]
    return out


@pytest.mark.parametrize("kind,ik_fmt,bs", [("csa", "e4m3vec", 16), ("csa", "mxfp4", 128),
                                            ("hca", "e4m3vec", 8)])
def test_compressor_writes_paged_entries(C, kind, ik_fmt, bs):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer, HCALayer
    wl = W.get("parity_decode").with_(ik_fmt=ik_fmt)
    mk = W.make_csa_layer if kind == "csa" else W.make_hca_layer
    L = mk(wl, ring_cap=1024)
    Ld = to_device(_paged(L, ["comp_k", "comp_ik"], bs))
    T = wl.T
    t_begin, t_end = [T - 600, T - 1, T - 257], [T, T, T - 1]
    S = L["stride"]
    max_new = max(e // S - b // S for b, e in zip(t_begin, t_end))
    layer = CSALayer(Ld) if kind == "csa" else HCALayer(Ld)
    layer.compress(torch.tensor(t_begin, device="cuda"), torch.tensor(t_end, device="cuda"),
                   max(max_new, 1))
    torch.cuda.synchronize()
    res = O.layer_compress(L, t_begin, t_end)
    kv = _logical(Ld["comp_k"], "comp_k")
    ik = _logical(Ld["comp_ik"], "comp_ik") if kind == "csa" else None
    n = 0
    for b, r in enumerate(res):
        if not len(r["j"]):
            continue
        check_compressed_e4m3(kv, b, r["j"], r["k"], r["k_mag"], wl.d_nope, where=f"b{b} kv")
        if ik is not None and ik_fmt == "mxfp4":
            check_compressed_mxfp4(ik, b, r["j"], r["ik"], r["ik_mag"], wl.d_I, where=f"b{b} ik")
        elif ik is not None:
            check_compressed_e4m3(ik, b, r["j"], r["ik"], r["ik_mag"], wl.d_I, where=f"b{b} ik")
        n += len(r["j"])
    assert n > 0
    assert C.check_device_errors() == 0


def test_paged_full_size_decode_row(C):
    # the 1M-context decode workload with 256-entry blocks for the indexer
    # keys and 64-entry blocks for the KV entries: a row's top-k and both
    # attention layers against the oracle
    from compressed_sparse_kv_softmax_b200.layer import CSALayer, HCALayer
    wl = W.get("long")
    Lc = W.make_csa_layer(wl)
    Lcp = _paged(Lc, ["comp_ik"], 256)
    Lcp = _paged(Lcp, ["comp_k"], 64)
    csa = CSALayer(to_device(Lcp))
    csa.select()
    out, lse = csa.attend()
    torch.cuda.synchronize()
    ref = O.layer_indexer_topk(Lc, wl.k, rows=[(0, 0)])
    ridx, rs = ref[(0, 0)]
    check_topk(csa.idx[0, 0].cpu().numpy(), ridx, rs, where="1M paged row")
    sel = csa.idx.cpu().numpy()
    a = O.layer_attention(Lc, sel=sel, rows=[(0, 0)])[(0, 0)]
    check_attention(out[0, 0].cpu().numpy()[None], lse[0, 0].cpu().numpy()[None], a[0][None],
                    a[1][None], where="1M paged CSA")
    Lh = W.make_hca_layer(wl)
    hca = HCALayer(to_device(_paged(Lh, ["comp_k"], 64)), max_entries=Lh["comp_k"]["cap"])
    out, lse = hca.attend()
    torch.cuda.synchronize()
    a = O.layer_attention(Lh, sel=None, rows=[(0, 0)])[(0, 0)]
    check_attention(out[0, 0].cpu().numpy()[None], lse[0, 0].cpu().numpy()[None], a[0][None],
                    a[1][None], where="1M paged HCA")
    assert C.check_device_errors() == 0
