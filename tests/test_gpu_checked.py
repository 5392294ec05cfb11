"""The checked build (libcskv_check.so, loaded with CSKV_CHECK=1).

* The whole GPU suite runs again on the checked build in a child process:
  every parity case passes there too, and no valid call records an
  out-of-range index (the suite's conftest reads the status word after each
  GPU test of a checked run).
* The attention parity cases run again with the split count forced
  (CSKV_SPLITS=1 and 5), which moves decode rows onto the kernel variants
  that run several units per CTA.
* Inputs whose device-side indices break the documented ranges (a selected
  entry past the row's visible count or the cache, a visible slot with a bad
  block-table entry, positions that need more entries than the compressor's
  host bound or its caches, ring positions already overwritten, a negative
  ring position, a row with more visible entries than max_entries) record
  DEV_BOUNDS in the checked build, and the access is left out.  These run only
  on the checked build, whose kernels test every such index before using it;
  the regular build's kernels leave the same accesses out (or keep them inside
  the planes) without recording them, which the file's last comment lists."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_common import require_gpu, to_device

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def C():
    C = require_gpu()
    C.check_device_errors()          # start from a clear status word
    return C


@pytest.fixture
def CK(C):
    if not C.build_checked():
        pytest.skip("runs on the checked build (CSKV_CHECK=1, see the suite test)")
    C.check_device_errors()
    return C


def test_checked_build_runs_the_gpu_suite(C):
    if C.build_checked():
        pytest.skip("already the checked build")
    env = dict(os.environ, CSKV_CHECK="1")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests"), "-m", "gpu",
                        "-x", "-q", "-p", "no:cacheprovider",
                        "--deselect", "tests/test_gpu_checked.py::test_checked_build_runs_the_gpu_suite",
                        "--deselect", "tests/test_gpu_checked.py::test_forced_split_counts_keep_parity"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-30:])
    assert r.returncode == 0, tail
    # the summary line: everything passed there, the bad-index cases included
    # (nothing skipped on the checked build)
    summary = [ln for ln in r.stdout.splitlines() if " passed" in ln][-1]
    assert int(summary.split(" passed")[0].split()[-1]) >= 130, summary
    assert "failed" not in summary and "skipped" not in summary, summary


@pytest.mark.parametrize("splits", ["1", "5"])
def test_forced_split_counts_keep_parity(C, splits):
    # CSKV_SPLITS (a tuning switch) moves the decode rows onto other kernel
    # instantiations: one CTA running every unit of a row in sequence, or a
    # few units per CTA; the attention parity cases must hold there too
    if os.environ.get("CSKV_SPLITS") or C.build_checked():
        pytest.skip("runs from the regular build's suite")
    env = dict(os.environ, CSKV_SPLITS=splits)
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests",
                                                                     "test_gpu_parity.py"),
                        "-m", "gpu", "-x", "-q", "-p", "no:cacheprovider", "-k",
                        "attention or window_only or dense_small or holes or multi_token"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-30:])
    assert r.returncode == 0, tail
    summary = [ln for ln in r.stdout.splitlines() if " passed" in ln][-1]
    assert int(summary.split(" passed")[0].split()[-1]) >= 10, summary
    assert "failed" not in summary, summary


# ------------------------------------------------------------ bad indices

def _bounds(C):
    ev = C.check_device_errors()
    assert ev & C.DEV_BOUNDS, f"no bounds event recorded ({ev:#x})"
    assert not ev & ~C.DEV_BOUNDS, f"unexpected events {ev:#x}"


def _csa_sel(L, k):
    wl = L["wl"]
    sel = np.full((wl.B, wl.Tq, k), -1, dtype=np.int32)
    for (b, t), (idx, _) in O.layer_indexer_topk(L, k).items():
        sel[b, t] = idx
    return sel


@pytest.mark.bounds_events
@pytest.mark.parametrize("ik_fmt", ["e4m3vec"])
def test_selected_entry_past_the_visible_count_is_left_out(CK, ik_fmt):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    wl = W.get("parity_decode").with_(ik_fmt=ik_fmt)
    L = W.make_csa_layer(wl)
    layer = CSALayer(to_device(L))
    sel = _csa_sel(L, wl.k)
    n_vis = int(L["ctx_len"][0]) // L["stride"]
    # the reference call: the offending entries given as -1 (no entry)
    good = sel.copy()
    good[0, 0, :3] = -1
    out_ref, lse_ref = (t.clone() for t in layer.attend(torch.from_numpy(good).cuda()))
    assert CK.check_device_errors() == 0
    bad = sel.copy()
    bad[0, 0, :3] = [n_vis, n_vis + 7, -5]      # past the visible count / cache; below -1
    out, lse = layer.attend(torch.from_numpy(bad).cuda())
    torch.cuda.synchronize()
    _bounds(CK)
    assert torch.equal(out, out_ref) and torch.equal(lse, lse_ref)


@pytest.mark.bounds_events
def test_visible_slot_with_a_bad_block_is_reported(CK):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer, HCALayer
    wl = W.get("parity_decode")
    # dense HCA attention over a paged cache whose first block id is out of range
    Lh = W.make_hca_layer(wl)
    Lh["comp_k"] = W.page_cache(Lh["comp_k"], 16, seed=3)
    Lhd = to_device(Lh)
    Lhd["comp_k"]["block_table"][0, 0] = int(Lhd["comp_k"]["num_blocks"]) + 3
    out, lse = HCALayer(Lhd, max_entries=Lh["comp_k"]["cap"]).attend()
    torch.cuda.synchronize()
    _bounds(CK)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    # the indexer over paged keys (tensor-core path: 128-entry blocks) whose
    # visible first block has no block (-1)
    Lc = W.make_csa_layer(wl)
    Lc["comp_ik"] = W.page_cache(Lc["comp_ik"], 128, seed=4)
    Lcd = to_device(Lc)
    Lcd["comp_ik"]["block_table"][1, 0] = -1
    layer = CSALayer(Lcd)
    layer.select()
    torch.cuda.synchronize()
    _bounds(CK)
    assert torch.isfinite(layer.score[layer.idx >= 0]).all()


@pytest.mark.bounds_events
def test_compressor_positions_past_the_cache_and_the_host_bound(CK):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    wl = W.get("tiny").with_(B=2, T=4096 + 7)
    L = W.make_csa_layer(wl, ring_cap=1024)
    Ld = to_device(L)
    cap, S = L["comp_k"]["cap"], L["stride"]
    before = Ld["comp_k"]["data"][1].clone()
    layer = CSALayer(Ld)
    # sequence 0: two entries below the cap and two past it (sequence 1's rows
    # in the planes); sequence 1: nothing new
    te = cap * S + 8
    layer.compress(torch.tensor([te - 16, 0], device="cuda"), torch.tensor([te, 0], device="cuda"),
                   4)
    torch.cuda.synchronize()
    _bounds(CK)
    assert torch.equal(Ld["comp_k"]["data"][1], before)
    # ten entries for a host bound of two: the first two are written
    T = wl.T
    layer.compress(torch.tensor([T - 40, T], device="cuda"), torch.tensor([T, T], device="cuda"),
                   2)
    torch.cuda.synchronize()
    _bounds(CK)


@pytest.mark.bounds_events
def test_compressor_ring_positions_already_overwritten(CK):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    # a ring of 8 slots (the host bound for one CSA entry) that already holds
    # three tokens past the entry: its first positions are gone
    wl = W.get("tiny").with_(T=403)
    L = W.make_csa_layer(wl, ring_cap=8)
    layer = CSALayer(to_device(L))
    layer.compress(torch.tensor([396], device="cuda"), torch.tensor([403], device="cuda"), 1)
    torch.cuda.synchronize()
    _bounds(CK)


@pytest.mark.bounds_events
def test_ring_store_negative_position_is_left_out(CK):
    B, cap = 2, 128
    g = torch.Generator().manual_seed(2)

    def cache(n, ring):
        return {"fmt": "f32", "d_nope": 64, "d_rope": 64, "ring": ring, "cap": n,
                "data": torch.randn(B, n, 128, generator=g)}
    ring, src = to_device(cache(cap, True)), to_device(cache(1, False))
    before = ring["data"].clone()
    CK.ring_store(B, torch.tensor([-3, 5], device="cuda"), [src], [ring])
    torch.cuda.synchronize()
    _bounds(CK)
    want = before.clone()
    want[1, 5] = src["data"][1, 0]
    assert torch.equal(ring["data"], want)


@pytest.mark.bounds_events
def test_row_with_more_visible_entries_than_max_entries(CK):
    from compressed_sparse_kv_softmax_b200.layer import CSALayer
    wl = W.get("parity_decode")
    L = W.make_csa_layer(wl)
    layer = CSALayer(to_device(L), max_entries=1000)   # rows see 2,499 entries
    layer.select()
    torch.cuda.synchronize()
    _bounds(CK)
    assert int(layer.idx.max()) < 1000


# What the regular build does with the same inputs (read from its kernels):
# a selected entry outside [0, cap) is skipped, one in [visible, cap) is
# attended; a block id outside [0, num_blocks) is clamped into the pool and a
# tile of scoring keys with no block is read as zeros past the planes, scales
# included; the compressor writes no entry past a cache's cap, with no block,
# or past max_new per sequence; a negative ring_store position writes
# nothing; a row's visible entries stop at max_entries.
