"""The parity record of bench.py (its `parity` object) on the host: the
oracle's own answer to a decode query passes with zero error, and planted
mistakes in the answer fail it the way the tests' rules say (a selection
swap beyond the near-tie band, an output error above 2e-3 of the RMS, an LSE
error above 1e-4)."""
import numpy as np
import pytest

import workloads as W


@pytest.fixture(scope="module")
def query():
    import bench
    wl = W.get("parity_decode").with_(B=2)
    Lc, Lh = W.make_csa_layer(wl), W.make_hca_layer(wl)
    trace = []
    first = bench.oracle_query(Lc, Lh, trace=trace)
    k = wl.k
    idx = np.full((wl.B, 1, k), -1, dtype=np.int32)
    for b, (_, sel) in enumerate(trace):
        idx[b, 0] = sel
    # the oracle's answer in the library's layout
    c_o = np.stack([first[2 * b][0] for b in range(wl.B)])[:, None]
    c_l = np.stack([first[2 * b][1] for b in range(wl.B)])[:, None]
    h_o = np.stack([first[2 * b + 1][0] for b in range(wl.B)])[:, None]
    h_l = np.stack([first[2 * b + 1][1] for b in range(wl.B)])[:, None]
    return bench, Lc, trace, first, (idx, c_o, c_l, h_o, h_l)


def test_the_oracles_own_answer_passes(query):
    bench, Lc, trace, first, got = query
    rec = bench.parity_record(Lc, got, trace, first)
    assert rec["pass"] and rec["topk_swaps"] == 0 and rec["topk_far"] == 0
    assert rec["csa_max_err_over_rms"] < 1e-12 and rec["hca_max_err_over_rms"] < 1e-12
    assert rec["max_lse_err"] < 1e-12


def test_a_far_swap_fails(query):
    bench, Lc, trace, first, (idx, c_o, c_l, h_o, h_l) = query
    s, sel = trace[0]
    picked = set(sel[sel >= 0].tolist())
    # the lowest-scoring visible entry that was not selected replaces the best one
    order = np.argsort(s)
    out = next(int(j) for j in order if int(j) not in picked)
    best = int(sel[np.argmax(s[sel[sel >= 0]])])
    bad = idx.copy()
    row = bad[0, 0]
    row[row == best] = out
    row[: (row >= 0).sum()] = np.sort(row[row >= 0])
    rec = bench.parity_record(Lc, (bad, c_o, c_l, h_o, h_l), trace, first)
    assert rec["topk_far"] >= 1 and not rec["pass"]


def test_output_and_lse_errors_fail(query):
    bench, Lc, trace, first, (idx, c_o, c_l, h_o, h_l) = query
    rms = np.sqrt(np.mean(h_o[1, 0] ** 2))
    h_bad = h_o.copy()
    h_bad[1, 0, 3, 7] += 3e-3 * rms
    rec = bench.parity_record(Lc, (idx, c_o, c_l, h_bad, h_l), trace, first)
    assert 2e-3 < rec["hca_max_err_over_rms"] and not rec["pass"]
    c_bad = c_l.copy()
    c_bad[0, 0, 5] += 2e-4
    rec = bench.parity_record(Lc, (idx, c_o, c_bad, h_o, h_l), trace, first)
    assert rec["max_lse_err"] > 1e-4 and not rec["pass"]
    # within the bounds: still a pass
    h_ok = h_o.copy()
    h_ok[1, 0, 3, 7] += 1e-3 * rms
    assert bench.parity_record(Lc, (idx, c_o, c_l, h_ok, h_l), trace, first)["pass"]
