"""Comparison rules between the CUDA path and the oracle.

  * top-k: the GPU set G and the oracle set R (entries >= 0) have equal size;
    G lists distinct visible entries in ascending order, then -1 padding; any
    entry in G\\R or R\\G has an oracle score within 1e-3 * |s_(k)| of the
    oracle's k-th score s_(k) (a near-tie swap); otherwise the sets are equal.
  * attention: max |o - o_ref| <= 2e-3 * RMS(o_ref) over the call's output,
    and |lse - lse_ref| <= LSE_TOL.
  * re-quantised entries: every stored code / BF16 pattern is one that exact
    rounding produces for some input within the float32 evaluation-error bound
    (POOL_EPS * sum_r a_r |x_r|) of the oracle's float64 value; at least 99.9%
    equal the oracle's own rounding.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O

TOPK_REL = 1e-3
ATTN_REL = 2e-3
# Natural-log units (1e-4 absolute on lse).  Both attention paths keep about 22
# significant bits in every product: the CUDA-core path computes in fp32, the
# tensor-core path splits every operand that is not exact in FP16 into FP16
# hi + lo parts (relative error ~2^-22) and accumulates in fp32.  A logit
# sm_scale * q . k over D = 512 dims with |q|, |k| ~ sqrt(D) then carries an
# error of order 2^-22 * sm_scale * |q| |k| ~ 1e-5 at the largest logits, and
# lse = m + log(sum) inherits at most that plus the fp32 rounding of the sum.
LSE_TOL = 1e-4
# Float32 evaluation error of a pooled value c = sum_r a_r x_r, relative to
# its magnitude scale m = sum_r a_r |x_r|: the sum itself contributes about
# pool * 2^-24 * m, and an error dg in a gate logit g_r = w . k + b (D terms,
# |dg| ~ sqrt(D) * 2^-24 * sum_d |w_d k_d| ~ 1e-6 here) moves the weights by
# a_r * dg, i.e. c by at most dg * m.  POOL_EPS bounds both with margin.
POOL_EPS = 2e-5
REL_EPS = POOL_EPS


def check_topk(gpu_idx, ref_idx, ref_scores, where=""):
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    ref_idx = np.asarray(ref_idx, dtype=np.int64)
    n_vis = ref_scores.shape[0]
    R = ref_idx[ref_idx >= 0]
    G = gpu_idx[gpu_idx >= 0]
    assert G.size == R.size, f"{where}: {G.size} selected, oracle {R.size}"
    assert np.all(gpu_idx[: G.size] >= 0) and np.all(gpu_idx[G.size:] == -1), f"{where}: padding"
    assert np.all(np.diff(G) > 0), f"{where}: not strictly ascending"
    assert np.all(G < n_vis), f"{where}: entry beyond the visible range"
    gs, rs = set(G.tolist()), set(R.tolist())
    if gs == rs:
        return 0
    sk = ref_scores[R[-1]]
    tol = TOPK_REL * abs(sk)
    diff = (gs - rs) | (rs - gs)
    bad = [j for j in diff if abs(ref_scores[j] - sk) > tol]
    assert not bad, (f"{where}: {len(bad)} swaps beyond the near-tie band, e.g. entry {bad[0]} "
                     f"score {ref_scores[bad[0]]} vs k-th {sk}")
    return len(gs - rs)


def check_attention(out, lse, ref_o, ref_lse, where=""):
    out = np.asarray(out, dtype=np.float64)
    ref_o = np.asarray(ref_o, dtype=np.float64)
    rms = np.sqrt(np.mean(ref_o ** 2))
    err = np.max(np.abs(out - ref_o))
    assert np.all(np.isfinite(out)), f"{where}: non-finite output"
    assert err <= ATTN_REL * rms, f"{where}: max|o-ref| = {err:.3e} > {ATTN_REL} * RMS {rms:.3e}"
    lerr = np.max(np.abs(np.asarray(lse, dtype=np.float64) - ref_lse))
    assert lerr <= LSE_TOL, f"{where}: max|lse-ref| = {lerr:.3e}"
    return err / rms, lerr


def check_codes(got, y, encode, decode, dy, min_exact=0.999, where=""):
    """got: stored codes; y: oracle values in code units (float64); dy: the
    evaluation-error bound in code units.  Every code must be the rounding of
    some value in [y - dy, y + dy]: rounding is monotone, so those are exactly
    the codes whose values lie between the roundings of the two ends."""
    got = np.asarray(got)
    y = np.asarray(y, dtype=np.float64)
    ref = encode(y)
    lo, hi = decode(encode(y - dy)), decode(encode(y + dy))
    v = decode(got)
    ok = (got == ref) | ((v >= lo) & (v <= hi))
    assert np.all(ok), (f"{where}: {np.sum(~ok)} codes outside the rounding band, e.g. got "
                        f"{got[~ok][:4]} want {ref[~ok][:4]} for {y[~ok][:4]}")
    exact = np.mean(got == ref)
    assert exact >= min_exact, f"{where}: only {exact:.5f} of codes equal the oracle's"
    return exact


def bf16_bits(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def check_pooled_f32(got, ref_vals, ref_mag, where=""):
    err = np.abs(np.asarray(got, dtype=np.float64) - ref_vals)
    bound = POOL_EPS * ref_mag + 1e-30
    worst = np.max(err / bound)
    assert worst <= 1.0, f"{where}: pooled error {worst:.2f}x the fp32 evaluation bound"
    return worst


def check_compressed_e4m3(cache, b, js, ref_vals, ref_mag, d_nope, where=""):
    """cache: GPU planes (torch); ref_vals: oracle pooled float64 [n][D];
    ref_mag: sum_r a_r |x_r| per element (the error scale of each sum).
    The scale block is 64 elements, or the whole vector for "e4m3vec"."""
    js = np.asarray(js)
    codes = cache["data"][b, js].cpu().numpy()
    blk = O.scale_block(cache["fmt"], d_nope)
    nb = d_nope // blk
    scales = cache["scale"][b, js][:, :nb].cpu().double().numpy()
    blocks = [slice(blk * i, blk * (i + 1)) for i in range(nb)]
    amax = np.stack([np.max(np.abs(ref_vals[:, s_]), axis=1) for s_ in blocks], axis=1)
    mmax = np.stack([np.max(ref_mag[:, s_], axis=1) for s_ in blocks], axis=1)
    ref_s = np.where(amax > 0, amax / 448.0, 1.0)
    # amax moves by at most POOL_EPS * (largest magnitude scale in the block)
    s_tol = POOL_EPS * np.where(amax > 0, mmax / np.maximum(amax, 1e-300), 0.0) + 1e-7
    serr = np.abs(scales / ref_s - 1.0)
    assert np.all(serr <= s_tol), f"{where}: scale rel err {np.max(serr):.3e}"
    s_el = np.repeat(scales, blk, axis=1)
    y = ref_vals[:, :d_nope] / s_el
    dy = POOL_EPS * ref_mag[:, :d_nope] / s_el
    exact = check_codes(codes, y, O.e4m3_encode, O.e4m3_decode, dy, where=where + " e4m3")
    d_rope = ref_vals.shape[1] - d_nope
    if d_rope:
        rope = bf16_bits(cache["rope"][b, js])
        check_codes(rope, ref_vals[:, d_nope:], O.bf16_encode, O.bf16_decode,
                    POOL_EPS * ref_mag[:, d_nope:], where=where + " bf16")
    return exact, float(np.max(serr)) if serr.size else 0.0


def check_compressed_mxfp4(cache, b, js, ref_vals, ref_mag, d_nope, where=""):
    """MXFP4 entries (packed E2M1 codes, one E8M0 exponent per 32 dims):
    every block's exponent X must be floor(log2 amax) - 2 for an amax inside
    the float32 evaluation band of the oracle's block maximum, and every code
    the E2M1 rounding of a value inside the band of the oracle's value divided
    by 2^X; at least 99.9% of the codes equal the oracle's own rounding."""
    js = np.asarray(js)
    packed = cache["data"][b, js].cpu().numpy()
    exps = cache["scale"][b, js][:, : d_nope // 32].cpu().numpy().astype(np.int64)
    X = exps - 127
    y = ref_vals[:, :d_nope].reshape(len(js), d_nope // 32, 32)
    dy = POOL_EPS * ref_mag[:, :d_nope].reshape(len(js), d_nope // 32, 32)
    amax = np.max(np.abs(y), axis=2)
    band = np.max(dy, axis=2)

    def shared_x(a):
        with np.errstate(divide="ignore"):
            return np.where(a > 0, np.floor(np.log2(np.where(a > 0, a, 1.0))) - 2, 0.0)
    x_lo, x_hi = shared_x(np.maximum(amax - band, 0.0)), shared_x(amax + band)
    x_lo = np.where(amax - band <= 0, np.minimum(x_lo, 0), x_lo)
    ok = (X >= np.minimum(x_lo, x_hi)) & (X <= np.maximum(x_lo, x_hi))
    assert np.all(ok), f"{where}: {np.sum(~ok)} block exponents outside the band"
    s = np.ldexp(1.0, X)[:, :, None]
    codes = O.mxfp4_unpack(packed).reshape(len(js), d_nope // 32, 32)
    exact = check_codes(codes.reshape(-1), (y / s).reshape(-1), O.e2m1_encode, O.e2m1_decode,
                        (dy / s).reshape(-1), where=where + " e2m1")
    return exact
