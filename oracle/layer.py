"""Per-stage oracle drivers over one layer's inputs (test infrastructure).

They read the seeded input planes (torch tensors from the `workloads`
generator), dequantise them with the oracle's own codecs and apply the
definitions in `method.py` query by query.
"""
from __future__ import annotations

import numpy as np

from .method import (attend, dequant_slots, indexer_scores, n_entries, pool_entries,
                     pool_entries_per_channel,
                     requantize, requantize_mxfp4, ring_slots, scale_block, topk,
                     window_positions)


def _np(t):
    if t is None:
        return None
    import torch
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def as_numpy_cache(c):
    """A cache as numpy planes [B][cap][...]; a paged cache (block table) is
    read back into that form: slot s of sequence b is pool row
    table[b][s // block_size] * block_size + s % block_size (slots of a
    logical block without a pool block read as NaN)."""
    if c is None:
        return None
    out = {k: c[k] for k in ("fmt", "d_nope", "d_rope", "ring", "cap")}
    for k in ("data", "scale", "rope"):
        out[k] = _np(c.get(k))
    if c.get("block_table") is not None:
        bt = _np(c["block_table"]).astype(np.int64)
        bs = int(c["block_size"])
        B, nb = bt.shape
        rows = (np.maximum(bt, 0)[:, :, None] * bs + np.arange(bs)[None, None, :]).reshape(B, -1)
        hole = np.repeat(bt < 0, bs, axis=1)
        for k in ("data", "scale", "rope"):
            if out[k] is None:
                continue
            v = out[k][0][rows]
            if k == "scale" and np.issubdtype(v.dtype, np.floating):
                v = np.where(hole[:, :, None], np.nan, v)
            out[k] = v
    return out


def _q_ik(L, b, t):
    q = _np(L["q_ik"])[b, t].astype(np.float64)
    if L["q_ik_scale"] is None:
        return q
    if L["comp_ik"]["fmt"] == "mxfp4":
        from .formats import mxfp4_decode
        d_I = L["comp_ik"]["d_nope"]
        return mxfp4_decode(_np(L["q_ik"])[b, t], _np(L["q_ik_scale"])[b, t][:, : d_I // 32])
    from .formats import e4m3_decode
    sc = _np(L["q_ik_scale"])[b, t].astype(np.float64)       # [H_I][cols]
    d_I = q.shape[-1]
    # the indexer queries share the indexer keys' scale layout
    block = scale_block(L["comp_ik"]["fmt"], d_I)
    nb = (d_I + block - 1) // block
    return e4m3_decode(_np(L["q_ik"])[b, t]) * np.repeat(sc[:, :nb], block, axis=1)[:, :d_I]


def _q(L, b, t):
    q = _np(L["q"])
    if q.dtype == np.uint16:
        from .formats import bf16_decode
        return bf16_decode(q[b, t])
    return q[b, t].astype(np.float64)


def layer_compress(L, t_begin, t_end):
    """Entries written when tokens [t_begin, t_end) of each sequence arrive:
    j in [n(t_begin), n(t_end)).  Returns per sequence a dict with the pooled
    float64 values ("k", "v", "ik") and, for the E4M3 layout, the stored
    form ("k_codes", "k_scales", "k_rope", "ik_codes", "ik_scales")."""
    pool, stride = L["pool"], L["stride"]
    ring_k = as_numpy_cache(L["ring_k"])
    ring_v = as_numpy_cache(L.get("ring_v"))
    ring_ik = as_numpy_cache(L.get("ring_ik"))
    gw = _np(L["gate_w"]).astype(np.float64)
    gb = _np(L["gate_b"]).astype(np.float64)
    # the per-channel gate variant: gate_b [pool][D] and the indexer keys' own
    # gate_w_ik [d_I], gate_b_ik [pool][d_I]
    per_channel = L.get("gate_mode", "scalar") == "channel"
    if per_channel and ring_ik is not None:
        gw_ik = _np(L["gate_w_ik"]).astype(np.float64)
        gb_ik = _np(L["gate_b_ik"]).astype(np.float64)
    res = []
    for b in range(len(t_begin)):
        js = list(range(n_entries(int(t_begin[b]), stride), n_entries(int(t_end[b]), stride)))

        def reader(cache):
            return lambda p: dequant_slots(cache, b, [ring_slots([p], cache["cap"])[0]])[0]

        vals = [reader(ring_k)]
        names = ["k"]
        if ring_v is not None:
            vals.append(reader(ring_v)); names.append("v")
        if ring_ik is not None and not per_channel:
            vals.append(reader(ring_ik)); names.append("ik")
        # sum_r a_r |x_{p_r}|: the magnitude scale of each pooled sum, which
        # bounds its floating-point evaluation error
        absvals = [(lambda f: (lambda p: np.abs(f(p))))(v) for v in vals]
        if per_channel:
            # one gate per channel; the indexer keys have gates of their own
            pooled, w = pool_entries_per_channel(reader(ring_k), vals, gw, gb, pool, stride, js)
            mags, _ = pool_entries_per_channel(reader(ring_k), absvals, gw, gb, pool, stride, js)
            if ring_ik is not None:
                ri = reader(ring_ik)
                pi, _ = pool_entries_per_channel(ri, [ri], gw_ik, gb_ik, pool, stride, js)
                mi, _ = pool_entries_per_channel(ri, [lambda p: np.abs(ri(p))], gw_ik, gb_ik,
                                                 pool, stride, js)
                names.append("ik")
                pooled, mags = list(pooled) + pi, list(mags) + mi
        else:
            pooled, w = pool_entries(reader(ring_k), vals, gw, gb, pool, stride, js)
            mags, _ = pool_entries(reader(ring_k), absvals, gw, gb, pool, stride, js)
        r = {"j": np.asarray(js, dtype=np.int64), "weights": w}
        for name, arr in zip(names, pooled):
            r[name] = arr
        for name, arr in zip(names, mags):
            r[name + "_mag"] = arr
        if ring_k["fmt"] != "f32":
            for name, cache in (("k", ring_k), ("ik", ring_ik)):
                if name in r and cache is not None and len(js):
                    d_nope = cache["d_nope"]
                    if cache["fmt"] == "mxfp4":
                        # FP4 indexer keys: packed E2M1 codes, E8M0 exponents
                        codes, exps = requantize_mxfp4(r[name])
                        r[name + "_codes"], r[name + "_scales"] = codes, exps
                        continue
                    codes, scales, rope = requantize(r[name], d_nope,
                                                     scale_block(cache["fmt"], d_nope))
                    r[name + "_codes"], r[name + "_scales"], r[name + "_rope"] = codes, scales, rope
        res.append(r)
    return res


def layer_indexer_topk(L, k, rows=None):
    """Scores and top-k of every (or the listed) query row (b, t).
    Returns {(b, t): (idx [k], scores over visible entries [n_vis])}."""
    wl = L["wl"]
    comp_ik = as_numpy_cache(L["comp_ik"])
    head_w = _np(L["head_w"]).astype(np.float64)
    q_pos = _np(L["q_pos"])
    if rows is None:
        rows = [(b, t) for b in range(wl.B) for t in range(wl.Tq)]
    out = {}
    for b, t in rows:
        n_vis = n_entries(int(q_pos[b, t]) + 1, L["stride"])
        kik = dequant_slots(comp_ik, b, np.arange(n_vis))
        s = indexer_scores(_q_ik(L, b, t), head_w[b, t], kik)
        out[(b, t)] = (topk(s, n_vis, k), s)
    return out


def _window(L, b, pos):
    wl = L["wl"]
    ring_k = as_numpy_cache(L["ring_k"])
    ring_v = as_numpy_cache(L.get("ring_v")) or ring_k
    wpos = window_positions(pos, wl.window)
    sk = ring_slots(wpos, ring_k["cap"])
    return dequant_slots(ring_k, b, sk), dequant_slots(ring_v, b, sk)


def layer_attention(L, sel=None, rows=None):
    """Hybrid attention of every (or the listed) query row.

    sel: None for dense attention over every visible compressed entry (HCA),
         else int array [B][Tq][k] of selected CSA entries (-1 = unused).
    Returns {(b, t): (o [Hq][Dv], lse [Hq])}."""
    wl = L["wl"]
    comp_k = as_numpy_cache(L["comp_k"])
    comp_v = as_numpy_cache(L.get("comp_v")) or comp_k
    q_pos = _np(L["q_pos"])
    if rows is None:
        rows = [(b, t) for b in range(wl.B) for t in range(wl.Tq)]
    out = {}
    for b, t in rows:
        pos = int(q_pos[b, t])
        if sel is None:
            js = np.arange(n_entries(pos + 1, L["stride"]))
        else:
            js = np.asarray(sel[b, t])
            js = js[js >= 0]
        ck = dequant_slots(comp_k, b, js)
        cv = dequant_slots(comp_v, b, js)
        wk, wv = _window(L, b, pos)
        o, lse = attend(_q(L, b, t), np.concatenate([ck, wk]), np.concatenate([cv, wv]),
                        wl.sm_scale)
        out[(b, t)] = (o, lse)
    return out


def layer_attention_dense_keys(L, b, t):
    """Query (b, t) with its full key and value lists as float64 arrays (used
    by identity checks)."""
    wl = L["wl"]
    pos = int(_np(L["q_pos"])[b, t])
    comp_k = as_numpy_cache(L["comp_k"])
    comp_v = as_numpy_cache(L.get("comp_v")) or comp_k
    js = np.arange(n_entries(pos + 1, L["stride"]))
    wk, wv = _window(L, b, pos)
    return (_q(L, b, t), dequant_slots(comp_k, b, js), dequant_slots(comp_v, b, js), wk, wv)
