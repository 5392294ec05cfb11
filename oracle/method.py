"""The method's arithmetic, written out plainly in float64 (test infrastructure).

Sources (web pages on DeepSeek-V4's hybrid attention):
  [webconsulting] «DeepSeek V4-Pro: Architektur, KV-Cache-Kompression und
      Hyper-Connections im Detail», sections "Das Wichtigste" and
      "Kompression und Selektion".
  [chaosnode] «DeepSeek-V4: 1 Million Token Context endlich nutzbar»,
      section "Hybrid Attention: CSA und HCA".
  [golem] «Chinas KI-Unabhaengigkeit?: Bei Deepseek V4 haben kleine
      Aenderungen grosse Wirkung», section "Komprimierte Erinnerung fuer
      laengere Kontexte".

Readings where the pages leave a step open are marked READING; each is also
listed in the design notes with its justification.
"""
from __future__ import annotations

import numpy as np

from .formats import (E4M3_MAX, bf16_decode, bf16_encode, e4m3_decode, e4m3_encode,
                      mxfp4_decode, mxfp4_quantize)


# ---------------------------------------------------------------- pooling ---

def n_entries(t: int, stride: int) -> int:
    """Number of compressed entries present after t tokens.

    READING: entry j pools the window that ends with group j, i.e. positions
    stride*(j+1)-pool .. stride*(j+1)-1, so it exists once position
    stride*(j+1)-1 < t: floor(t / stride) entries.  For 4x CSA at 1,048,576
    tokens that is 262,144 entries; for 128x HCA at 131,072 tokens, 1,024.
    """
    return t // stride


def pool_positions(j: int, pool: int, stride: int) -> np.ndarray:
    """Token positions covered by entry j, slot r = 0..pool-1.

    CSA groups 4 tokens and lets information cross group boundaries
    [webconsulting "Kompression und Selektion"]: READING: a window of `pool`
    tokens ending with group j (for CSA: the previous group and group j);
    positions < 0 are absent.  HCA pools 128 tokens, window = stride = 128.
    """
    return stride * (j + 1) - pool + np.arange(pool)


def pool_entries(gate_src, values, gate_w, gate_b, pool: int, stride: int, j_list):
    """Softmax-gated pooling with a learned positional bias [chaosnode].

    gate_src(p) -> float64 [D]   the key vector of token p (gate input)
    values: list of callables v(p) -> float64 [d]; each is pooled with the
            same weights (K, V of the tiny layout, and the raw indexer key)
    For entry j: logits g_r = gate_w . k_{p_r} + gate_b[r] over the slots r
    whose position p_r >= 0, a = softmax(g), c = sum_r a_r v(p_r).
    READING: one scalar gate per token read from its key; the bias is per
    slot of the window.
    Returns (list of pooled arrays [len(j_list)][d] per value, weights [n][pool]).
    """
    outs = [[] for _ in values]
    weights = []
    for j in j_list:
        pos = pool_positions(j, pool, stride)
        valid = pos >= 0
        g = np.full(pool, -np.inf)
        for r in range(pool):
            if valid[r]:
                g[r] = float(np.dot(gate_w, gate_src(int(pos[r])))) + gate_b[r]
        gmax = np.max(g[valid])
        e = np.where(valid, np.exp(g - gmax), 0.0)
        a = e / e.sum()
        weights.append(a)
        for i, v in enumerate(values):
            acc = None
            for r in range(pool):
                if valid[r]:
                    term = a[r] * v(int(pos[r]))
                    acc = term if acc is None else acc + term
            outs[i].append(acc)
    return [np.asarray(o) for o in outs], np.asarray(weights)


def pool_entries_per_channel(gate_src, values, gate_w, gate_b, pool: int, stride: int,
                             j_list):
    """Softmax-gated pooling with one gate per channel (the per-channel
    variant of the gated pooling with learned positional bias [chaosnode]).

    gate_src(p) -> float64 [D]   the key vector of token p (gate input)
    values: callables v(p) -> float64 [D], pooled channel by channel with the
            key's weights (K and V of the separate-V layout share D)
    gate_w: [D]; gate_b: [pool][D].  For entry j and channel c:
        g_{r,c} = gate_w[c] * k_{p_r}[c] + gate_b[r][c]   over present slots r,
        a_{.,c} = softmax_r(g_{.,c}),   out[c] = sum_r a_{r,c} v(p_r)[c].
    READING: each channel's gate reads that channel of the key alone, with a
    per-slot, per-channel bias; the pages name the softmax gate and the
    positional bias but not their shapes.
    Returns (list of pooled arrays [len(j_list)][D] per value, weights
    [n][pool][D])."""
    gate_w = np.asarray(gate_w, dtype=np.float64)
    gate_b = np.asarray(gate_b, dtype=np.float64)
    outs = [[] for _ in values]
    weights = []
    for j in j_list:
        pos = pool_positions(j, pool, stride)
        valid = pos >= 0
        D = gate_w.shape[0]
        g = np.full((pool, D), -np.inf)
        for r in range(pool):
            if valid[r]:
                g[r] = gate_w * gate_src(int(pos[r])) + gate_b[r]
        gmax = np.max(g[valid], axis=0)                 # per channel
        e = np.where(valid[:, None], np.exp(g - gmax[None, :]), 0.0)
        a = e / e.sum(axis=0, keepdims=True)
        weights.append(a)
        for i, v in enumerate(values):
            acc = np.zeros(D)
            for r in range(pool):
                if valid[r]:
                    acc = acc + a[r] * v(int(pos[r]))
            outs[i].append(acc)
    return [np.asarray(o) for o in outs], np.asarray(weights)


def scale_block(fmt: str, d_nope: int) -> int:
    """Dims per fp32 scale: 64 for the KV-cache layout ("e4m3"), the whole
    vector for the indexer layout ("e4m3vec": one scale per key or query
    head)."""
    return d_nope if fmt == "e4m3vec" else 64


def requantize(c: np.ndarray, d_nope: int, block: int = 64):
    """Store pooled entries in the cache format: FP8 E4M3 for the first d_nope
    dims with one fp32 scale per `block`-element block, BF16 for the rest
    [chaosnode; golem: the last 64 values carry RoPE and stay BF16].  The KV
    cache uses 64-element blocks; the indexer keys one block per vector.

    READING: scale = amax/448 over the block (1 when the block is all zero),
    code = E4M3(c / scale) rounded to nearest-even and saturated.
    Returns codes uint8 [n][d_nope], scales float64 [n][nb], rope bits uint16.
    """
    c = np.asarray(c, dtype=np.float64)
    n = c.shape[0]
    nb = (d_nope + block - 1) // block
    codes = np.empty((n, d_nope), dtype=np.uint8)
    scales = np.empty((n, nb), dtype=np.float64)
    for b in range(nb):
        blk = c[:, block * b: min(block * (b + 1), d_nope)]
        amax = np.max(np.abs(blk), axis=1)
        s = np.where(amax > 0, amax / E4M3_MAX, 1.0)
        scales[:, b] = s
        codes[:, block * b: block * b + blk.shape[1]] = e4m3_encode(blk / s[:, None])
    rope = bf16_encode(c[:, d_nope:])
    return codes, scales, rope


def requantize_mxfp4(c: np.ndarray):
    """Store pooled indexer keys in the MXFP4 layout (the FP4 lightning
    indexer): packed E2M1 codes and one E8M0 exponent per 32 dims, the OCP MX
    conversion (see formats.mxfp4_quantize)."""
    return mxfp4_quantize(np.asarray(c, dtype=np.float64))


# ---------------------------------------------------------------- indexer ---

def indexer_scores(q_ik: np.ndarray, head_w: np.ndarray, k_ik: np.ndarray) -> np.ndarray:
    """Lightning-indexer relevance of every CSA entry for one query
    [webconsulting "Kompression und Selektion"; chaosnode; golem: learned].

    READING (the pages give no formula): the multi-head weighted-ReLU score of
    the predecessor's lightning indexer,
        s_j = sum_h head_w[h] * max(0, q_ik[h] . k_ik[j]).
    q_ik [H_I][d_I], head_w [H_I], k_ik [n][d_I] -> s [n].
    """
    dots = k_ik @ q_ik.T                     # [n][H_I]
    return np.maximum(dots, 0.0) @ head_w


def topk(scores: np.ndarray, n_visible: int, k: int) -> np.ndarray:
    """Indices of the k highest-scoring visible entries (top 1,024 for V4-Pro,
    512 for V4-Flash [golem]).  READING: ties go to the lower index; when
    fewer than k entries are visible all are taken; unused slots are -1.
    Returned in selection order (score descending, index ascending)."""
    n = int(n_visible)
    idx = np.arange(n)
    order = np.lexsort((idx, -scores[:n]))   # primary: -score, secondary: index
    take = order[: min(k, n)]
    out = np.full(k, -1, dtype=np.int64)
    out[: take.size] = take
    return out


# -------------------------------------------------------------- attention ---

def window_positions(pos: int, window: int) -> np.ndarray:
    """Raw tokens of the sliding window for a query at position pos: the last
    `window` positions, the query's own token included [webconsulting "Das
    Wichtigste"; golem].  READING: inclusive of pos."""
    return np.arange(max(0, pos - window + 1), pos + 1)


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, sm_scale: float):
    """One softmax over all keys for every head (MQA: all heads share K, V).
    q [Hq][D], K [m][D], V [m][Dv] -> o [Hq][Dv], lse [Hq] (natural log)."""
    logits = sm_scale * (q @ K.T)            # [Hq][m]
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    ssum = e.sum(axis=1, keepdims=True)
    o = (e / ssum) @ V
    lse = (mx + np.log(ssum))[:, 0]
    return o, lse


def hybrid_attention(q, comp_k, comp_v, win_k, win_v, sm_scale):
    """Attention of one query over the union of its compressed entries (the
    selected CSA entries, or every visible HCA entry [chaosnode: dense over the
    compressed blocks]) and its raw sliding window [golem: both mechanisms
    additionally use the window].  READING: one softmax over the
    concatenation, which is what a log-sum-exp merge of the two partial
    softmaxes computes."""
    K = np.concatenate([comp_k, win_k], axis=0)
    V = np.concatenate([comp_v, win_v], axis=0)
    return attend(q, K, V, sm_scale)


# ------------------------------------------------------------ cache access ---

def ring_slots(positions, cap: int) -> np.ndarray:
    """Raw-token ring: position p lives in slot p mod cap."""
    return np.asarray(positions, dtype=np.int64) % cap


def dequant_slots(cache: dict, b: int, slots) -> np.ndarray:
    """Float64 values of the given slots of sequence b.

    cache: numpy planes {"fmt", "d_nope", "d_rope", "data", "scale", "rope"}.
    E4M3 layouts: x[d] = E4M3(code[d]) * scale[d // block] for d < d_nope
    (block 64, or the whole vector for "e4m3vec"), and x[d_nope + r] =
    BF16(rope[r]).  f32 layout: the stored values."""
    slots = np.asarray(slots, dtype=np.int64)
    if cache["fmt"] == "f32":
        return cache["data"][b, slots].astype(np.float64)
    if cache["fmt"] == "mxfp4":
        # packed E2M1 codes and one E8M0 exponent per 32 dims (no RoPE part)
        d_nope = cache["d_nope"]
        return mxfp4_decode(cache["data"][b, slots], cache["scale"][b, slots][:, : d_nope // 32])
    d_nope, d_rope = cache["d_nope"], cache["d_rope"]
    block = scale_block(cache["fmt"], d_nope)
    nb = (d_nope + block - 1) // block
    codes = cache["data"][b, slots]
    sc = cache["scale"][b, slots][:, :nb].astype(np.float64)
    nope = e4m3_decode(codes) * np.repeat(sc, block, axis=1)[:, :d_nope]
    if d_rope == 0:
        return nope
    rope = bf16_decode(cache["rope"][b, slots])
    return np.concatenate([nope, rope], axis=1)
