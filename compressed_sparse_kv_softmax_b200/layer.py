"""Per-layer drivers over device buffers (marshalling around the C ABI).

A CSA layer step is: csa_compress of the newly arrived tokens, indexer_topk,
hybrid attention over the selected entries plus the window.  An HCA layer step
is: hca_compress, hybrid attention over every visible entry plus the window.
A window-only layer (the first two layers of the model) is hybrid attention
with no compressed cache.  Buffers are torch tensors on one CUDA device; the
caches are dicts of planes as described in the package docstring.
"""
from __future__ import annotations

import torch

from . import attn_workspace_size, cache_struct, indexer_workspace_size, prepare, workspace


def _dims(c):
    return int(c["d_nope"]) + int(c["d_rope"])


_CACHES = ("ring_k", "ring_v", "ring_ik", "comp_k", "comp_v", "comp_ik")


def _descriptors(L):
    """C descriptors of the layer's caches, built once (the planes do not move)."""
    return {key: cache_struct(L.get(key)) for key in _CACHES}


def _addr(t):
    return None if t is None else t.data_ptr()


class _Prepared:
    """A layer's calls with their arguments marshalled once per combination
    of the buffers they take (and the current stream): a decode step repeats
    them every token on the same buffers, so a step costs the host little
    more than the launches.  The key holds every address a call reads, so a
    layer whose input or output tensors are swapped for others gets new
    calls."""

    def __init__(self):
        self._calls = {}

    def __call__(self, key, name, *args):
        key = (name, torch.cuda.current_stream().cuda_stream) + key
        call = self._calls.get(key)
        if call is None:
            call = self._calls[key] = prepare(name, *args)
        call()


class CSALayer:
    """One CSA layer: raw rings, compressed caches, the indexer and attention.

    L: dict with ring_k, ring_v (or None), ring_ik, comp_k, comp_v (or None),
    comp_ik, q, q_ik, q_ik_scale, head_w, gate_w, gate_b, pool, stride, q_pos,
    ctx_len and the shape fields of `wl` (B, Tq, Hq, H_I, d_I, k, window,
    prefill, sm_scale)."""

    def __init__(self, L, k=None, max_entries=None):
        wl = L["wl"]
        self.L, self.wl = L, wl
        self.B, self.Tq, self.Hq = wl.B, wl.Tq, wl.Hq
        self.k = int(k if k is not None else wl.k)
        self.max_entries = int(max_entries if max_entries is not None else L["comp_ik"]["cap"])
        dev = L["q"].device
        self.Dv = _dims(L["comp_v"] or L["comp_k"])
        self.idx = torch.empty(self.B, self.Tq, self.k, dtype=torch.int32, device=dev)
        self.score = torch.empty(self.B, self.Tq, self.k, dtype=torch.float32, device=dev)
        self.out = torch.empty(self.B, self.Tq, self.Hq, self.Dv, dtype=torch.float32, device=dev)
        self.lse = torch.empty(self.B, self.Tq, self.Hq, dtype=torch.float32, device=dev)
        self.ws_idx = workspace(indexer_workspace_size(self.B, self.Tq, self.max_entries, self.k),
                                dev)
        self.ws_attn = workspace(attn_workspace_size(self.B, self.Tq, self.Hq, self.Dv, self.k,
                                                     wl.window), dev)
        self.cs = _descriptors(L)
        self._call = _Prepared()

    def compress(self, t_begin, t_end, max_new):
        L, c = self.L, self.cs
        key = (_addr(t_begin), _addr(t_end), int(max_new), _addr(L["gate_w"]),
               _addr(L["gate_b"]), _addr(L.get("gate_w_ik")), _addr(L.get("gate_b_ik")))
        if L.get("gate_mode", "scalar") == "channel":
            self._call(key, "csa_compress_channel_gate", self.B, t_begin, t_end, max_new,
                       c["ring_k"], c["ring_v"], c["ring_ik"], L["gate_w"], L["gate_b"],
                       L.get("gate_w_ik"), L.get("gate_b_ik"), L["pool"], L["stride"],
                       c["comp_k"], c["comp_v"], c["comp_ik"])
            return
        self._call(key, "csa_compress", self.B, t_begin, t_end, max_new, c["ring_k"],
                   c["ring_v"], c["ring_ik"], L["gate_w"], L["gate_b"], L["pool"], L["stride"],
                   c["comp_k"], c["comp_v"], c["comp_ik"])

    def select(self, q_pos=None, phase="both"):
        """indexer_topk; q_pos [B][Tq] (device) overrides the layer's positions.
        phase "score" / "pick" runs only indexer_score / indexer_select."""
        L, wl = self.L, self.wl
        q_pos = L["q_pos"] if q_pos is None else q_pos
        name = {"both": "indexer_topk", "score": "indexer_score", "pick": "indexer_select"}[phase]
        key = (_addr(q_pos), _addr(L["q_ik"]), _addr(L["q_ik_scale"]), _addr(L["head_w"]),
               _addr(self.idx), _addr(self.score), _addr(self.ws_idx))
        self._call(key, name, self.B, self.Tq, q_pos, L["q_ik"], L["q_ik_scale"], L["head_w"],
                   wl.H_I, wl.d_I, self.cs["comp_ik"], L["stride"], self.k, self.max_entries,
                   self.idx, self.score, self.ws_idx)
        return self.idx

    def attend(self, sel=None, pos=None):
        """Hybrid attention over `sel` (default: the last selection); pos
        overrides q_pos (prefill) or ctx_len (decode)."""
        L, wl, c = self.L, self.wl, self.cs
        sel = self.idx if sel is None else sel
        pos = (L["q_pos"] if wl.prefill else L["ctx_len"]) if pos is None else pos
        key = (_addr(sel), _addr(pos), _addr(L["q"]), _addr(self.out), _addr(self.lse),
               _addr(self.ws_attn))
        if wl.prefill:
            self._call(key, "hybrid_attn_prefill", self.B, self.Tq, pos, L["q"], self.Hq,
                       wl.sm_scale, c["comp_k"], c["comp_v"], L["stride"], sel, self.k, self.k,
                       c["ring_k"], c["ring_v"], wl.window, self.out, self.lse, self.ws_attn)
        else:
            self._call(key, "hybrid_attn_decode", self.B, pos, L["q"], self.Hq, wl.sm_scale,
                       c["comp_k"], c["comp_v"], L["stride"], sel, self.k, self.k,
                       c["ring_k"], c["ring_v"], wl.window, self.out, self.lse, self.ws_attn)
        return self.out, self.lse

    def step(self):
        self.select()
        return self.attend()


class HCALayer:
    """One HCA layer: raw ring, compressed cache, dense attention plus window.
    With dense=False (no compressed cache) it is a window-only layer."""

    def __init__(self, L, max_entries=None, dense=True):
        wl = L["wl"]
        self.L, self.wl, self.dense = L, wl, dense
        self.B, self.Tq, self.Hq = wl.B, wl.Tq, wl.Hq
        self.max_entries = int(max_entries if max_entries is not None else L["comp_k"]["cap"])
        dev = L["q"].device
        self.Dv = _dims(L["comp_v"] or L["comp_k"])
        self.out = torch.empty(self.B, self.Tq, self.Hq, self.Dv, dtype=torch.float32, device=dev)
        self.lse = torch.empty(self.B, self.Tq, self.Hq, dtype=torch.float32, device=dev)
        self.ws_attn = workspace(attn_workspace_size(self.B, self.Tq, self.Hq, self.Dv,
                                                     self.max_entries if dense else 0,
                                                     wl.window), dev)
        self.cs = _descriptors(L)
        self._call = _Prepared()

    def compress(self, t_begin, t_end, max_new):
        L, c = self.L, self.cs
        name = ("hca_compress_channel_gate" if L.get("gate_mode", "scalar") == "channel"
                else "hca_compress")
        key = (_addr(t_begin), _addr(t_end), int(max_new), _addr(L["gate_w"]),
               _addr(L["gate_b"]))
        self._call(key, name, self.B, t_begin, t_end, max_new, c["ring_k"], c["ring_v"],
                   L["gate_w"], L["gate_b"], L["pool"], L["stride"], c["comp_k"], c["comp_v"])

    def attend(self, pos=None):
        """Dense hybrid attention; pos overrides q_pos (prefill) or ctx_len (decode)."""
        L, wl, c = self.L, self.wl, self.cs
        ck = c["comp_k"] if self.dense else None
        cv = c["comp_v"] if self.dense else None
        me = self.max_entries if self.dense else 0
        pos = (L["q_pos"] if wl.prefill else L["ctx_len"]) if pos is None else pos
        key = (_addr(pos), _addr(L["q"]), _addr(self.out), _addr(self.lse), _addr(self.ws_attn))
        if wl.prefill:
            self._call(key, "hybrid_attn_prefill", self.B, self.Tq, pos, L["q"], self.Hq,
                       wl.sm_scale, ck, cv, L["stride"], None, 0, me, c["ring_k"], c["ring_v"],
                       wl.window, self.out, self.lse, self.ws_attn)
        else:
            self._call(key, "hybrid_attn_decode", self.B, pos, L["q"], self.Hq, wl.sm_scale,
                       ck, cv, L["stride"], None, 0, me, c["ring_k"], c["ring_v"], wl.window,
                       self.out, self.lse, self.ws_attn)
        return self.out, self.lse

    step = attend
