"""Seeded synthetic layer inputs.

Recipe (all draws from one `torch.Generator` seeded per layer):
  * FP8 planes (raw tokens, compressed entries, indexer keys, indexer queries):
    x ~ N(0,1) per element, per-64-element block scale s ~ U[0.5, 2], stored
    code = E4M3(clamp(x / s, +-448)), stored scale = s.  The dequantised input
    is therefore E4M3(code) * s.
  * BF16 RoPE dims: N(0,1) rounded to BF16.   fp32 planes: N(0,1).
  * q: N(0,1) as BF16 (fp32 and pre-scaled by 1/sqrt(D) for the tiny workload).
  * indexer head weights: N(0,1)/sqrt(H_I).   gate w, b: N(0, 0.1^2).
  * needles: at a needle position p the CSA entry p // stride gets, as its
    indexer key, the query's indexer head with the largest weight scaled by 4,
    and as its KV entry the first head's query (E4M3-encoded); the HCA entry
    p // 128 gets the same KV needle.
  * ring slots that hold no live position carry NaN scales / NaN values, so a
    kernel that reads one produces NaN.

Nothing here pools, scores, selects or attends: this module only produces
inputs.  Tensors are created on `device` from a generator on that device.
"""
from __future__ import annotations

import math

import torch

from .configs import Workload

_E4M3_MAX = 448.0


def e4m3_from_float(x: torch.Tensor) -> torch.Tensor:
    """Encode fp32 values as E4M3 codes (uint8) with torch's cast, clamped first
    because torch maps out-of-range values to NaN."""
    return x.clamp(-_E4M3_MAX, _E4M3_MAX).to(torch.float8_e4m3fn).view(torch.uint8)


def _n_slots(t: int, stride: int) -> int:
    # number of compressed entries a cache must hold for t tokens
    return t // stride


class _Rng:
    def __init__(self, seed: int, device):
        self.device = torch.device(device)
        self.g = torch.Generator(device=self.device)
        self.g.manual_seed(seed)

    def normal(self, *shape, std=1.0):
        return torch.randn(*shape, generator=self.g, device=self.device, dtype=torch.float32) * std

    def uniform(self, lo, hi, *shape):
        return lo + (hi - lo) * torch.rand(*shape, generator=self.g, device=self.device,
                                           dtype=torch.float32)

    def integers(self, lo, hi, *shape):
        return torch.randint(lo, hi, shape, generator=self.g, device=self.device)


def _scale_cols(d_nope: int, pad: int, block: int = 64) -> int:
    nb = (d_nope + block - 1) // block
    return ((nb + pad - 1) // pad) * pad


def _fp8_planes(rng: _Rng, lead, d_nope: int, scale_pad: int, block: int = 64):
    """codes uint8 [*lead, d_nope], scales f32 [*lead, cols] (pad columns NaN);
    one scale per `block` dims."""
    nb = (d_nope + block - 1) // block
    x = rng.normal(*lead, d_nope)
    s = rng.uniform(0.5, 2.0, *lead, nb)
    s_el = s.repeat_interleave(block, dim=-1)[..., :d_nope]
    codes = e4m3_from_float(x / s_el)
    cols = _scale_cols(d_nope, scale_pad, block)
    scale = torch.full((*lead, cols), float("nan"), device=rng.device, dtype=torch.float32)
    scale[..., :nb] = s
    return codes, scale


# E2M1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes 0..7) and the midpoints
# between them: a draw is stored as the code of the interval it falls in
_E2M1_EDGES = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def _mxfp4_planes(rng: _Rng, lead, d: int):
    """FP4 (MXFP4) vectors: per element a draw y ~ N(0, 4) stored as the E2M1
    code of its magnitude interval (magnitudes above 5 read 6) with its sign,
    two codes per byte (even element in the low nibble); per 32 elements an
    E8M0 exponent byte 126 + U{-1, 0, 1} (scale 2^-2 .. 2^0).  The values are
    those of N(0,1)-like activations in the OCP MX layout.
    Returns (packed uint8 [*lead, d/2], exponents uint8 [*lead, d/32])."""
    y = rng.normal(*lead, d, std=2.0)
    mag = torch.bucketize(y.abs(), _E2M1_EDGES.to(y.device))
    codes = (mag | ((y < 0).to(mag.dtype) << 3)).to(torch.uint8)
    packed = codes[..., 0::2] | (codes[..., 1::2] << 4)
    exps = (126 + rng.integers(-1, 2, *lead, d // 32)).to(torch.uint8)
    return packed, exps


def _cache(rng: _Rng, wl: Workload, B: int, n: int, *, d_nope: int, d_rope: int,
           fmt: str, scale_pad: int, ring: bool):
    """A cache of n slots per sequence in the workload's storage format."""
    c = {"fmt": fmt, "d_nope": d_nope, "d_rope": d_rope, "ring": ring, "cap": n}
    if fmt == "mxfp4":
        c["data"], c["scale"] = _mxfp4_planes(rng, (B, n), d_nope)
        return c
    if fmt == "f32":
        c["data"] = rng.normal(B, n, d_nope + d_rope)
    else:
        block = d_nope if fmt == "e4m3vec" else 64
        c["data"], c["scale"] = _fp8_planes(rng, (B, n), d_nope, scale_pad, block)
        if d_rope:
            c["rope"] = rng.normal(B, n, d_rope).to(torch.bfloat16)
    return c


def _poison_ring(c: dict, t_end: int):
    """Mark slots that hold no live position (pos < 0) with NaN."""
    cap = c["cap"]
    live = min(cap, t_end)
    if live == cap:
        return
    dead = torch.arange(live, cap)  # slots p % cap for p in [t_end-cap, 0) map here when t_end < cap
    if c["fmt"] == "f32":
        c["data"][:, dead] = float("nan")
    elif c["fmt"] == "mxfp4":
        c["scale"][:, dead] = 255          # the E8M0 NaN
    else:
        c["scale"][:, dead] = float("nan")
        if "rope" in c:
            c["rope"][:, dead] = float("nan")


def _needle_positions(rng: _Rng, wl: Workload, t: int):
    if wl.needles == 0 or wl.prefill:
        return torch.zeros(wl.B, 0, dtype=torch.int64)
    if wl.needle_mode == "loguniform":
        u = rng.uniform(0.0, math.log(t), wl.B, wl.needles)
        d = torch.floor(torch.exp(u)).to(torch.int64).clamp_(0, t - 1)
        return (t - 1 - d).cpu()
    return rng.integers(0, t, wl.B, wl.needles).cpu()


def _queries(rng: _Rng, wl: Workload):
    B, Tq = wl.B, wl.Tq
    if wl.fmt == "f32":
        q = rng.normal(B, Tq, wl.Hq, wl.D)
        if wl.q_prescale:
            q = q * (1.0 / math.sqrt(wl.D))
        return q
    return rng.normal(B, Tq, wl.Hq, wl.D).to(torch.bfloat16)


def _positions(wl: Workload, device):
    """q_pos [B][Tq] int64 and ctx_len [B] int64 (tokens incl. the last query)."""
    if wl.prefill:
        pos = torch.arange(wl.T, wl.T + wl.Tq, device=device, dtype=torch.int64)
        pos = pos.unsqueeze(0).expand(wl.B, wl.Tq).contiguous()
    else:
        pos = torch.full((wl.B, 1), wl.T - 1, device=device, dtype=torch.int64)
    return pos, pos[:, -1] + 1


def _plant_kv_needle(cache: dict, b: int, j: int, q_head0: torch.Tensor, rng: _Rng):
    d_nope = cache["d_nope"]
    if cache["fmt"] == "f32":
        cache["data"][b, j, :d_nope] = q_head0[:d_nope].float()
        return
    v = q_head0[:d_nope].float() * 0.5
    s = cache["scale"][b, j, : (d_nope + 63) // 64]
    cache["data"][b, j] = e4m3_from_float(v / s.repeat_interleave(64)[:d_nope])


def _channel_gates(rng: _Rng, L: dict, D: int, pool: int, d_I):
    """Parameters of the per-channel gate variant: gate_w [D] and gate_b
    [pool][D] ~ N(0, 1) (wide enough that the weights are far from uniform),
    and the indexer keys' own gate_w_ik [d_I], gate_b_ik [pool][d_I]."""
    L["gate_mode"] = "channel"
    L["gate_w"] = rng.normal(D)
    L["gate_b"] = rng.normal(pool, D)
    if d_I is not None:
        L["gate_w_ik"] = rng.normal(d_I)
        L["gate_b_ik"] = rng.normal(pool, d_I)


def make_csa_layer(wl: Workload, device="cpu", seed: int | None = None, ring_cap: int | None = None):
    """Inputs of one CSA layer: raw KV / indexer-key rings, the compressed CSA
    cache and indexer-key cache, queries, indexer queries and weights, gates."""
    rng = _Rng(wl.seed * 7919 + 11 if seed is None else seed, device)
    t_end = wl.t_end
    n_c = _n_slots(t_end, wl.csa_stride)
    cap = ring_cap or _default_ring(wl, wl.csa_pool, wl.csa_stride)
    L = {"kind": "csa", "wl": wl, "t_end": t_end}
    kw = dict(d_nope=wl.d_nope, d_rope=wl.d_rope, fmt=wl.fmt, scale_pad=8)
    L["ring_k"] = _cache(rng, wl, wl.B, cap, ring=True, **kw)
    L["ring_v"] = _cache(rng, wl, wl.B, cap, ring=True, **kw) if wl.separate_v else None
    ik_fmt = "f32" if wl.fmt == "f32" else wl.ik_fmt
    ik_kw = dict(d_nope=wl.d_I, d_rope=0, fmt=ik_fmt, scale_pad=1 if ik_fmt == "e4m3vec" else 2)
    L["ring_ik"] = _cache(rng, wl, wl.B, cap, ring=True, **ik_kw)
    for key in ("ring_k", "ring_v", "ring_ik"):
        if L[key] is not None:
            _poison_ring(L[key], t_end)
    L["comp_k"] = _cache(rng, wl, wl.B, max(n_c, 1), ring=False, **kw)
    L["comp_v"] = _cache(rng, wl, wl.B, max(n_c, 1), ring=False, **kw) if wl.separate_v else None
    L["comp_ik"] = _cache(rng, wl, wl.B, max(n_c, 1), ring=False, **ik_kw)
    L["n_comp"] = n_c
    L["q"] = _queries(rng, wl)
    if wl.fmt == "f32":
        L["q_ik"] = rng.normal(wl.B, wl.Tq, wl.H_I, wl.d_I)
        L["q_ik_scale"] = None
    elif ik_fmt == "mxfp4":
        L["q_ik"], L["q_ik_scale"] = _mxfp4_planes(rng, (wl.B, wl.Tq, wl.H_I), wl.d_I)
    else:
        L["q_ik"], L["q_ik_scale"] = _fp8_planes(rng, (wl.B, wl.Tq, wl.H_I), wl.d_I, 1,
                                                 wl.d_I if ik_fmt == "e4m3vec" else 64)
    L["head_w"] = rng.normal(wl.B, wl.Tq, wl.H_I) / math.sqrt(wl.H_I)
    L["gate_w"] = rng.normal(wl.D, std=0.1)
    L["gate_b"] = rng.normal(wl.csa_pool, std=0.1)
    if wl.gate_mode == "channel":
        _channel_gates(rng, L, wl.D, wl.csa_pool, wl.d_I)
    L["pool"], L["stride"] = wl.csa_pool, wl.csa_stride
    L["q_pos"], L["ctx_len"] = _positions(wl, device)
    L["needles"] = _needle_positions(rng, wl, t_end)
    for b in range(wl.B):
        hstar = int(torch.argmax(L["head_w"][b, 0]).item())
        for p in L["needles"][b].tolist():
            j = p // wl.csa_stride
            if j >= n_c:
                continue
            if wl.fmt == "f32":
                L["comp_ik"]["data"][b, j] = L["q_ik"][b, 0, hstar] * 4.0
            elif ik_fmt == "mxfp4":
                # the head's codes, every block exponent 2 higher (x4)
                L["comp_ik"]["data"][b, j] = L["q_ik"][b, 0, hstar]
                L["comp_ik"]["scale"][b, j] = L["q_ik_scale"][b, 0, hstar] + 2
            else:
                L["comp_ik"]["data"][b, j] = L["q_ik"][b, 0, hstar]
                nbq = L["q_ik_scale"].shape[-1]
                L["comp_ik"]["scale"][b, j, :nbq] = L["q_ik_scale"][b, 0, hstar, :nbq] * 4.0
            _plant_kv_needle(L["comp_k"], b, j, L["q"][b, 0, 0], rng)
    if wl.page_block:
        for i, key in enumerate(("comp_k", "comp_v", "comp_ik")):
            if L.get(key) is not None:
                L[key] = page_cache(L[key], wl.page_block, seed=wl.seed * 31 + i)
    return L


def make_hca_layer(wl: Workload, device="cpu", seed: int | None = None, ring_cap: int | None = None):
    """Inputs of one HCA layer: raw KV ring, the compressed HCA cache, queries, gates."""
    rng = _Rng(wl.seed * 7919 + 23 if seed is None else seed, device)
    t_end = wl.t_end
    n_h = _n_slots(t_end, wl.hca_stride)
    cap = ring_cap or _default_ring(wl, wl.hca_pool, wl.hca_stride)
    L = {"kind": "hca", "wl": wl, "t_end": t_end}
    kw = dict(d_nope=wl.d_nope, d_rope=wl.d_rope, fmt=wl.fmt, scale_pad=8)
    L["ring_k"] = _cache(rng, wl, wl.B, cap, ring=True, **kw)
    L["ring_v"] = _cache(rng, wl, wl.B, cap, ring=True, **kw) if wl.separate_v else None
    for key in ("ring_k", "ring_v"):
        if L[key] is not None:
            _poison_ring(L[key], t_end)
    L["comp_k"] = _cache(rng, wl, wl.B, max(n_h, 1), ring=False, **kw)
    L["comp_v"] = _cache(rng, wl, wl.B, max(n_h, 1), ring=False, **kw) if wl.separate_v else None
    L["n_comp"] = n_h
    L["q"] = _queries(rng, wl)
    L["gate_w"] = rng.normal(wl.D, std=0.1)
    L["gate_b"] = rng.normal(wl.hca_pool, std=0.1)
    if wl.gate_mode == "channel":
        _channel_gates(rng, L, wl.D, wl.hca_pool, None)
    L["pool"], L["stride"] = wl.hca_pool, wl.hca_stride
    L["q_pos"], L["ctx_len"] = _positions(wl, device)
    L["needles"] = _needle_positions(rng, wl, t_end)
    for b in range(wl.B):
        for p in L["needles"][b].tolist():
            j = p // wl.hca_stride
            if j < n_h:
                _plant_kv_needle(L["comp_k"], b, j, L["q"][b, 0, 0], rng)
    if wl.page_block:
        for i, key in enumerate(("comp_k", "comp_v")):
            if L.get(key) is not None:
                L[key] = page_cache(L[key], wl.page_block, seed=wl.seed * 31 + 7 + i)
    return L


def _default_ring(wl: Workload, pool: int, stride: int) -> int:
    """Smallest power of two holding the window and, for a prefill chunk, every
    position the chunk's queries and pooling windows can reach."""
    need = max(wl.window, pool)
    if wl.prefill:
        need = wl.Tq + max(wl.window, pool)
    cap = 1
    while cap < need:
        cap *= 2
    return cap


def random_selection(wl: Workload, k: int, seed: int = 17, device="cpu"):
    """A seeded stand-in for an indexer selection: for every query row, k
    distinct visible CSA entries in ascending order (all visible entries when
    fewer than k), -1 padded.  int32 [B][Tq][k]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    pos, _ = _positions(wl, "cpu")
    out = torch.full((wl.B, wl.Tq, k), -1, dtype=torch.int32)
    for b in range(wl.B):
        for t in range(wl.Tq):
            n = int(pos[b, t] + 1) // wl.csa_stride
            if n <= k:
                out[b, t, :n] = torch.arange(n, dtype=torch.int32)
            else:
                # oversample, de-duplicate, keep k at random, sort
                u = torch.empty(0, dtype=torch.int64)
                while u.numel() < k:
                    u = torch.unique(torch.cat([u, torch.randint(0, n, (2 * k,), generator=g)]))
                pick = u[torch.randperm(u.numel(), generator=g)[:k]].sort().values
                out[b, t] = pick.to(torch.int32)
    return out.to(device)


def page_cache(c: dict, block_size: int, seed: int = 0, spare_blocks: int = 3,
               unmapped_tail: int = 0) -> dict:
    """Paged copy of a compressed cache (ring = 0): every sequence's slots cut
    into blocks of `block_size`, the blocks placed in a shared pool in a
    seeded random order (with `spare_blocks` unused blocks), and the block
    table [B][cap / block_size] int32 that maps logical block (b, i) to its
    pool block.  The capacity is rounded up to whole blocks (the new slots
    hold zeros), and `unmapped_tail` further logical blocks per sequence get
    no pool block (table entry -1), as in a pool that allocates on demand.
    Storage only: every logical slot keeps its bytes."""
    assert not c["ring"] and block_size >= 1 and block_size & (block_size - 1) == 0
    data = c["data"]
    B, cap = data.shape[0], int(c["cap"])
    nb = (cap + block_size - 1) // block_size
    n = B * nb + spare_blocks
    g = torch.Generator().manual_seed(seed)
    phys = torch.randperm(n, generator=g)[: B * nb]        # pool block of each logical block
    out = dict(c)
    for key in ("data", "scale", "rope"):
        t = c.get(key)
        if t is None:
            continue
        tail = tuple(t.shape[2:])
        padded = torch.zeros((B, nb * block_size) + tail, dtype=t.dtype, device=t.device)
        padded[:, :cap] = t
        pool = torch.zeros((1, n * block_size) + tail, dtype=t.dtype, device=t.device)
        pool.view((n, block_size) + tail)[phys.to(t.device)] = \
            padded.reshape((B * nb, block_size) + tail)
        out[key] = pool
    table = phys.view(B, nb).to(torch.int32)
    if unmapped_tail:
        table = torch.cat([table, torch.full((B, unmapped_tail), -1, dtype=torch.int32)], 1)
    out["cap"] = (nb + unmapped_tail) * block_size
    out["block_table"] = table.to(data.device)
    out["block_size"] = block_size
    out["num_blocks"] = n
    return out
