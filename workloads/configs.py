"""Workload shapes.

The five named workloads restate the decode and chunked-prefill cases that the
DeepSeek-V4 coverage describes: CSA pools 4 tokens with overlapping windows and
keeps the top 512 (V4-Flash) or 1,024 (V4-Pro) entries picked by the lightning
indexer; HCA pools 128 tokens and attends densely; both add a 128-token raw
sliding window; the cache holds FP8 for non-RoPE dims and BF16 for the last 64
(RoPE) dims (golem.de "Komprimierte Erinnerung fuer laengere Kontexte";
chaosnode.de "Hybrid Attention: CSA und HCA"; webconsulting.at "Das
Wichtigste").  Smaller `parity_*` workloads keep the same structure at sizes a
CPU reference finishes in seconds while spanning several kernel tiles and a
ragged tail.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    B: int                 # sequences
    T: int                 # decode: tokens incl. the query; prefill: cached tokens before the chunk
    Tq: int = 1            # query tokens per sequence (1 = decode)
    prefill: bool = False  # True: Tq new tokens at positions T .. T+Tq-1
    Hq: int = 64           # query heads sharing one KV head (MQA)
    fmt: str = "e4m3"      # "e4m3": FP8 E4M3 + per-64 fp32 scales + BF16 RoPE dims; "f32"
    ik_fmt: str = "e4m3vec"  # indexer keys / queries: "e4m3vec" (one fp32 scale per
                             # vector), "e4m3" (per-64 blocks) or "mxfp4" (FP4 E2M1 with
                             # an E8M0 exponent per 32 dims); f32 workloads: "f32"
    d_nope: int = 448
    d_rope: int = 64
    separate_v: bool = False   # f32 tiny workload keeps separate K and V
    H_I: int = 64          # lightning-indexer heads
    d_I: int = 128         # lightning-indexer head dim
    k: int = 1024          # CSA top-k
    csa_pool: int = 8
    csa_stride: int = 4
    hca_pool: int = 128
    hca_stride: int = 128
    window: int = 128
    needles: int = 0
    needle_mode: str = "uniform"   # "uniform" | "loguniform"
    q_prescale: bool = False       # tiny workload: Q already multiplied by 1/sqrt(head dim)
    gate_mode: str = "scalar"      # "scalar": g_r = w . k + b[r]; "channel": one gate per
                                   # channel, g_{r,c} = w_c k_c + b[r][c]
    page_block: int = 0            # > 0: compressed caches paged in blocks of this many
                                   # entries (shuffled pool + block table)
    seed: int = 0

    @property
    def D(self) -> int:
        return self.d_nope + self.d_rope

    @property
    def sm_scale(self) -> float:
        return 1.0 if self.q_prescale else 1.0 / math.sqrt(self.D)

    @property
    def t_end(self) -> int:
        """Tokens present after this step (decode: T; prefill: T + Tq)."""
        return self.T + self.Tq if self.prefill else self.T

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # tiny CPU-checkable decode, all fp32, separate K and V, head dim 128
    "tiny": Workload("tiny", B=1, T=4096, Hq=8, fmt="f32", d_nope=64, d_rope=64,
                     separate_v=True, H_I=4, d_I=32, k=64, q_prescale=True),
    # V4-Flash-like batched decode
    "flash": Workload("flash", B=8, T=65536, k=512, needles=16),
    # V4-Pro-like decode
    "pro": Workload("pro", B=4, T=131072, k=1024, needles=16),
    # 1M-token decode (the measured workload)
    "long": Workload("long", B=1, T=1048576, k=1024, needles=64, needle_mode="loguniform"),
    # chunked prefill: 8,192 new tokens on a 1M cached context
    "prefill": Workload("prefill", B=1, T=1048576, Tq=8192, prefill=True, k=1024),
    # parity-sized variants of the FP8 layout
    "parity_decode": Workload("parity_decode", B=3, T=9_999, k=256, needles=4),
    "parity_prefill": Workload("parity_prefill", B=1, T=3_000, Tq=300, prefill=True, k=128),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]
