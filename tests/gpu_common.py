"""Shared set-up of the GPU parity tests: device placement of generated layers
and the loud failure when the CUDA library or a GPU is missing."""
from __future__ import annotations

import numpy as np
import pytest
import torch


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but no CUDA device is visible")
    import compressed_sparse_kv_softmax_b200 as C   # raises ImportError without libcskv.so
    return C


def to_device(L, dev="cuda"):
    """Copy a generated layer (CPU tensors) to the device; the CPU copy stays
    the oracle's input."""
    out = {}
    for k, v in L.items():
        if isinstance(v, torch.Tensor):
            out[k] = v.to(dev)
        elif isinstance(v, dict):
            out[k] = {kk: (vv.to(dev) if isinstance(vv, torch.Tensor) else vv)
                      for kk, vv in v.items()}
        else:
            out[k] = v
    return out


def sample_rows(B, Tq, n=64):
    """All rows when few, else first 8, last 8 and evenly spaced ones."""
    rows = [(b, t) for b in range(B) for t in range(Tq)]
    if len(rows) <= n:
        return rows
    idx = sorted(set(list(range(8)) + list(range(len(rows) - 8, len(rows))) +
                     np.linspace(8, len(rows) - 9, n - 16).astype(int).tolist()))
    return [rows[i] for i in idx]
