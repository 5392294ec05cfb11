"""Seeded synthetic inputs for the hybrid compressed attention path.

This package holds shapes and random-number recipes only: it performs none of
the method's arithmetic (no pooling, scoring, selection or attention).  Both
the CUDA path's tests/bench and the CPU oracle consume what it produces.
"""
from .configs import Workload, WORKLOADS, get
from .generate import (make_csa_layer, make_hca_layer, e4m3_from_float, random_selection,
                       page_cache)

__all__ = ["Workload", "WORKLOADS", "get",
           "make_csa_layer", "make_hca_layer", "e4m3_from_float", "random_selection", "page_cache"]
