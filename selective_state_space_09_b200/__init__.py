"""B200-native fused linear-recurrence scan (rglru, rotlru, S6, SSD, GLA) behind a C ABI.

``h_t = a_t (.) h_{t-1} + b_t, y_t = readout(h_t)`` run forward and backward over the whole
sequence in one pass of hand-written sm_100a kernels, with a segment checkpoint-and-recompute
backward.  The C ABI is declared in ``include/lrscan.h``; ``lrscan`` is its thin Python binding
(argument marshalling only).  ``inputs`` holds the seeded workload generators.

Attribute access such as ``selective_state_space_09_b200.rglru`` loads the CUDA library and fails
loudly if it has not been built; there is no CPU fallback.
"""
import importlib

__all__ = ["lrscan", "inputs", "rglru", "rotlru", "s6", "ssd", "gla"]


def __getattr__(name):
    if name in ("lrscan", "inputs"):
        return importlib.import_module("." + name, __name__)
    if name in ("rglru", "rotlru", "s6", "ssd", "gla", "LrScanError"):
        return getattr(importlib.import_module(".lrscan", __name__), name)
    raise AttributeError(name)
