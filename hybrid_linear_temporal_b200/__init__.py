"""Hybrid Linear Temporal Attention forward pass for NVIDIA B200 (sm_100a).

The layer of the Kairos paper (arXiv 2606.16533, section 2.2): sliding-window
attention, dilated sliding-window attention and a gated delta memory, summed
with per-head gates.  All computation runs in ``libhlta.so`` (hand-written
CUDA for sm_100a behind the C ABI of ``include/hlta.h``); this package is the
Python binding.
"""
from .binding import (HLTA, Config, HltaError, load_library, header_symbols, LIB_PATH,
                      BRANCH_SWA, BRANCH_DSWA, BRANCH_GDN, BRANCH_ALL, GDN_DECAYED, GDN_PAGES,
                      WINDOW_CAUSAL, WINDOW_CENTRED)

__all__ = ["HLTA", "Config", "HltaError", "load_library", "header_symbols", "LIB_PATH",
           "BRANCH_SWA", "BRANCH_DSWA", "BRANCH_GDN", "BRANCH_ALL", "GDN_DECAYED", "GDN_PAGES",
           "WINDOW_CAUSAL", "WINDOW_CENTRED"]
