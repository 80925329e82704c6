"""fp64 CPU oracle of the Hybrid Linear Temporal Attention layer (forward pass
and its reverse-mode derivatives).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, the package smoke check and
the benchmark's CPU-baseline leg, never by the product path.  It shares no
code with the CUDA library; the only thing both sides use is ``workloads``,
which generates inputs and holds none of the layer's arithmetic.

Two independent implementations:

* ``hlta_oracle.c`` (compiled here with gcc + OpenMP, loaded with ctypes):
  explicit-mask softmax attention (SWA / DSWA), the token-by-token gated delta
  recurrence, and its chunk regrouping.
* ``twin``: a NumPy restatement of the same definitions in pure Python loops,
  for tiny cases only.

Parity pins of every function: ``tests/test_oracle.py``.
"""
from .core import (attention, attention_rows, forward, gdn, gdn_chunked, num_threads,
                   build, library_path, dswa_span, attention_backward, gdn_backward, backward)
from .chunk_backward import gdn_backward_chunked
from . import fp8

__all__ = ["attention", "attention_rows", "forward", "gdn", "gdn_chunked", "num_threads",
           "build", "library_path", "dswa_span", "attention_backward", "gdn_backward", "backward",
           "gdn_backward_chunked"]
