"""CPU oracle for the SVDQuant W4A4 linear layer.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only tests/,
__graft_entry__.smoke() and bench.py's CPU-baseline leg (and its
``--impl reference`` arm) may import, call or run anything in this package.
The CUDA library never links or calls it, and it shares no code, tables or
helpers with the CUDA path; the two meet only through the seeded input
generators in workloads.py.

Modules:
  formats   -- E2M1 / E4M3 / binary16 / bfloat16 / INT4 codecs
  svdquant  -- smoothing, truncated SVD split, residual, group quantization,
               the two branches and the epilogue, in float64

Every function is pinned by tests/test_oracle_*.py against definitions,
closed forms, invariants and brute force; no function is "parity unpinned".
"""
from . import formats, svdquant  # noqa: F401
