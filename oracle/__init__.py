"""Plain CPU oracle of the CSA2 hot path (float64 numpy, fp32 where a decision is quantised).

TEST INFRASTRUCTURE ONLY.  It exists to check the CUDA library; it shares no
code with it and is never on the product path.  Only tests/,
__graft_entry__.smoke() and bench.py's CPU-baseline leg may import it.

Parity status: every function here is pinned by tests/test_oracle_*.py against
the pages' figures, closed forms, invariants or brute force, except the points
the pages leave open (compressor weights, indexer formula, exponent rounding,
softmax scale), which are readings and therefore "parity unpinned" with respect
to the real model (they are pinned only as restatements of those readings).
"""
from . import formats, csa2  # noqa: F401
