"""CPU oracle for the HISA / DSA indexers.

TEST INFRASTRUCTURE ONLY: a plain float64 restatement of the method used to
check the CUDA library.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it.  It shares no code with the
CUDA path and the product path never calls it.
"""
from . import hisa_oracle, ofp8, run  # noqa: F401
