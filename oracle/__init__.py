"""CPU oracle (fp64, numpy) of the eviction/compaction path.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the package smoke check and
the CPU-baseline leg of the benchmark, never by the product path.  It shares no
code with the CUDA library.
"""
from . import path, cache, beacon, decode, stepkv, stream  # noqa: F401
