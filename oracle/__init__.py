"""CPU oracle for the Lightning Indexer forward pass (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg import this
package. The CUDA library never does.
"""
from .oracle import Oracle, build, default  # noqa: F401
