"""Lightning Indexer forward pass on B200 (sm_100a).

The compute path lives in the CUDA library ``libli.so`` (sources under ``csrc/``, C-ABI in
``include/li.h``). This package holds the thin ctypes binding over that library and the seeded
synthetic input generators used by the tests and the benchmark.
"""
