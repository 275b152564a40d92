"""B200-native FwPKM retrieve + chunk-write loop.

The hot path lives in ``libfwpkm.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/fwpkm.h``).  ``sparse_weight_memory_chunk_b200.fwpkm`` is the
thin ctypes binding; ``inputs`` draws seeded synthetic workloads.  Importing the
package does not load the CUDA library; the binding loads it on first use and
raises if it is missing.
"""
