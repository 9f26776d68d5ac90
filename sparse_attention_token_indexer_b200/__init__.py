"""B200 (sm_100a) DSA token indexer and ADIndex group bank / refine.

The compute path is libadx.so (hand-written CUDA for sm_100a, C ABI in include/adx.h);
``indexer`` holds the Python entry points (argument marshalling only) and ``inputs`` the
seeded synthetic workloads. Importing the package does not load the library; the first
call does, and fails loudly if it has not been built.
"""

__all__ = ["indexer", "inputs"]
