"""B200-native cached Flow-Matching Euler step with a prefix K/V cache.

The product is the C-ABI library ``libqi21.so`` (include/qi21.h) built from
``csrc/``; ``binding`` is its ctypes binding (same names) and ``runner`` a
device-buffer driver used by the tests and the benchmark. Submodules are
imported explicitly so that the build step runs before the library exists.
"""
__all__ = ["binding", "runner", "build"]
