"""B200 (sm_100a) group-wise MinMax INT4/INT2 weight quantizer and weight-only linear.

The compute lives in ``libbq.so`` (CUDA kernels behind the C ABI of
``include/bq.h``); ``bq`` is its thin ctypes binding and ``synth`` the seeded
input generators.  Importing the package does not load the library; the first
``bq`` call does, and raises if it is missing.
"""
__all__ = ["bq", "synth", "build"]
