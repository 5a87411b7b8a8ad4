"""B200-native selective diagonal state-space scan with an exact, chunk-tiled gradient.

The compute lives in ``libssm_scan.so`` (hand-written sm_100a CUDA behind a C ABI, declared in
``include/ssm_scan.h``).  ``ssm_scan`` is the thin ctypes binding over it; ``inputs`` holds the
seeded synthetic input generators.  Importing this package loads nothing: the shared library is
opened on first use and its absence raises immediately (there is no CPU fallback).
"""

__all__ = ["inputs", "ssm_scan"]
