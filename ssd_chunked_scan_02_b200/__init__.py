"""B200-native SSD (structured state space duality) layer.

The compute lives in ``libssd_b200.so`` (hand-written sm_100a CUDA behind the
C ABI declared in ``include/ssd.h``); ``ssd_chunked_scan_02_b200.ssd`` is the
thin ctypes binding with the same entry-point names, and
``ssd_chunked_scan_02_b200.inputs`` draws seeded synthetic inputs.  Importing
the package loads nothing: the shared library is opened on first use, and a
missing library is an error (there is no CPU fallback).
"""
