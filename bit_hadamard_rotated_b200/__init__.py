"""Packed low-bit, Hadamard-rotated linears on B200 (sm_100a).

The compute lives in libhq.so (include/hq.h); this package is its Python
binding (``hq``), the build script (``build``), the seeded synthetic inputs
(``synth``) and the multi-rank benchmark helpers (``dist``).
"""
from .hq import *  # noqa: F401,F403
