"""B200-native speculative-decoding attention / acceptance kernels (sm_100a, C-ABI library).

The compute path is the shared library ``libsdattn.so`` built from ``csrc/`` (hand-written CUDA
for sm_100a behind an ``extern "C"`` interface declared in ``include/sd_attn.h``).  The Python
binding in :mod:`.sdattn` only marshals arguments; :mod:`.inputs` draws seeded synthetic inputs.
Importing the package loads nothing; the library is loaded on first use and a missing or
unbuildable library raises immediately (there is no CPU fallback).
"""

__all__ = ["inputs", "sdattn"]
