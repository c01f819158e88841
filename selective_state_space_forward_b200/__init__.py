"""B200-native Mamba-2 / SSD selective-state-space mixer scan.

The compute path is the C-ABI library ``libssd.so`` (hand-written CUDA for
sm_100a, declared in ``include/ssd.h``); ``ssd`` is its thin ctypes binding and
``synthetic`` draws the seeded workloads.  Importing the package loads
nothing: the binding opens the library on first use and raises if it is
missing.
"""
__all__ = ["ssd", "synthetic"]
