"""B200-native Mamba-2 selective-scan (SSD) library.

The compute runs in ``libssd.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/ssd.h``).  ``ssd`` is the thin Python binding over it;
``datagen`` draws the seeded synthetic workloads.  Importing the package does
not load the CUDA library; ``ssd.load()`` does, and fails loudly if it is
missing.
"""
__all__ = ["ssd", "datagen"]
