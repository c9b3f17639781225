"""B200-native HiLS (Hierarchical Landmark Sparse) attention, forward hot path.

The compute lives in ``libhils.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/hils.h``).  :mod:`.hils` is a thin ctypes binding with
the same entry-point names; :mod:`.inputs` draws the seeded synthetic inputs.
Importing this package loads nothing; the binding loads the library on first
use and raises if it is missing.
"""
