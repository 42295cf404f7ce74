"""B200-native Dust estimator hot path.

The CUDA kernels live in ``csrc/`` and are built into ``lib/libdust.so``, a
C-ABI library (declared in ``include/dust.h``).  ``dust`` is the thin Python
binding over it: it marshals torch CUDA tensors into pointers and streams and
calls the library; every step of the path runs in the library's kernels.
``inputs`` draws the seeded synthetic workloads.
"""
