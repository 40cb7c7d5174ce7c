"""Multi-Scale Retention hot path for B200 (sm_100a).

The compute lives in ``libretention.so`` (hand-written CUDA kernels behind a
C ABI declared in ``include/retention.h``); ``ops`` is the thin ctypes binding
that marshals torch tensors into those calls, ``workloads`` draws the seeded
synthetic inputs, ``build`` compiles the library.  Importing this package
does not load the library; the first call into ``ops`` does, and raises if
the library has not been built.
"""
