"""B200-native 2-D TM Maxwell FDTD: forward, exact discrete adjoint and
adjoint-state model gradients, batched over shots.

The compute path is the C-ABI library ``libmwtm.so`` (CUDA, sm_100a) declared
in ``include/mw_tm.h``; ``mwtm`` is its thin ctypes binding.  ``synth`` builds
seeded synthetic inputs.  Importing the package does not load the library;
the first call into ``mwtm`` does, and raises if it is missing.
"""
__all__ = ["mwtm", "synth", "api"]
