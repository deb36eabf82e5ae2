"""B200-native mLSTM forward with exponential gating.

The compute lives in a C-ABI shared library (``libxlstm_mlstm.so``, sources in
``csrc/``, declarations in ``include/xlstm_mlstm.h``) built for sm_100a.
``capi`` is the thin ctypes binding with the same entry-point names; ``inputs``
draws the seeded synthetic workloads.  Importing this package loads nothing:
the library is opened on first use and a missing library is an error, never a
fallback.
"""
__all__ = ["capi", "inputs", "build"]
