"""DSA region-sparse GQA on B200 (sm_100a).

The compute lives in ``libdsa.so`` (hand-written CUDA kernels behind a C-ABI, see
``include/dsa.h``); :mod:`sparse_long_context_dsa_b200.dsa` is the thin ctypes binding
with the same call names.  :mod:`sparse_long_context_dsa_b200.workloads` draws the
seeded synthetic inputs.  Importing the package loads nothing; the binding loads the
library on first use and raises if it is missing.
"""
__all__ = ["dsa", "workloads"]
