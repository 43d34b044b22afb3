"""B200-native Muon optimizer step (sm_100a kernels behind a C ABI).

The compute lives in ``libmuon.so`` (built from ``csrc/``); this package only
marshals arguments into it.  Importing the package does not load the library;
the first call that needs it does, and raises if it is missing.
"""

__all__ = ["workloads"]
