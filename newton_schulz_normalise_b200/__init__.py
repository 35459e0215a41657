"""B200-native Muon / DMuon optimizer step.

The compute path lives in the CUDA library ``libdmuon.so`` (C ABI declared in
``include/dmuon.h``); ``newton_schulz_normalise_b200.binding`` marshals torch
tensors into that ABI.  Importing this package does not load the library; the
binding does, and raises if it is missing.
"""
__all__ = ["binding", "workloads"]
