"""fp64 CPU oracles of the Muon / DMuon step (``muon_oracle``) and of the
AdamW step for non-matrix parameters (``adamw_oracle``).

Test infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference legs, never by the library.
"""
from .muon_oracle import (  # noqa: F401
    DEFAULT_EPS, NS_A, NS_B, NS_C, NS_COEFFS, RMS_FACTOR,
    apply_update, frobenius_normalise, muon_step, muon_update,
    nesterov_momentum, newton_schulz_direct, newton_schulz_gram, rms_scale,
)
