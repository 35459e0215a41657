"""The fp64 oracle against closed forms, special cases and worked examples."""
import pytest

import oracle.muon_oracle as ora
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(pin):
    pin(ora)


def test_every_oracle_function_is_pinned():
    """Each public oracle function is exercised by at least one pin."""
    import inspect
    import oracle_pins
    src = inspect.getsource(oracle_pins)
    for name in ("nesterov_momentum", "frobenius_normalise", "newton_schulz_direct",
                 "newton_schulz_gram", "rms_scale", "apply_update", "muon_update",
                 "muon_step"):
        assert f"ora.{name}(" in src, name
