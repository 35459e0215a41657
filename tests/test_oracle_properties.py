"""Property-based pins of the Newton-Schulz oracle (no GPU): over random
small shapes, scales and step counts, the direct iteration equals its SVD
closed form U f_K(S) V^T, the Gram form equals the direct form, and the map
is odd, commutes with transposition and ignores the input's scale."""
import numpy as np
import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402

import oracle.muon_oracle as ora  # noqa: E402
from oracle_pins import closed_form_ns, rel  # noqa: E402

shapes = st.tuples(st.integers(1, 24), st.integers(1, 40))


def _x(seed, m, n, scale=1.0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((m, n)) * scale


@settings(max_examples=60, deadline=None)
@given(shape=shapes, seed=st.integers(0, 2 ** 31 - 1), steps=st.integers(0, 7))
def test_direct_matches_svd_closed_form(shape, seed, steps):
    m, n = shape
    X0 = ora.frobenius_normalise(_x(seed, m, n))
    got = ora.newton_schulz_direct(X0, steps)
    assert got.shape == (m, n)
    assert rel(got, closed_form_ns(X0, steps)) < 1e-10


@settings(max_examples=60, deadline=None)
@given(shape=shapes, seed=st.integers(0, 2 ** 31 - 1), steps=st.integers(1, 6))
def test_gram_matches_direct(shape, seed, steps):
    m, n = shape
    X0 = ora.frobenius_normalise(_x(seed, m, n))
    assert rel(ora.newton_schulz_gram(X0, steps), ora.newton_schulz_direct(X0, steps)) < 1e-9


@settings(max_examples=40, deadline=None)
@given(shape=shapes, seed=st.integers(0, 2 ** 31 - 1),
       log_scale=st.floats(-4, 4, allow_nan=False, allow_infinity=False))
def test_odd_transposable_scale_free(shape, seed, log_scale):
    m, n = shape
    G = _x(seed, m, n)
    O = ora.muon_update(G, np.zeros((m, n)), 0.95, 5)[1]
    O_neg = ora.muon_update(-G, np.zeros((m, n)), 0.95, 5)[1]
    O_t = ora.muon_update(G.T, np.zeros((n, m)), 0.95, 5)[1]
    O_s = ora.muon_update(G * 10.0 ** log_scale, np.zeros((m, n)), 0.95, 5)[1]
    assert np.allclose(O_neg, -O, rtol=0, atol=1e-12)
    assert np.allclose(O_t, O.T, rtol=0, atol=1e-10)
    # eps = 1e-7 is added to the norm, so the scale drops out only up to the
    # relative size of eps (eps / ||U||), amplified by the log-log slope of the
    # composed quintic, at most 10.04 over (0, 1] (at s = 0.871)
    u = 1.95 * np.linalg.norm(G)  # ||U|| = (1 + mu) ||G|| from zero momentum
    assert rel(O_s, O) < 11 * 1e-7 * (1 / u + 1 / (u * 10.0 ** log_scale)) + 1e-12
