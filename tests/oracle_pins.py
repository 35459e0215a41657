"""Pins for the fp64 oracle: checks against mathematics, not against itself.

Each ``pin_*`` takes an object exposing the oracle's functions (the real
``oracle.muon_oracle`` module, or a copy with a planted mistake in
``test_oracle_mutants.py``) and raises AssertionError when the function under
test disagrees with what the definitions fix:

* closed form: Newton-Schulz is an odd matrix polynomial, so for
  X0 = U diag(s) V^T its result is U diag(f_K(s)) V^T with f_K the scalar
  quintic p(s) = a s + b s^3 + c s^5 composed K times (SVD from LAPACK);
* the polar factor of the result equals the polar factor U V^T of the input;
* direct and Gram-space recursions agree to 1e-10 (fp64, tiny inputs);
* singular values of the result lie in [0.6, 1.2] when the normalised input's
  smallest singular value is >= 0.005 (where f_5 stays in that band);
* special cases: rank one, diagonal, zero input, zero steps, orthonormal rows,
  orthogonal equivariance, transpose and sign symmetry, scale invariance;
* exact integer momentum cases and hand-derived worked examples
  (``tests/golden/worked_examples.json``, exact rational arithmetic).
"""
from __future__ import annotations

import json
import math
from pathlib import Path

import numpy as np

COEFFS = (3.4445, -4.7750, 2.0315)   # the library's documented quintic constants
GOLDEN = json.loads((Path(__file__).parent / "golden" / "worked_examples.json").read_text())


def quintic(s, steps, coeffs=COEFFS):
    """Scalar composition f_K(s): p applied K times (not the matrix code)."""
    a, b, c = coeffs
    s = np.asarray(s, dtype=np.float64)
    for _ in range(steps):
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def closed_form_ns(X0, steps):
    """U f_K(S) V^T from an SVD of X0 (X0 has rows <= cols)."""
    U, S, Vt = np.linalg.svd(X0, full_matrices=False)
    return (U * quintic(S, steps)) @ Vt


def rel(x, y):
    y = np.asarray(y, np.float64)
    d = np.linalg.norm(np.asarray(x, np.float64) - y)
    n = np.linalg.norm(y)
    return d / n if n > 0 else d


def _rng(seed):
    return np.random.default_rng(seed)


def _normalised(rows, cols, seed):
    X = _rng(seed).standard_normal((rows, cols))
    return X / np.linalg.norm(X)


SHAPES = [(8, 32), (16, 16), (24, 40), (5, 7), (64, 256)]


def pin_closed_form_direct(ora):
    for i, (m, n) in enumerate(SHAPES):
        X0 = _normalised(m, n, 100 + i)
        for K in (1, 2, 5):
            got = ora.newton_schulz_direct(X0, K)
            assert got.shape == (m, n)
            e = rel(got, closed_form_ns(X0, K))
            assert e < 1e-12, (m, n, K, e)


def pin_closed_form_gram(ora):
    for i, (m, n) in enumerate(SHAPES):
        X0 = _normalised(m, n, 200 + i)
        got = ora.newton_schulz_gram(X0, 5)
        assert got.shape == (m, n)
        e = rel(got, closed_form_ns(X0, 5))
        assert e < 1e-10, (m, n, e)


def pin_direct_equals_gram(ora):
    for i, (m, n) in enumerate([(8, 32), (16, 16), (32, 96), (64, 256)]):
        X0 = _normalised(m, n, 300 + i)
        d = ora.newton_schulz_direct(X0, 5)
        g = ora.newton_schulz_gram(X0, 5)
        assert rel(g, d) < 1e-10, (m, n, rel(g, d))


def pin_polar_factor(ora):
    """Singular vectors of the output match the input's polar factor U V^T."""
    for i, (m, n) in enumerate([(8, 32), (12, 12), (20, 50)]):
        X0 = _normalised(m, n, 400 + i)
        U, _, Vt = np.linalg.svd(X0, full_matrices=False)
        O = ora.newton_schulz_direct(X0, 5)
        Uo, So, Vto = np.linalg.svd(O, full_matrices=False)
        assert np.all(So > 0)
        assert rel(Uo @ Vto, U @ Vt) < 1e-9
        # U^T O V is diagonal with non-negative entries
        D = U.T @ O @ Vt.T
        off = D - np.diag(np.diag(D))
        assert np.linalg.norm(off) < 1e-12 * np.linalg.norm(D)
        assert np.all(np.diag(D) > 0)


def pin_singular_value_band(ora):
    # rectangular Gaussians with cols >= 2 rows: normalised s_min well above 0.005
    for i, (m, n) in enumerate([(16, 64), (32, 64), (48, 200)]):
        X0 = _normalised(m, n, 500 + i)
        s_in = np.linalg.svd(X0, compute_uv=False)
        assert s_in.min() >= 0.005
        s = np.linalg.svd(ora.newton_schulz_direct(X0, 5), compute_uv=False)
        assert s.min() >= 0.6 and s.max() <= 1.2, (s.min(), s.max())
    # constructed spectrum across [0.005, 1]
    rng = _rng(510)
    m, n = 24, 40
    Q1, _ = np.linalg.qr(rng.standard_normal((m, m)))
    Q2, _ = np.linalg.qr(rng.standard_normal((n, m)))
    sig = np.geomspace(0.005, 1.0, m)
    X0 = (Q1 * sig) @ Q2.T
    s = np.linalg.svd(ora.newton_schulz_direct(X0, 5), compute_uv=False)
    assert s.min() >= 0.6 and s.max() <= 1.2, (s.min(), s.max())


def pin_diagonal_entrywise(ora):
    d = np.array([1.0, 0.7071067811865476, 0.5, 0.25, 0.125, 0.0625, 0.01, -0.3])
    X0 = np.diag(d)
    got = ora.newton_schulz_direct(X0, 5)
    assert np.allclose(got, np.diag(quintic(d, 5)), rtol=0, atol=1e-13)
    got = ora.newton_schulz_gram(X0, 5)
    assert np.allclose(got, np.diag(quintic(d, 5)), rtol=0, atol=1e-11)
    # published-constant sanity of the scalar map itself (recomputed, not page data)
    assert abs(quintic(1.0, 1) - 0.701) < 1e-15
    assert abs(quintic(1.0, 5) - 0.696436409470) < 1e-11
    assert abs(quintic(0.5, 5) - 0.765438530454) < 1e-11


def pin_rank_one(ora):
    rng = _rng(600)
    u = rng.standard_normal(6)
    v = rng.standard_normal(11)
    U = np.outer(u, v)
    X0 = ora.frobenius_normalise(U, 0.0)
    O = ora.newton_schulz_direct(X0, 5)
    expect = quintic(1.0, 5) * np.outer(u / np.linalg.norm(u), v / np.linalg.norm(v))
    assert rel(O, expect) < 1e-12


def pin_orthonormal_rows(ora):
    rng = _rng(610)
    m, n = 6, 15
    Q, _ = np.linalg.qr(rng.standard_normal((n, m)))
    U = Q.T                                    # orthonormal rows
    X0 = ora.frobenius_normalise(U, 0.0)        # all singular values 1/sqrt(m)
    O = ora.newton_schulz_direct(X0, 5)
    assert rel(O, quintic(1 / math.sqrt(m), 5) * math.sqrt(m) * X0) < 1e-12


def pin_zero_and_zero_steps(ora):
    Z = np.zeros((4, 9))
    X0 = ora.frobenius_normalise(Z)
    assert np.all(X0 == 0)
    assert np.all(ora.newton_schulz_direct(X0, 5) == 0)
    assert np.all(ora.newton_schulz_gram(X0, 5) == 0)
    X0 = _normalised(5, 9, 620)
    assert np.array_equal(ora.newton_schulz_direct(X0, 0), X0)
    assert rel(ora.newton_schulz_gram(X0, 0), X0) < 1e-15


def pin_normalise(ora):
    X = _rng(630).standard_normal((7, 13)) * 3.0
    X0 = ora.frobenius_normalise(X, 0.0)
    assert abs(np.linalg.norm(X0) - 1.0) < 1e-14
    X0e = ora.frobenius_normalise(X, 0.5)
    assert abs(np.linalg.norm(X0e) - np.linalg.norm(X) / (np.linalg.norm(X) + 0.5)) < 1e-14


def pin_equivariance_and_symmetry(ora):
    rng = _rng(640)
    m, n = 9, 21
    X0 = _normalised(m, n, 641)
    P, _ = np.linalg.qr(rng.standard_normal((m, m)))
    R, _ = np.linalg.qr(rng.standard_normal((n, n)))
    base = ora.newton_schulz_direct(X0, 5)
    assert rel(ora.newton_schulz_direct(P @ X0 @ R, 5), P @ base @ R) < 1e-12
    assert rel(ora.newton_schulz_direct(-X0, 5), -base) < 1e-15
    # NS on the tall transpose equals the transpose of NS on the wide matrix
    assert rel(ora.newton_schulz_direct(X0.T, 5), base.T) < 1e-12
    # scale invariance of normalise + NS
    U = rng.standard_normal((m, n))
    a = ora.newton_schulz_direct(ora.frobenius_normalise(U, 0.0), 5)
    b = ora.newton_schulz_direct(ora.frobenius_normalise(37.5 * U, 0.0), 5)
    assert rel(a, b) < 1e-13


def pin_momentum_exact(ora):
    G = np.array([[1.0, -2.0, 3.0], [4.0, 0.0, -6.0]])
    B = np.array([[2.0, 2.0, -2.0], [0.0, 8.0, 4.0]])
    Bn, U = ora.nesterov_momentum(G, B, 0.5, True)
    assert np.array_equal(Bn, np.array([[2.0, -1.0, 2.0], [4.0, 4.0, -4.0]]))
    assert np.array_equal(U, np.array([[2.0, -2.5, 4.0], [6.0, 2.0, -8.0]]))
    Bn2, U2 = ora.nesterov_momentum(G, B, 0.5, False)
    assert np.array_equal(Bn2, Bn) and np.array_equal(U2, Bn)
    # zero buffer, mu = 0.95: B' = G, U = 1.95 G
    Bn, U = ora.nesterov_momentum(G, np.zeros_like(G), 0.95, True)
    assert np.array_equal(Bn, G) and np.allclose(U, 1.95 * G, rtol=1e-15, atol=0)


def pin_apply_exact(ora):
    W = np.array([[1.0, -2.0], [0.5, 4.0], [0.0, 1.0]])     # 3 x 2: scale uses 3
    O = np.array([[1.0, 0.0], [0.0, -1.0], [2.0, 1.0]])
    lr, wd = 0.1, 0.5
    got = ora.apply_update(W, O, lr, wd)
    s = 0.2 * math.sqrt(3.0)
    expect = 0.95 * W - 0.1 * s * O
    assert np.allclose(got, expect, rtol=0, atol=1e-15)
    assert abs(ora.rms_scale(3, 2) - s) < 1e-15
    assert abs(ora.rms_scale(256, 512) - 0.2 * math.sqrt(512)) < 1e-13


def pin_golden_rank1(ora):
    for key in ("rank1_row_1x2", "rank1_col_2x1", "rank1_row_momentum_1x2"):
        c = GOLDEN["cases"][key]
        shape = (c["rows"], c["cols"])
        G = np.array(c["G"]).reshape(shape)
        B = np.array(c["B"]).reshape(shape)
        W = np.array(c["W"]).reshape(shape)
        Wn, Bn, O = ora.muon_step(W, G, B, lr=c["lr"], wd=c["wd"], mu=c["mu"],
                                  steps=c["ns_steps"], eps=c["eps"], nesterov=True)
        assert np.allclose(Bn.ravel(), c["B_new"], rtol=0, atol=1e-15), key
        assert np.allclose(O.ravel(), c["O"], rtol=1e-13, atol=0), key
        assert np.allclose(Wn.ravel(), c["W_new"], rtol=1e-14, atol=1e-16), key


def pin_golden_diag(ora):
    for key in ("diag_2x2", "diag_3x3"):
        c = GOLDEN["cases"][key]
        G = np.array(c["G"])
        B = np.array(c["B"])
        W = np.array(c["W"])
        for variant in ("direct", "gram"):
            Wn, Bn, O = ora.muon_step(W, G, B, lr=c["lr"], wd=c["wd"], mu=c["mu"],
                                      steps=c["ns_steps"], eps=c["eps"], variant=variant)
            assert np.allclose(O, np.diag(c["O_diag"]), rtol=0, atol=1e-11), (key, variant)
            assert np.allclose(Wn, np.array(c["W_new"]), rtol=0, atol=1e-12), (key, variant)


def pin_update_orientation(ora):
    """A tall matrix is handled as the transpose of the wide one."""
    rng = _rng(700)
    G = rng.standard_normal((30, 12))
    B = rng.standard_normal((30, 12))
    Bn_t, O_t = ora.muon_update(G, B, 0.9, 5, 1e-7)
    Bn_w, O_w = ora.muon_update(G.T, B.T, 0.9, 5, 1e-7)
    assert O_t.shape == (30, 12)
    assert rel(O_t, O_w.T) < 1e-13
    assert rel(Bn_t, Bn_w.T) == 0.0
    # the update is the closed form of the normalised Nesterov direction
    U = G + 0.9 * (0.9 * B + G)
    X0 = U.T / (np.linalg.norm(U) + 1e-7)
    assert rel(O_t, closed_form_ns(X0, 5).T) < 1e-12


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
