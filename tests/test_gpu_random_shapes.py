"""The step's update against the fp64 oracle on seeded random shapes (1 to
400 rows and columns, both orientations, bf16 and fp32), several shape
groups per call: this crosses the resident kernel, the one-CTA and CTA-pair
GEMMs, the Gram and direct forms and the ragged-edge rules at sizes the
fixed cases do not name."""
import numpy as np
import pytest

from parity_helpers import check_momentum, gpu_update, make_inputs, oracle_update, rel_fro, to64

pytestmark = pytest.mark.gpu


def _shapes(seed, count):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(count):
        r, c = (int(x) for x in rng.integers(1, 401, size=2))
        out.append((r, c))
    return out


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_random_shapes_bf16(dmuon_lib, seed):
    shapes = _shapes(seed, 8)
    shapes += [shapes[0]] * 2  # a group of three of one shape
    Ws, Gs, Ms = make_inputs(shapes, seed=500 + seed, m_std=1e-3)
    Os, Bn = gpu_update(dmuon_lib, Gs, Ms)
    for i, shape in enumerate(shapes):
        _, Oo = oracle_update(Gs[i], Ms[i])
        e = rel_fro(to64(Os[i]), Oo)
        assert e <= 3e-2, (shape, e)
        check_momentum(Bn[i], Gs[i], Ms[i], 0.95)


def test_random_shapes_fp32(dmuon_lib):
    shapes = _shapes(9, 6)
    Ws, Gs, Ms = make_inputs(shapes, seed=509, pdt="f32", m_std=0.02, g_std=0.02)
    Os, Bn = gpu_update(dmuon_lib, Gs, Ms)
    for i, shape in enumerate(shapes):
        _, Oo = oracle_update(Gs[i], Ms[i])
        e = rel_fro(to64(Os[i]), Oo)
        assert e <= 1e-4, (shape, e)
        check_momentum(Bn[i], Gs[i], Ms[i], 0.95)
