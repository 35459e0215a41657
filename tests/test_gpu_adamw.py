"""dmuon_adamw_step (the non-matrix parameters beside Muon) against the fp64
AdamW oracle, step by step, through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import adamw_oracle as ora
from parity_helpers import to64

pytestmark = pytest.mark.gpu

SIZES = [1, 3, 4, 5, 4096, 4097, 16387, 70000, (64, 33), (2048,), (7, 5, 3)]
HYPER = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)


def _tensors(dtype, seed, sizes=SIZES):
    g = torch.Generator(device="cuda").manual_seed(seed)
    shape = [s if isinstance(s, tuple) else (s,) for s in sizes]
    P = [(torch.randn(s, device="cuda", generator=g) * 0.02).to(dtype) for s in shape]
    return P, shape, g


def _bf16_ulp(x):
    a = np.abs(x)
    a = np.where(a > 0, a, 1e-30)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_adamw_matches_oracle_over_steps(dmuon_lib, dtype):
    P, shapes, gen = _tensors(dtype, 91)
    M = [torch.zeros(s, device="cuda") for s in shapes]
    V = [torch.zeros(s, device="cuda") for s in shapes]
    h = HYPER
    for step in range(1, 4):
        G = [(torch.randn(s, device="cuda", generator=gen) * 1e-3).to(dtype) for s in shapes]
        p0 = [to64(p) for p in P]
        m0 = [to64(m) for m in M]
        v0 = [to64(v) for v in V]
        dmuon_lib.dmuon_adamw_step(P, G, M, V, h["lr"], h["beta1"], h["beta2"], h["eps"], h["wd"], step)
        torch.cuda.synchronize()
        for i in range(len(P)):
            g = to64(G[i])
            pw, mw, vw = ora.adamw_step(p0[i], g, m0[i], v0[i], h["lr"], h["beta1"], h["beta2"], h["eps"], h["wd"], step)
            # fp32 moments: a few ulps of the terms that form them
            mb = 1e-6 * (h["beta1"] * np.abs(m0[i]) + (1 - h["beta1"]) * np.abs(g)) + 1e-30
            vb = 1e-6 * (h["beta2"] * np.abs(v0[i]) + (1 - h["beta2"]) * g * g) + 1e-38
            assert np.all(np.abs(to64(M[i]) - mw) <= mb), (i, step)
            assert np.all(np.abs(to64(V[i]) - vw) <= vb), (i, step)
            # the step's size taken from the magnitudes of the terms that form m
            # (m itself can cancel), over the same denominator
            vhat = vw / (1 - h["beta2"] ** step)
            terms = (h["beta1"] * np.abs(m0[i]) + (1 - h["beta1"]) * np.abs(g)) / (1 - h["beta1"] ** step)
            step_mag = h["lr"] * terms / (np.sqrt(vhat) + h["eps"])
            got = to64(P[i])
            if dtype == torch.float32:  # four roundings at |p| (decay, product, step product, difference)
                bound = 4 * 2.0 ** -23 * np.abs(p0[i]) + step_mag * 1e-5 + 1e-30
            else:  # one rounding to bf16 of an fp32 result that is itself within 1e-5 of exact
                bound = _bf16_ulp(pw) + step_mag * 1e-5
            assert np.all(np.abs(got - pw) <= bound), (i, step, float(np.max(np.abs(got - pw) / bound)))


def test_adamw_unaligned_equals_aligned(dmuon_lib):
    """Buffers off a 16-byte boundary take the element-by-element path; it
    performs the same arithmetic, so the results are bit-identical."""
    n = 5003
    gen = torch.Generator(device="cuda").manual_seed(5)
    data = [torch.randn(n, device="cuda", generator=gen) * s for s in (0.02, 1e-3, 1e-4, 1e-6)]
    data[3] = data[3].abs()

    def run(offset):
        views = []
        for d in data:
            buf = torch.zeros(n + offset, device="cuda")
            buf[offset:] = d
            views.append(buf[offset:])
        assert all(v.data_ptr() % 16 == (4 * offset) % 16 for v in views)
        P, G, M, V = views
        for step in (1, 2):
            dmuon_lib.dmuon_adamw_step([P], [G], [M], [V], 1e-3, 0.9, 0.99, 1e-8, 0.05, step)
        torch.cuda.synchronize()
        return P.clone(), M.clone(), V.clone()

    a = run(0)
    b = run(1)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_adamw_empty_and_zero_size(dmuon_lib):
    dmuon_lib.dmuon_adamw_step([], [], [], [], 1e-3, 0.9, 0.95, 1e-8, 0.0, 1)
    e = torch.empty(0, device="cuda")
    p = torch.ones(10, device="cuda")
    g = torch.ones(10, device="cuda")
    m = torch.zeros(10, device="cuda")
    v = torch.zeros(10, device="cuda")
    dmuon_lib.dmuon_adamw_step([e, p], [e, g], [e, m], [e, v], 0.5, 0.9, 0.95, 0.0, 0.0, 1)
    torch.cuda.synchronize()
    assert torch.allclose(p, torch.full_like(p, 0.5))  # first step moves by lr * sign(g)


def test_adamw_rejects_bad_arguments(dmuon_lib):
    p = [torch.zeros(4, device="cuda")]
    for kw in (dict(step=0), dict(beta1=1.0), dict(beta2=-0.1), dict(eps=-1.0), dict(lr=float("nan"))):
        args = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.0, step=1)
        args.update(kw)
        with pytest.raises(dmuon_lib.DmuonError):
            dmuon_lib.dmuon_adamw_step(p, p, p, p, args["lr"], args["beta1"], args["beta2"], args["eps"],
                                       args["wd"], args["step"])
