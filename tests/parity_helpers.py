"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, and compare."""
import numpy as np
import torch

import oracle.muon_oracle as ora
from newton_schulz_normalise_b200 import workloads as wl


def to64(t):
    return t.detach().float().cpu().double().numpy()


def rel_fro(x, y):
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    n = np.linalg.norm(y)
    return np.linalg.norm(x - y) / (n if n > 0 else 1.0)


def make_inputs(shapes, seed, pdt="bf16", m_std=0.0, g_std=1e-3, device="cuda"):
    w = wl.Workload("test", tuple((r, c, 1) for r, c in shapes), pdt, pdt, "f32",
                    w_std=0.02, g_std=g_std, m_std=m_std, seed=seed)
    return wl.generate(w, device=device, shapes=shapes)


def gpu_update(binding, Gs, Ms, mu=0.95, steps=5, **opt):
    """dmuon_compute_update on clones; returns (O list fp32, B' list)."""
    Gc = [g.clone() for g in Gs]
    Mc = [m.clone() for m in Ms]
    Os = [torch.empty(g.shape, device=g.device, dtype=torch.float32) for g in Gs]
    binding.dmuon_compute_update(Gc, Mc, Os, mu, steps, **opt)
    torch.cuda.synchronize()
    return Os, Mc


def gpu_step(binding, Ws, Gs, Ms, lr=0.02, wd=0.1, mu=0.95, steps=5, **opt):
    Wc = [w.clone() for w in Ws]
    Mc = [m.clone() for m in Ms]
    binding.dmuon_step_ex(Wc, [g.clone() for g in Gs], Mc, lr, wd, mu, steps, **opt)
    torch.cuda.synchronize()
    return Wc, Mc


def oracle_update(G, M, mu=0.95, steps=5, variant="direct", nesterov=True, eps=1e-7):
    return ora.muon_update(to64(G), to64(M), mu, steps, eps, nesterov, variant)


def check_momentum(Bn_gpu, G, M, mu, tol=1e-6):
    """|B'_gpu - B'_ora| <= tol * (|mu B| + |G|) elementwise (the buffer is
    fp32; the relative bound is taken against the terms that form it)."""
    g, b = to64(G), to64(M)
    ref = mu * b + g
    err = np.abs(to64(Bn_gpu) - ref)
    bound = tol * (np.abs(mu * b) + np.abs(g)) + 1e-30
    assert np.all(err <= bound), float((err / bound).max())
