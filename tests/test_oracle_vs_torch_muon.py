"""Secondary cross-check of the oracle's conventions against an independent
implementation, torch.optim.Muon, on the CPU (no GPU).

torch.optim.Muon keeps its momentum in the lerp form b <- mu b + (1 - mu) g
and steps along (1 - mu) g + mu b (Nesterov).  From zero momentum that is
(1 - mu) times the oracle's buffer B' = mu B + G and direction U = G + mu B'
at every step, and the Frobenius normalisation removes the factor: with
adjust_lr_fn="match_rms_adamw" (scale 0.2 sqrt(max(rows, cols))) and the same
decoupled decay, both must give the same weights step after step.  torch runs
its Newton-Schulz in bf16, so the updates agree to about 1e-2; a different
scale, orientation, decay order or momentum form would be off by O(1).
This is not the oracle and nothing of it is used by the library."""
import numpy as np
import pytest
import torch

import oracle.muon_oracle as ora

Muon = getattr(torch.optim, "Muon", None)
pytestmark = pytest.mark.skipif(Muon is None, reason="torch.optim.Muon not available")


@pytest.mark.parametrize("shape", [(64, 256), (256, 64), (128, 128), (96, 200)])
def test_oracle_matches_torch_muon_over_steps(shape):
    r, c = shape
    gen = torch.Generator().manual_seed(r * 7 + c)
    lr, wd, mu = 0.02, 0.1, 0.95
    W = torch.nn.Parameter(torch.randn(r, c, generator=gen) * 0.02)
    opt = Muon([W], lr=lr, weight_decay=wd, momentum=mu, nesterov=True, adjust_lr_fn="match_rms_adamw")
    W_ora = W.detach().double().numpy().copy()
    B_ora = np.zeros((r, c))
    A_mag = np.zeros((r, c))
    for step in range(3):
        G = torch.randn(r, c, generator=gen) * 1e-3
        W_prev = W.detach().double().numpy().copy()
        W.grad = G.clone()
        opt.step()
        # the oracle steps from torch's own previous weights, so the check is per step
        W_next, B_ora, _ = ora.muon_step(W_prev, G.double().numpy(), B_ora, lr, wd, mu, 5)
        d_torch = W.detach().double().numpy() - W_prev
        d_ora = W_next - W_prev
        assert np.linalg.norm(d_torch - d_ora) <= 3e-2 * np.linalg.norm(d_ora), (shape, step)
        # torch's fp32 buffer against (1 - mu) B' in fp64: it carries one fp32
        # rounding per step of the gradients' uncancelled magnitude
        # A = sum_k mu^(t-k) |g_k| (entries of B' itself can cancel)
        A_mag = mu * A_mag + np.abs(G.double().numpy())
        buf = opt.state[W]["momentum_buffer"].double().numpy()
        bound = 1e-6 * (step + 1) * (1 - mu) * A_mag + 1e-30
        assert np.all(np.abs(buf - (1 - mu) * B_ora) <= bound), (shape, step)
        W_ora = W_next
