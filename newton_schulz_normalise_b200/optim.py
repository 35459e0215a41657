"""torch.optim facade over the library: Muon for the matrix parameters,
AdamW for the rest, in one optimizer.

"DeepSpeed 現已支援 Muon Optimizer" (setupai.cc), section 技術深入: Muon
orthogonalises the update of 2-D weights and of convolution filters once
they are flattened; training pairs it with AdamW for the parameters that are
not matrices (embeddings, biases, the final classification layer); RMS
matching lets both share AdamW's learning rate and weight decay.  The DMuon
announcement (m.zaocj.com) adds that it drops into training with three lines
of code:

    from newton_schulz_normalise_b200.optim import DMuon
    opt = DMuon(model.parameters(), lr=0.02, weight_decay=0.1)
    ...; loss.backward(); opt.step()

Which parameters take Muon: those with two or more dimensions, viewed as
(shape[0], product of the rest) -- a Linear weight as it is, a Conv2d filter
bank (out, in, kh, kw) as out x (in*kh*kw).  A parameter group may set
``use_muon=False`` (embeddings, the output head) or ``use_muon=True``.  All
arithmetic runs in the library's kernels: ``dmuon_step_ex`` once per group
and dtype, ``dmuon_adamw_step`` once per group, dtype and step count.
Parameters and gradients must be CUDA tensors, contiguous, both bf16 or both
fp32; optimizer state is fp32.
"""
from __future__ import annotations

import torch

from . import binding as B

_CODES = {torch.bfloat16: B.DMUON_BF16, torch.float32: B.DMUON_F32}


def matrix_shape(p: torch.Tensor):
    """The (rows, cols) Muon sees for a parameter with two or more dims."""
    if p.dim() < 2:
        raise ValueError(f"a Muon parameter needs at least 2 dims, got shape {tuple(p.shape)}")
    rows = p.shape[0]
    return rows, p.numel() // rows if rows else 0


def takes_muon(group: dict, p: torch.Tensor) -> bool:
    """Muon for p in this group: the group's ``use_muon`` if set, else p.dim() >= 2."""
    flag = group.get("use_muon")
    if flag is None:
        return p.dim() >= 2
    if flag and p.dim() < 2:
        raise ValueError(f"use_muon=True on a parameter of shape {tuple(p.shape)}")
    return bool(flag)


class DMuon(torch.optim.Optimizer):
    """Muon (momentum, Newton-Schulz orthogonalisation, RMS-matched scale,
    decoupled decay) on matrix parameters and AdamW on the others.

    Args: lr, weight_decay (shared by both, as RMS matching allows),
    momentum (Muon's mu), ns_steps, nesterov, betas and eps (AdamW).
    """

    def __init__(self, params, lr=0.02, weight_decay=0.1, momentum=0.95, ns_steps=5, nesterov=True,
                 betas=(0.9, 0.95), eps=1e-8):
        if lr < 0 or weight_decay < 0:
            raise ValueError("lr and weight_decay must be >= 0")
        defaults = dict(lr=lr, weight_decay=weight_decay, momentum=momentum, ns_steps=ns_steps,
                        nesterov=nesterov, betas=tuple(betas), eps=eps, use_muon=None)
        super().__init__(params, defaults)

    @torch.no_grad()
    def step(self, closure=None):
        loss = None
        if closure is not None:
            with torch.enable_grad():
                loss = closure()
        for group in self.param_groups:
            muon = {}   # dtype -> (params, grads, momenta) as 2-D views
            adamw = {}  # (dtype, step) -> (params, grads, exp_avg, exp_avg_sq)
            for p in group["params"]:
                g = p.grad
                if g is None:
                    continue
                if not p.is_cuda:
                    raise RuntimeError("DMuon runs on CUDA tensors only")
                if g.dtype != p.dtype or p.dtype not in _CODES:
                    raise TypeError(f"params and grads must both be bf16 or both fp32 (got {p.dtype}, {g.dtype})")
                if not p.is_contiguous() or not g.is_contiguous():
                    raise ValueError("DMuon needs contiguous parameters and gradients")
                state = self.state[p]
                if takes_muon(group, p):
                    shape = matrix_shape(p)
                    if "momentum_buffer" not in state:
                        state["momentum_buffer"] = torch.zeros(shape, device=p.device, dtype=torch.float32)
                    lists = muon.setdefault(p.dtype, ([], [], []))
                    lists[0].append(p.view(shape))
                    lists[1].append(g.view(shape))
                    lists[2].append(state["momentum_buffer"])
                else:
                    if "step" not in state:
                        state["step"] = 0
                        state["exp_avg"] = torch.zeros(p.shape, device=p.device, dtype=torch.float32)
                        state["exp_avg_sq"] = torch.zeros(p.shape, device=p.device, dtype=torch.float32)
                    state["step"] += 1
                    lists = adamw.setdefault((p.dtype, state["step"]), ([], [], [], []))
                    lists[0].append(p)
                    lists[1].append(g)
                    lists[2].append(state["exp_avg"])
                    lists[3].append(state["exp_avg_sq"])
            lr, wd = group["lr"], group["weight_decay"]
            for dtype, (P, G, M) in muon.items():
                code = _CODES[dtype]
                opts = B.options(code, code, nesterov=group["nesterov"])
                B.dmuon_step_ex(P, G, M, lr, wd, group["momentum"], group["ns_steps"], opts=opts)
            b1, b2 = group["betas"]
            for (dtype, t), (P, G, M, V) in adamw.items():
                B.dmuon_adamw_step(P, G, M, V, lr, b1, b2, group["eps"], wd, t)
        return loss
