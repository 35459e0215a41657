"""Seeded synthetic parameter sets for the Muon step.

This module only draws random numbers: it holds none of the method's
arithmetic, so both the CUDA path's tests/benchmarks and the CPU oracle can be
fed from it.  The pages run the method on private training jobs and name no
dataset; every workload here is synthetic, shaped like the weight matrices of
the model families the step is used on.

A workload is a list of matrix groups (rows, cols, count) plus dtypes and the
distributions of the weight W, the gradient G and the momentum buffer M.
Tensors are drawn matrix by matrix, in list order, from one torch.Generator
seeded with the workload's seed; bf16 tensors are drawn in fp32 and rounded,
so the stored bf16 values are the inputs both sides see.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    # (rows, cols, count) in the order the matrices are drawn / passed
    groups: tuple
    param_dtype: str = "bf16"      # "bf16" | "f32"
    grad_dtype: str = "bf16"
    mom_dtype: str = "f32"
    w_std: float = 0.02
    g_std: float = 1e-3
    m_std: float = 0.0             # 0 => momentum starts at zero
    seed: int = 0
    lr: float = 0.02
    wd: float = 0.1
    mu: float = 0.95
    ns_steps: int = 5
    interleave: int = 1            # >1: groups repeat per layer (layer-major order)
    notes: str = ""

    def shapes(self):
        """Matrix shapes in draw order."""
        out = []
        if self.interleave > 1:
            for _ in range(self.interleave):
                for r, c, n in self.groups:
                    out.extend([(r, c)] * n)
        else:
            for r, c, n in self.groups:
                out.extend([(r, c)] * n)
        return out

    def numel(self) -> int:
        return sum(r * c for r, c in self.shapes())


_LLAMA8B_LAYER = ((4096, 4096, 1), (4096, 1024, 1), (4096, 1024, 1), (4096, 4096, 1),
                  (4096, 14336, 1), (4096, 14336, 1), (14336, 4096, 1))

WORKLOADS = {
    # one fp32 weight; grad and momentum non-zero; the fp32 accuracy case
    "single-256x512-fp32": Workload(
        "single-256x512-fp32", ((256, 512, 1),), "f32", "f32", "f32",
        w_std=0.02, g_std=0.02, m_std=0.02, seed=0),
    # 64 square bf16 weights with fp32 momentum: the uniform-shape batched path
    "batch64-1024x1024-bf16": Workload(
        "batch64-1024x1024-bf16", ((1024, 1024, 64),), seed=1),
    # 24-layer transformer, hidden 2048: Wqkv, Wo, W_up, W_down per layer
    "transformer24-h2048-bf16": Workload(
        "transformer24-h2048-bf16",
        ((2048, 6144, 1), (2048, 2048, 1), (2048, 8192, 1), (8192, 2048, 1)),
        seed=2, interleave=24),
    # skewed shapes: many tiny, some medium, a few huge wide and tall
    "skewed-shapes-bf16": Workload(
        "skewed-shapes-bf16",
        ((64, 256, 512), (256, 1024, 128), (4096, 14336, 8), (14336, 4096, 8)),
        seed=3),
    # the skewed set's tiny group on its own (the resident small-matrix kernel)
    "batch512-64x256-bf16": Workload(
        "batch512-64x256-bf16", ((64, 256, 512),), seed=3),
    # the skewed set's medium group on its own (the resident medium-matrix kernel)
    "batch128-256x1024-bf16": Workload(
        "batch128-256x1024-bf16", ((256, 1024, 128),), seed=3),
    # Llama-style 8B matrix set: 32 layers of q, k, v, o, gate, up, down
    "llama8b-matrices-bf16": Workload(
        "llama8b-matrices-bf16", _LLAMA8B_LAYER, seed=4, interleave=32),
    # one layer of that set (every shape and product of it at 1/32 of the
    # size: small enough for profiler captures, 1.75 GB > L2)
    "llama8b-layer-bf16": Workload(
        "llama8b-layer-bf16", _LLAMA8B_LAYER, seed=4, interleave=1),
}

_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def torch_dtype(name: str) -> torch.dtype:
    return _DT[name]


def generate(w: Workload, device="cpu", indices=None, shapes=None):
    """Draw (W, G, M) for every matrix of the workload (or for ``indices``).

    Draw order is fixed: for matrix i, W then G then M, each as fp32 normals
    times its std, rounded to its dtype.  Matrices not in ``indices`` are still
    drawn (and discarded) so that a subset is bit-identical to the full set.
    ``shapes`` overrides the workload's shape list (tests of odd shapes).
    """
    shapes = list(shapes) if shapes is not None else w.shapes()
    want = set(range(len(shapes))) if indices is None else set(indices)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    Ws, Gs, Ms = [], [], []
    for i, (r, c) in enumerate(shapes):
        if i > max(want, default=-1):
            break
        W = torch.randn((r, c), generator=gen, device=device, dtype=torch.float32) * w.w_std
        G = torch.randn((r, c), generator=gen, device=device, dtype=torch.float32) * w.g_std
        if w.m_std > 0:
            M = torch.randn((r, c), generator=gen, device=device, dtype=torch.float32) * w.m_std
        else:
            M = torch.zeros((r, c), device=device, dtype=torch.float32)
        if i in want:
            Ws.append(W.to(_DT[w.param_dtype]))
            Gs.append(G.to(_DT[w.grad_dtype]))
            Ms.append(M.to(_DT[w.mom_dtype]))
    return Ws, Gs, Ms


def random_matrix(rows, cols, seed, std=1.0, dtype=torch.float32, device="cpu"):
    """A single seeded N(0, std^2) matrix (odd-shape and edge-case tests)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = torch.randn((rows, cols), generator=gen, device=device, dtype=torch.float32) * std
    return x.to(dtype)
