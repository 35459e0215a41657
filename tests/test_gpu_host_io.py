"""dmuon_step_host_io: gradients from pinned host memory, updated parameters
copied back to host, copies pipelined with the computation.  Checked against
dmuon_step on the same inputs and against the oracle."""
import os
import subprocess
import sys
import textwrap
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle.muon_oracle as ora
from parity_helpers import check_momentum, gpu_step, make_inputs, to64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shapes", [[(1024, 1024)] * 20, [(256, 1024)] * 70 + [(1024, 256)] * 3, [(300, 130)]],
                         ids=["1024sq-x20", "mixed-x73", "tall-x1"])
def test_host_io_matches_device_step(dmuon_lib, shapes):
    lr, wd, mu = 0.02, 0.1, 0.95
    Ws, Gs, Ms = make_inputs(shapes, seed=77, m_std=1e-3)
    W_ref, M_ref = gpu_step(dmuon_lib, Ws, Gs, Ms, lr, wd, mu)
    hG = [g.cpu().pin_memory() for g in Gs]
    hW = [torch.full(w.shape, float("nan"), dtype=w.dtype).pin_memory() for w in Ws]
    for _ in range(2):  # second call runs with cached plans
        W = [w.clone() for w in Ws]
        M = [m.clone() for m in Ms]
        dmuon_lib.dmuon_step_host_io(W, hG, M, lr, wd, mu, 5, params_host_out=hW)
        torch.cuda.synchronize()
        for i, (r, c) in enumerate(shapes):
            assert torch.equal(hW[i], W[i].cpu()), i           # the copy-out is the device result
            assert torch.equal(M[i], M_ref[i]), i               # same momentum arithmetic
            # same update up to the plan the autotuner chose for the chunking
            d = np.linalg.norm(to64(W[i]) - to64(W_ref[i]))
            # two updates each within 3e-2 of the oracle; ||O||_F is about sqrt(min(r, c))
            bound = lr * ora.rms_scale(r, c) * 6e-2 * np.sqrt(min(r, c)) + 2 ** -8 * np.linalg.norm(to64(W_ref[i]))
            assert d <= bound, (i, d, bound)
    check_momentum(M[0], Gs[0], Ms[0], mu)


def test_host_io_without_copy_out(dmuon_lib):
    shapes = [(512, 512)] * 3
    Ws, Gs, Ms = make_inputs(shapes, seed=78)
    W_ref, _ = gpu_step(dmuon_lib, Ws, Gs, Ms)
    W = [w.clone() for w in Ws]
    M = [m.clone() for m in Ms]
    dmuon_lib.dmuon_step_host_io(W, [g.cpu().pin_memory() for g in Gs], M, 0.02, 0.1, 0.95, 5)
    torch.cuda.synchronize()
    for a, b in zip(W, W_ref):
        assert (a.float() - b.float()).abs().max().item() <= 2 ** -7 * b.float().abs().max().item()


def test_host_io_pageable_and_unaligned_buffers(dmuon_lib):
    """Host buffers the copy kernel cannot take (pageable memory, a pinned
    buffer at a 2-byte offset) go through copy-engine transfers; the result
    is the same as with pinned, aligned buffers."""
    shapes = [(256, 512)] * 4 + [(128, 384)] * 3
    lr, wd, mu = 0.02, 0.1, 0.95
    Ws, Gs, Ms = make_inputs(shapes, seed=79, m_std=1e-3)

    def run(hG, hW):
        W = [w.clone() for w in Ws]
        M = [m.clone() for m in Ms]
        for _ in range(2):
            dmuon_lib.dmuon_step_host_io(W, hG, M, lr, wd, mu, 5, params_host_out=hW)
        torch.cuda.synchronize()
        return W, M

    pinned = run([g.cpu().pin_memory() for g in Gs], [torch.empty(w.shape, dtype=w.dtype).pin_memory() for w in Ws])

    def offset_pinned(t):  # pinned storage, data pointer 2 bytes past a 16-byte boundary
        big = torch.empty(t.numel() + 8, dtype=t.dtype).pin_memory()
        v = big[1:1 + t.numel()].view(t.shape)
        v.copy_(t)
        return v

    hG_mixed = [g.cpu() for g in Gs[:4]] + [offset_pinned(g.cpu()) for g in Gs[4:]]
    hW_mixed = [torch.empty(w.shape, dtype=w.dtype) for w in Ws[:4]] + [offset_pinned(w.cpu()) for w in Ws[4:]]
    assert all(h.data_ptr() % 16 == 2 for h in hG_mixed[4:])
    mixed = run(hG_mixed, hW_mixed)
    for a, b in zip(pinned[0] + pinned[1], mixed[0] + mixed[1]):
        assert torch.equal(a, b)
    for i in range(len(shapes)):
        assert torch.equal(hW_mixed[i], mixed[0][i].cpu()), i


def test_host_io_merged_chunks_match_group_order(dmuon_lib):
    """Once every plan is cached, a host-I/O call whose groups include a
    compute-bound one (4096^2, direct form: 1.4 TFLOP per 33.5 MB) and a
    copy-bound one (1024 x 4096, Gram form) issues their chunks interleaved
    instead of group by group.  The first call, which tunes and runs group by
    group, and the second, merged, run the same plans on the same chunks:
    same bits."""
    shapes = [(4096, 4096)] * 3 + [(1024, 4096)] * 4 + [(4096, 1024)] + [(512, 512)] * 3 + [(300, 130)] * 2
    lr, wd, mu = 0.02, 0.1, 0.95
    Ws, Gs, Ms = make_inputs(shapes, seed=80, m_std=1e-3)
    W_ref, M_ref = gpu_step(dmuon_lib, Ws, Gs, Ms, lr, wd, mu)
    hG = [g.cpu().pin_memory() for g in Gs]
    runs = []
    for _ in range(2):
        W = [w.clone() for w in Ws]
        M = [m.clone() for m in Ms]
        hW = [torch.full(w.shape, float("nan"), dtype=w.dtype).pin_memory() for w in Ws]
        dmuon_lib.dmuon_step_host_io(W, hG, M, lr, wd, mu, 5, params_host_out=hW)
        torch.cuda.synchronize()
        for i in range(len(shapes)):
            assert torch.equal(hW[i], W[i].cpu()), i
            assert torch.equal(M[i], M_ref[i]), i
        runs.append(W)
    for i, (r, c) in enumerate(shapes):
        assert torch.equal(runs[0][i], runs[1][i]), i
        d = np.linalg.norm(to64(runs[1][i]) - to64(W_ref[i]))
        bound = lr * ora.rms_scale(r, c) * 6e-2 * np.sqrt(min(r, c)) + 2 ** -8 * np.linalg.norm(to64(W_ref[i]))
        assert d <= bound, (i, d, bound)


@pytest.mark.parametrize("shapes,merged", [
    ([(4096, 4096)] * 3 + [(1024, 4096)] * 4, True),      # compute-bound square group beside a copy-bound one
    ([(1024, 4096)] * 4 + [(256, 1024)] * 64, False),     # every group copy-bound: group order stays
], ids=["mixed", "all-copy-bound"])
def test_host_io_merge_decision(shapes, merged):
    """The chunks of a host-I/O call are merged across shape groups only when
    one group is compute-bound and another copy-bound (checked through the
    library's trace in a fresh process, after a first call that tunes)."""
    script = f"""
        import sys
        sys.path[:0] = ["tests", "."]
        import torch
        from newton_schulz_normalise_b200 import binding as B
        from parity_helpers import make_inputs
        shapes = {shapes!r}
        Ws, Gs, Ms = make_inputs(shapes, seed=81, m_std=1e-3)
        hG = [g.cpu().pin_memory() for g in Gs]
        hW = [torch.empty(w.shape, dtype=w.dtype).pin_memory() for w in Ws]
        for i in range(2):
            print("CALL", i, file=sys.stderr, flush=True)
            B.dmuon_step_host_io(Ws, hG, Ms, 0.02, 0.1, 0.95, 5, params_host_out=hW)
            torch.cuda.synchronize()
    """
    env = dict(os.environ, DMUON_TRACE="1")
    r = subprocess.run([sys.executable, "-c", textwrap.dedent(script)], capture_output=True, text=True, timeout=300,
                       cwd=Path(__file__).resolve().parents[1], env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    second = r.stderr.split("CALL 1")[-1]
    assert "CALL 0" in r.stderr and "chunks merged" not in r.stderr.split("CALL 1")[0]  # the first call tunes
    assert ("chunks merged" in second) == merged, second[-2000:]


def test_host_io_few_row_groups_iterate_in_fp32(dmuon_lib):
    """Host I/O with bf16 weights whose iterate has at most 5 rows (fp32
    iterate) beside ordinary bf16 groups: the fp32 groups meet the fp32 bar,
    the others the bf16 one, and the copied-out parameters are the device's."""
    shapes = [(5, 700)] * 6 + [(1024, 3)] * 2 + [(6, 512)] * 4 + [(512, 1024)] * 3
    Ws, Gs, Ms = make_inputs(shapes, seed=82, m_std=1e-3)
    hG = [g.cpu().pin_memory() for g in Gs]
    for call in range(2):  # the second call runs with cached plans (pieces, merge decision)
        W = [w.clone() for w in Ws]
        M = [m.clone() for m in Ms]
        hW = [torch.empty(w.shape, dtype=w.dtype).pin_memory() for w in Ws]
        dmuon_lib.dmuon_step_host_io(W, hG, M, 0.02, 0.1, 0.95, 5, params_host_out=hW)
        torch.cuda.synchronize()
        for i, (r, c) in enumerate(shapes):
            assert torch.equal(hW[i], W[i].cpu()), (call, i)
            _, Oo = ora.muon_update(to64(Gs[i]), to64(Ms[i]), 0.95, 5, 1e-7, True, "direct")
            w_apply = ora.apply_update(to64(Ws[i]), Oo, 0.02, 0.1)
            tol = 1e-4 if min(r, c) <= 5 else 3e-2
            # the update's error budget plus one bf16 rounding of W'
            budget = 0.02 * ora.rms_scale(r, c) * tol * np.linalg.norm(Oo) + 2 ** -8 * np.linalg.norm(w_apply)
            d = np.linalg.norm(to64(W[i]) - w_apply)
            assert d <= budget, (call, i, d, budget)
