"""dmuon_compute_update_noalloc: the entry point for callers that cannot
allocate device memory in their step (a framework allocator that owns all of
device memory, or a loop that cannot take cudaMalloc's implicit device
synchronisation).  Its scratch is the library's fixed static array.

Checked through the C ABI against the regular dmuon_compute_update, on two
calls in a row (the static array keeps the previous call's contents), within
the parity tolerances of the other tests.  Collected last on purpose.
"""
import numpy as np
import pytest
import torch

from parity_helpers import check_momentum, gpu_update, make_inputs, rel_fro, to64

pytestmark = pytest.mark.gpu


def _noalloc(binding, G, M, mu=0.95, steps=5):
    Mc = M.clone()
    O = torch.full(G.shape, float("nan"), device=G.device, dtype=torch.float32)
    binding.dmuon_compute_update_noalloc(G.clone(), Mc, O, mu, steps)
    torch.cuda.synchronize()
    return O, Mc


def test_noalloc_matches_compute_update_twice(dmuon_lib):
    # two calls in a row on different shapes: a wide bf16 matrix, then a tall one
    for seed, shape in ((101, (512, 1024)), (102, (300, 130))):
        _, Gs, Ms = make_inputs([shape], seed=seed, m_std=1e-3)
        O_ref, B_ref = gpu_update(dmuon_lib, Gs, Ms)
        O_new, B_new = _noalloc(dmuon_lib, Gs[0], Ms[0])
        assert torch.isfinite(O_new).all()
        assert rel_fro(to64(O_new), to64(O_ref[0])) <= 3e-2, shape
        check_momentum(B_new, Gs[0], Ms[0], 0.95)
        assert np.array_equal(to64(B_new), to64(B_ref[0]))


def test_noalloc_fp32_twice(dmuon_lib):
    for seed in (103, 104):
        _, Gs, Ms = make_inputs([(256, 512)], seed=seed, pdt="f32", m_std=0.02, g_std=0.02)
        O_ref, _ = gpu_update(dmuon_lib, Gs, Ms)
        O_new, B_new = _noalloc(dmuon_lib, Gs[0], Ms[0])
        assert rel_fro(to64(O_new), to64(O_ref[0])) <= 1e-4
        check_momentum(B_new, Gs[0], Ms[0], 0.95)


def test_noalloc_rejects_oversize_before_launch(dmuon_lib):
    G = torch.zeros(4096, 4096, device="cuda", dtype=torch.bfloat16)
    M = torch.zeros(4096, 4096, device="cuda", dtype=torch.float32)
    O = torch.zeros(4096, 4096, device="cuda", dtype=torch.float32)
    with pytest.raises(dmuon_lib.DmuonError) as e:
        dmuon_lib.dmuon_compute_update_noalloc(G, M, O, 0.95)
    assert e.value.code == dmuon_lib.DMUON_ERR_INVALID
    assert "scratch" in str(e.value)
    torch.cuda.synchronize()
    assert torch.count_nonzero(M) == 0 and torch.count_nonzero(O) == 0
