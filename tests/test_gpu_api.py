"""ABI entry points around the step: the autotune cache (save / load /
clear), caller-owned scratch, the workspace size query and kernel timing."""
import numpy as np
import pytest
import torch

from parity_helpers import gpu_update, make_inputs, oracle_update, rel_fro, to64

pytestmark = pytest.mark.gpu


def test_cache_save_load_roundtrip(dmuon_lib, tmp_path):
    shapes = [(192, 640)] * 3
    _, Gs, Ms = make_inputs(shapes, seed=13)
    O1, _ = gpu_update(dmuon_lib, Gs, Ms)          # tunes this shape key
    entries = dmuon_lib.dmuon_cache_entries()
    assert any(e.startswith("192 640 bf16 5 ") for e in entries)
    path = tmp_path / "plans.txt"
    dmuon_lib.dmuon_cache_save(str(path))
    assert path.read_text().startswith("dmuon-cache 1 ")
    dmuon_lib.dmuon_cache_clear()
    assert dmuon_lib.dmuon_cache_entries() == []
    dmuon_lib.dmuon_cache_load(str(path))
    assert sorted(dmuon_lib.dmuon_cache_entries()) == sorted(entries)
    O2, _ = gpu_update(dmuon_lib, Gs, Ms)          # replays the loaded plan, no tuning
    for a, b in zip(O1, O2):
        assert torch.equal(a, b)
    bad = tmp_path / "bad.txt"
    bad.write_text("not a cache\n")
    with pytest.raises(dmuon_lib.DmuonError):
        dmuon_lib.dmuon_cache_load(str(bad))
    other = tmp_path / "other_gpu.txt"
    other.write_text(path.read_text().replace("dmuon-cache 1 ", "dmuon-cache 1 H100_", 1))
    with pytest.raises(dmuon_lib.DmuonError):
        dmuon_lib.dmuon_cache_load(str(other))


def test_caller_workspace(dmuon_lib):
    shapes = [(256, 768)] * 4 + [(640, 200)] * 2
    need = dmuon_lib.dmuon_workspace_size(shapes)
    buf = torch.empty(need + 4096, dtype=torch.uint8, device="cuda")
    _, Gs, Ms = make_inputs(shapes, seed=17, m_std=1e-3)
    try:
        dmuon_lib.dmuon_set_workspace(buf)
        Os, _ = gpu_update(dmuon_lib, Gs, Ms)
        for i in range(len(shapes)):
            _, Oo = oracle_update(Gs[i], Ms[i])
            assert rel_fro(to64(Os[i]), Oo) <= 3e-2
        # too small: refused before any launch, buffers untouched
        dmuon_lib.dmuon_set_workspace(buf[:1 << 16])
        Mc = [m.clone() for m in Ms]
        out = [torch.zeros(g.shape, device="cuda") for g in Gs]
        with pytest.raises(dmuon_lib.DmuonError) as e:
            dmuon_lib.dmuon_compute_update(Gs, Mc, out, 0.95)
        assert e.value.code == dmuon_lib.DMUON_ERR_OOM
        torch.cuda.synchronize()
        assert all(torch.equal(a, b) for a, b in zip(Mc, Ms))
        assert all(torch.count_nonzero(o) == 0 for o in out)
    finally:
        dmuon_lib.dmuon_set_workspace(None)


def test_timing_and_launch_count(dmuon_lib):
    shapes = [(512, 512)] * 4
    Ws, Gs, Ms = make_inputs(shapes, seed=19)
    W = [w.clone() for w in Ws]
    dmuon_lib.dmuon_step(W, Gs, [m.clone() for m in Ms], 0.02, 0.1, 0.95)  # plan first
    torch.cuda.synchronize()
    dmuon_lib.dmuon_timing_reset()
    dmuon_lib.dmuon_timing_enable(True)
    n0 = dmuon_lib.dmuon_launch_count()
    dmuon_lib.dmuon_step(W, Gs, [m.clone() for m in Ms], 0.02, 0.1, 0.95)
    torch.cuda.synchronize()
    dmuon_lib.dmuon_timing_enable(False)
    launched = dmuon_lib.dmuon_launch_count() - n0
    kinds = [dmuon_lib.dmuon_timing_get(k) for k in range(4)]
    dmuon_lib.dmuon_timing_reset()
    assert launched == sum(k["launches"] for k in kinds) > 0
    assert kinds[1]["launches"] == 1 and kinds[1]["bytes"] == 512 * 512 * 4 * 12
    assert all(k["ms"] >= 0 for k in kinds)
    assert kinds[0]["flops"] > 0 or kinds[0]["launches"] == 0


def test_tensor_list_step_is_bit_identical(dmuon_lib):
    """A step through pre-marshalled TensorLists equals the plain-list step,
    on two steps in a row (the marshalled arrays are reused)."""
    shapes = [(64, 256)] * 4 + [(320, 200)] * 2
    Ws, Gs, Ms = make_inputs(shapes, seed=71, m_std=1e-3)
    W1, M1 = [w.clone() for w in Ws], [m.clone() for m in Ms]
    W2, M2 = [w.clone() for w in Ws], [m.clone() for m in Ms]
    tW, tG, tM = dmuon_lib.TensorList(W2), dmuon_lib.TensorList(Gs), dmuon_lib.TensorList(M2)
    for _ in range(2):
        dmuon_lib.dmuon_step(W1, Gs, M1, 0.02, 0.1, 0.95, 5)
        dmuon_lib.dmuon_step(tW, tG, tM, 0.02, 0.1, 0.95, 5)
    torch.cuda.synchronize()
    for a, b in zip(W1 + M1, W2 + M2):
        assert torch.equal(a, b)
