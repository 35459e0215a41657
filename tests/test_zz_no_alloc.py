"""dmuon_compute_update_noalloc: the entry point for callers that cannot
allocate device memory in their step (a framework allocator that owns all of
device memory, or a loop that cannot take cudaMalloc's implicit device
synchronisation).  Its scratch is the library's fixed static array.

Checked through the C ABI, on two calls in a row (the static array keeps the
previous call's contents):
* against the fp64 oracle at the parity bar of the other tests (3e-2 bf16,
  1e-4 fp32), and bit for bit against dmuon_compute_update, which runs the
  same plan;
* in fresh processes: with every library allocation made to fail
  (DMUON_FAULT=alloc) it still runs, matches the oracle and leaves the
  device's free memory unchanged; a bounded device wait that runs out in one
  call (DMUON_FAULT=wait) is reported by the next call, which launches
  nothing, and the call after that runs again.
Collected last on purpose.
"""
import json
import os
import subprocess
import sys
import textwrap
from pathlib import Path

import pytest
import torch

from parity_helpers import check_momentum, gpu_update, make_inputs, oracle_update, rel_fro, to64

pytestmark = pytest.mark.gpu
ROOT = Path(__file__).resolve().parents[1]


def _noalloc(binding, G, M, mu=0.95, steps=5, **kw):
    Mc = M.clone()
    O = torch.full(G.shape, float("nan"), device=G.device, dtype=torch.float32)
    binding.dmuon_compute_update_noalloc(G.clone(), Mc, O, mu, steps, **kw)
    torch.cuda.synchronize()
    return O, Mc


@pytest.mark.parametrize("pdt,tol,cases", [
    ("bf16", 3e-2, ((101, (512, 1024)), (102, (300, 130)))),
    ("f32", 1e-4, ((103, (256, 512)), (104, (130, 70)))),
])
def test_noalloc_matches_oracle_and_compute_update_twice(dmuon_lib, pdt, tol, cases):
    for seed, shape in cases:
        std = 0.02 if pdt == "f32" else 1e-3
        _, Gs, Ms = make_inputs([shape], seed=seed, pdt=pdt, m_std=std, g_std=std)
        O_ref, B_ref = gpu_update(dmuon_lib, Gs, Ms)  # tunes and caches the plan for this shape
        _, O_ora = oracle_update(Gs[0], Ms[0])
        for _ in range(2):  # two calls in a row on the same static array
            O_new, B_new = _noalloc(dmuon_lib, Gs[0], Ms[0])
            assert rel_fro(to64(O_new), O_ora) <= tol, (shape, rel_fro(to64(O_new), O_ora))
            check_momentum(B_new, Gs[0], Ms[0], 0.95)
            assert torch.equal(O_new, O_ref[0]), shape  # same plan: same kernels, same result
            assert torch.equal(B_new, B_ref[0])


@pytest.mark.parametrize("shape", [(64, 256), (256, 1024), (1024, 256)], ids=["small", "medium", "medium-tall"])
def test_noalloc_forced_resident_kernel(dmuon_lib, shape):
    """A forced resident plan: the small-matrix kernel (64 x 256) and the
    medium one (one CTA pair, Gram form; wide and tall storage)."""
    _, Gs, Ms = make_inputs([shape], seed=105, m_std=1e-3)
    O_ref, _ = gpu_update(dmuon_lib, Gs, Ms, variant="batched")
    _, O_ora = oracle_update(Gs[0], Ms[0])
    for _ in range(2):
        O_new, B_new = _noalloc(dmuon_lib, Gs[0], Ms[0], variant="batched")
        assert rel_fro(to64(O_new), O_ora) <= 3e-2
        assert torch.equal(O_new, O_ref[0])
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


def _fresh(script, fault):
    env = dict(os.environ, DMUON_FAULT=fault)
    r = subprocess.run([sys.executable, "-c", textwrap.dedent(script)], capture_output=True, text=True,
                       timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    return json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1])


_PRELUDE = """
    import json, sys
    sys.path[:0] = ["tests", "."]
    import numpy as np, torch
    from newton_schulz_normalise_b200 import binding as B
    from parity_helpers import make_inputs, oracle_update, rel_fro, to64
    _, Gs, Ms = make_inputs([(384, 640)], seed=106, m_std=1e-3)
    G, M = Gs[0], Ms[0]
    _, O_ora = oracle_update(G, M)
    def call():
        Mc = M.clone()
        O = torch.full(G.shape, float("nan"), device="cuda", dtype=torch.float32)
        torch.cuda.synchronize()
        try:
            B.dmuon_compute_update_noalloc(G, Mc, O, 0.95, 5)
            rc = 0
        except B.DmuonError as e:
            rc = e.code
        torch.cuda.synchronize()
        return rc, O, Mc
"""


def test_noalloc_allocates_nothing_fresh_process(dmuon_lib):
    out = _fresh(_PRELUDE + """
    rc0, O0, _ = call()              # first call: looks up the array's address
    Mc = M.clone()                   # buffers of the measured call, made before it
    O1 = torch.full(G.shape, float("nan"), device="cuda", dtype=torch.float32)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    B.dmuon_compute_update_noalloc(G, Mc, O1, 0.95, 5)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    # the regular entry point fails under the injected allocation failure
    try:
        B.dmuon_compute_update([G], [M.clone()], [torch.empty(G.shape, device="cuda")], 0.95, 5)
        reg = 0
    except B.DmuonError as e:
        reg = e.code
    print(json.dumps({"rc": rc0, "err": [rel_fro(to64(O0), O_ora), rel_fro(to64(O1), O_ora)],
                      "same": bool(torch.equal(O0, O1)), "free": [free0, free1], "regular": reg}))
    """, "alloc")
    assert out["rc"] == 0
    assert max(out["err"]) <= 3e-2 and out["same"]
    assert out["free"][0] == out["free"][1], out["free"]
    assert out["regular"] == -4  # DMUON_ERR_OOM: the regular path's scratch allocation was refused


def test_noalloc_reports_device_timeout_at_next_call(dmuon_lib):
    out = _fresh(_PRELUDE + """
    rc1, O1, _ = call()   # runs, then the injected bounded wait gives up on the device
    rc2, O2, M2 = call()  # reads the error word: reports, clears, launches nothing
    rc3, O3, _ = call()   # runs again
    print(json.dumps({"rc": [rc1, rc2, rc3], "err1": rel_fro(to64(O1), O_ora), "err3": rel_fro(to64(O3), O_ora),
                      "untouched": bool(torch.isnan(O2).all()) and bool(torch.equal(M2, M))}))
    """, "wait")
    assert out["rc"] == [0, -5, 0], out
    assert out["untouched"]
    assert out["err1"] <= 3e-2 and out["err3"] <= 3e-2
