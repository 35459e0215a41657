"""Failure detection on the GPU without a fault: a wait that nothing
completes gives up after a short limit, the kernel reports it through the
host-visible error word and returns, and the context stays usable.
Allocation failures are injected on the host."""
import os
import subprocess
import sys
from pathlib import Path

import pytest
import torch

from parity_helpers import gpu_update, make_inputs, oracle_update, rel_fro, to64

pytestmark = pytest.mark.gpu
ROOT = Path(__file__).resolve().parent.parent


def test_bounded_wait_times_out_and_context_survives(dmuon_lib):
    rc = dmuon_lib.dmuon_selftest_wait(50)
    assert rc == dmuon_lib.DMUON_ERR_DEVICE_TIMEOUT, dmuon_lib.last_error()
    assert "gave up" in dmuon_lib.last_error()
    # the next calls run normally
    Ws, Gs, Ms = make_inputs([(96, 200)], seed=5)
    Os, _ = gpu_update(dmuon_lib, Gs, Ms)
    _, Oo = oracle_update(Gs[0], Ms[0])
    assert rel_fro(to64(Os[0]), Oo) <= 3e-2
    assert dmuon_lib.dmuon_selftest_wait(20) == dmuon_lib.DMUON_ERR_DEVICE_TIMEOUT


def test_selftest_argument_check(dmuon_lib):
    assert dmuon_lib.dmuon_selftest_wait(0) == dmuon_lib.DMUON_ERR_INVALID


def test_injected_allocation_failure_leaves_buffers_untouched():
    """DMUON_FAULT=alloc: the scratch allocation fails, the call returns
    DMUON_ERR_OOM before any launch, the caller's buffers are unchanged.
    (A fresh process: the library allocates its scratch once.)"""
    code = r'''
import sys, torch
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
from newton_schulz_normalise_b200 import binding as B
from parity_helpers import make_inputs
Ws, Gs, Ms = make_inputs([(128, 256)] * 2, seed=3, m_std=1e-3)
W0 = [w.clone() for w in Ws]; M0 = [m.clone() for m in Ms]
rc = B.lib.dmuon_step(B._ptrs(Ws), B._ptrs(Gs), B._ptrs(Ms), B._shapes(Ws), 2, 0.02, 0.1, 0.95, 5, None)
torch.cuda.synchronize()
assert rc == B.DMUON_ERR_OOM, (rc, B.last_error())
assert all(torch.equal(a, b) for a, b in zip(Ws, W0)) and all(torch.equal(a, b) for a, b in zip(Ms, M0))
print("ok", B.last_error())
'''
    env = dict(os.environ, DMUON_FAULT="alloc")
    r = subprocess.run([sys.executable, "-c", code, str(ROOT)], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "injected" in r.stdout
