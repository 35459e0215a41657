"""Host-side logic of the DMuon torch.optim facade (no GPU): which
parameters take Muon and the matrix each one is viewed as."""
import pytest
import torch

from newton_schulz_normalise_b200.optim import DMuon, matrix_shape, takes_muon


def test_matrix_views():
    assert matrix_shape(torch.empty(128, 64)) == (128, 64)              # Linear weight
    assert matrix_shape(torch.empty(16, 8, 3, 3)) == (16, 72)           # Conv2d filters flattened
    assert matrix_shape(torch.empty(4, 2, 3, 5, 7)) == (4, 210)         # Conv3d
    with pytest.raises(ValueError):
        matrix_shape(torch.empty(7))


def test_default_split_by_rank():
    g = {"use_muon": None}
    assert takes_muon(g, torch.empty(10, 10))
    assert takes_muon(g, torch.empty(3, 3, 3, 3))
    assert not takes_muon(g, torch.empty(10))          # bias, norm weight
    assert not takes_muon(g, torch.empty(()))          # scalar


def test_group_override():
    assert not takes_muon({"use_muon": False}, torch.empty(1000, 64))   # embedding, output head
    assert takes_muon({"use_muon": True}, torch.empty(5, 6))
    with pytest.raises(ValueError):
        takes_muon({"use_muon": True}, torch.empty(6))


def test_param_groups_and_defaults():
    w = torch.nn.Parameter(torch.empty(8, 4))
    b = torch.nn.Parameter(torch.empty(8))
    emb = torch.nn.Parameter(torch.empty(50, 4))
    opt = DMuon([{"params": [w, b]}, {"params": [emb], "use_muon": False, "lr": 3e-4}], lr=0.02)
    g0, g1 = opt.param_groups
    assert g0["use_muon"] is None and g0["lr"] == 0.02 and g0["momentum"] == 0.95 and g0["ns_steps"] == 5
    assert g1["use_muon"] is False and g1["lr"] == 3e-4 and g1["betas"] == (0.9, 0.95)
    with pytest.raises(ValueError):
        DMuon([w], lr=-1.0)


def test_step_refuses_cpu_tensors():
    w = torch.nn.Parameter(torch.zeros(4, 4))
    w.grad = torch.zeros(4, 4)
    with pytest.raises(RuntimeError):
        DMuon([w]).step()
