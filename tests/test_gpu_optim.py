"""The DMuon torch.optim facade on CUDA: each step equals the library calls
it stands for, bit for bit (Muon through dmuon_step_ex on the 2-D views,
convolution filters flattened; AdamW through dmuon_adamw_step), and the
Muon update of a flattened conv filter matches the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle.muon_oracle as ora
from newton_schulz_normalise_b200.optim import DMuon
from parity_helpers import rel_fro, to64

pytestmark = pytest.mark.gpu


class Net(torch.nn.Module):
    def __init__(self):
        super().__init__()
        self.emb = torch.nn.Embedding(100, 64)
        self.conv = torch.nn.Conv2d(8, 16, 3)            # filters 16 x 8 x 3 x 3 -> 16 x 72
        self.fc = torch.nn.Linear(64, 128)
        self.norm = torch.nn.LayerNorm(128)
        self.head = torch.nn.Linear(128, 100, bias=False)


def _model(dtype, seed):
    torch.manual_seed(seed)
    net = Net().to("cuda", dtype)
    gen = torch.Generator(device="cuda").manual_seed(seed + 1)
    for p in net.parameters():
        p.grad = (torch.randn(p.shape, device="cuda", generator=gen) * 1e-3).to(dtype)
    return net


def _groups(net):
    return [{"params": [net.conv.weight, net.conv.bias, net.fc.weight, net.fc.bias, net.norm.weight, net.norm.bias]},
            {"params": [net.emb.weight, net.head.weight], "use_muon": False}]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_facade_equals_library_calls(dmuon_lib, dtype):
    net = _model(dtype, 3)
    ref = _model(dtype, 3)
    opt = DMuon(_groups(net), lr=0.02, weight_decay=0.1)
    code = dmuon_lib.DMUON_BF16 if dtype == torch.bfloat16 else dmuon_lib.DMUON_F32
    muon_p = [ref.conv.weight, ref.fc.weight]
    adam_p = [ref.conv.bias, ref.fc.bias, ref.norm.weight, ref.norm.bias]
    head_p = [ref.emb.weight, ref.head.weight]
    mom = [torch.zeros(p.shape[0], p.numel() // p.shape[0], device="cuda") for p in muon_p]
    st = {id(p): (torch.zeros(p.shape, device="cuda"), torch.zeros(p.shape, device="cuda")) for p in adam_p + head_p}
    for t in (1, 2):
        opt.step()
        with torch.no_grad():
            dmuon_lib.dmuon_step_ex([p.view(p.shape[0], -1) for p in muon_p],
                                    [p.grad.view(p.shape[0], -1) for p in muon_p], mom, 0.02, 0.1, 0.95, 5,
                                    opts=dmuon_lib.options(code, code))
            for ps in (adam_p, head_p):
                dmuon_lib.dmuon_adamw_step(ps, [p.grad for p in ps], [st[id(p)][0] for p in ps],
                                           [st[id(p)][1] for p in ps], 0.02, 0.9, 0.95, 1e-8, 0.1, t)
        torch.cuda.synchronize()
        for (n1, a), (n2, b) in zip(net.named_parameters(), ref.named_parameters()):
            assert torch.equal(a, b), (n1, t)
    assert opt.state[net.conv.weight]["momentum_buffer"].shape == (16, 72)
    assert opt.state[net.head.weight]["step"] == 2


def test_flattened_conv_update_matches_oracle(dmuon_lib):
    """One Muon step on a conv filter bank through the facade, against the
    oracle's step on the flattened matrix."""
    torch.manual_seed(7)
    conv = torch.nn.Conv2d(32, 64, 3).to("cuda", torch.bfloat16)        # 64 x 288
    W0 = conv.weight.detach().clone()
    gen = torch.Generator(device="cuda").manual_seed(8)
    conv.weight.grad = (torch.randn(conv.weight.shape, device="cuda", generator=gen) * 1e-3).bfloat16()
    conv.bias.grad = None
    DMuon([conv.weight], lr=0.02, weight_decay=0.1).step()
    torch.cuda.synchronize()
    G = to64(conv.weight.grad.view(64, -1))
    W = to64(W0.view(64, -1))
    W_ora, _, _ = ora.muon_step(W, G, np.zeros_like(G), 0.02, 0.1, 0.95, 5)
    dW_gpu = to64(conv.weight.view(64, -1)) - W
    dW_ora = W_ora - W
    assert rel_fro(dW_gpu, dW_ora) <= 6e-2   # bf16 update (3e-2) seen through bf16 rounding of W
