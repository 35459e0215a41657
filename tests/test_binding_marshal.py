"""Host-side marshalling of the Python binding (no GPU): a TensorList gives
the C ABI the same pointer and shape arrays as the plain list it wraps."""
import ctypes

import pytest
import torch

from newton_schulz_normalise_b200 import binding as B


def _arr(a, n):
    return [a[i] for i in range(n)]


def test_tensor_list_matches_plain_list():
    ts = [torch.empty(r, c, dtype=torch.bfloat16) for r, c in [(64, 256), (3, 5), (1024, 7)]]
    tl = B.TensorList(ts)
    assert len(tl) == 3 and tl[1] is ts[1] and list(tl) == ts
    assert _arr(B._ptrs(tl), 3) == _arr(B._ptrs(ts), 3) == [t.data_ptr() for t in ts]
    assert _arr(B._shapes(tl), 6) == _arr(B._shapes(ts), 6) == [64, 256, 3, 5, 1024, 7]
    assert tl.dtype == B.DMUON_BF16
    assert B.TensorList([torch.empty(2, 2)]).dtype == B.DMUON_F32


def test_marshalling_rejects_non_matrices():
    tl = B.TensorList([torch.empty(4, 4), torch.empty(2, 3, 4)])   # fine for AdamW (any rank) ...
    assert tl.shapes is None and len(tl) == 2
    with pytest.raises(ValueError):                                 # ... but not as Muon matrices
        B._shapes(tl)
    with pytest.raises(ValueError):
        B._shapes([torch.empty(8, 8).t()[:, :4]])


def test_empty_list():
    tl = B.TensorList([])
    assert len(tl) == 0 and tl.dtype == B.DMUON_BF16
    assert isinstance(B._ptrs([]), ctypes.Array)
