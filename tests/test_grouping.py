"""Grouping of a step's matrices by iterate shape (host logic, no GPU),
checked through dmuon_debug_groups, the function the library's step runs."""
import pytest

from newton_schulz_normalise_b200 import workloads as wl


def test_llama_set_forms_three_groups(dmuon_lib):
    shapes = wl.WORKLOADS["llama8b-matrices-bf16"].shapes()
    groups = dmuon_lib.dmuon_debug_groups(shapes)
    assert [(g["m"], g["n"], g["count"], g["ntall"]) for g in groups] == [
        (4096, 4096, 64, 0),      # q, o
        (1024, 4096, 64, 64),     # k, v: stored 4096 x 1024
        (4096, 14336, 96, 32),    # gate, up and the transposed down projection share one iterate shape
    ]
    # chunks within the 8 GiB scratch budget: 31 square matrices, all 64 of
    # 1024 x 4096, 16 of 4096 x 14336
    assert [g["chunk"] for g in groups] == [31, 64, 16]
    assert not any(g["iter_f32"] for g in groups)
    # inside a group the matrices stored m x n come first, each part in order
    big = groups[2]["members"]
    assert big[:64] == sorted(i for i, (r, c) in enumerate(shapes) if (r, c) == (4096, 14336))
    assert big[64:] == sorted(i for i, (r, c) in enumerate(shapes) if (r, c) == (14336, 4096))


def test_host_io_chunks_hold_about_16_mb_of_gradients(dmuon_lib):
    shapes = wl.WORKLOADS["llama8b-matrices-bf16"].shapes()
    groups = dmuon_lib.dmuon_debug_groups(shapes, grads_host=True)
    assert [g["chunk"] for g in groups] == [1, 2, 1]  # 32 MB, 8 MB and 112 MB of bf16 gradients per matrix
    sq = dmuon_lib.dmuon_debug_groups([(1024, 1024)] * 64, grads_host=True)
    assert sq[0]["chunk"] == 8 and sq[0]["count"] == 64


def test_first_appearance_order_and_members(dmuon_lib):
    shapes = [(300, 100), (64, 256), (100, 300), (256, 64), (64, 256), (5, 5)]
    groups = dmuon_lib.dmuon_debug_groups(shapes)
    assert [(g["m"], g["n"], g["count"], g["ntall"]) for g in groups] == [(100, 300, 2, 1), (64, 256, 3, 1),
                                                                          (5, 5, 1, 0)]
    assert [g["members"] for g in groups] == [[2, 0], [1, 4, 3], [5]]


def test_few_row_iterates_are_fp32(dmuon_lib):
    groups = dmuon_lib.dmuon_debug_groups([(3, 600), (600, 3), (5, 64), (6, 600), (1, 1)])
    assert [(g["m"], g["n"], g["iter_f32"]) for g in groups] == [(3, 600, True), (5, 64, True), (6, 600, False),
                                                                 (1, 1, True)]
    assert groups[0]["ntall"] == 1
    f32 = dmuon_lib.dmuon_debug_groups([(256, 512), (64, 64)], param_dtype=dmuon_lib.DMUON_F32)
    assert all(g["iter_f32"] for g in f32)


def test_bad_shapes_are_rejected(dmuon_lib):
    with pytest.raises(dmuon_lib.DmuonError):
        dmuon_lib.dmuon_debug_groups([(4, 0)])
    with pytest.raises(dmuon_lib.DmuonError):
        dmuon_lib.dmuon_debug_groups([(4, 4)], param_dtype=7)
    assert dmuon_lib.dmuon_debug_groups([]) == []
