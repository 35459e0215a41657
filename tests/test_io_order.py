"""The order in which a step issues its chunks (host logic, no GPU):
group by group, or for a host-I/O call with every plan cached, chunks of a
compute-bound and a copy-bound group merged and the first and last chunks'
quarters split off.  Checked through dmuon_debug_io_order, the same function
the library's step runs."""
import random

import pytest

MB = 1 << 20


def covers_every_matrix_once(groups, pieces):
    seen = {g: [] for g in range(len(groups))}
    for g, first, cnt in pieces:
        assert cnt >= 1
        seen[g].extend(range(first, first + cnt))
    for g, (count, *_rest) in enumerate(groups):
        assert sorted(seen[g]) == list(range(count)), g


def test_uncached_call_runs_group_by_group(dmuon_lib):
    groups = [(5, 2, 1.0, 8 * MB, 0), (3, 3, 0.1, 1 * MB, 0)]
    assert dmuon_lib.dmuon_debug_io_order(groups, cached=False) == [(0, 0, 2), (0, 2, 2), (0, 4, 1), (1, 0, 3)]


def test_all_copy_bound_keeps_group_order_and_splits_the_ends(dmuon_lib):
    # 16 MB chunks move in 0.32 ms at the nominal 50 GB/s; both groups compute for less
    groups = [(8, 1, 0.1, 16 * MB, 0), (64, 32, 0.06, 0.5 * MB, 0)]
    pieces = dmuon_lib.dmuon_debug_io_order(groups, cached=True)
    covers_every_matrix_once(groups, pieces)
    assert [p[0] for p in pieces] == [0] * 8 + [1] * 3  # group order; 32 + 24 + 8
    assert pieces[-2:] == [(1, 32, 24), (1, 56, 8)]     # the last chunk's quarter runs alone


def test_compute_and_copy_bound_groups_are_merged(dmuon_lib):
    # a square direct group (1.3 ms per 33.5 MB matrix: compute-bound) beside
    # a wide Gram group (1.6 ms per 117 MB matrix: copy-bound)
    groups = [(6, 1, 1.6, 117 * MB, 0), (3, 1, 1.3, 33.5 * MB, 0)]
    pieces = dmuon_lib.dmuon_debug_io_order(groups, cached=True)
    covers_every_matrix_once(groups, pieces)
    order = [p[0] for p in pieces]
    assert order == [0, 1, 0, 0, 1, 0, 0, 1, 0]  # group 1's chunks at 1/6, 1/2, 5/6 of the call
    # single-matrix chunks cannot be split
    assert all(p[2] == 1 for p in pieces)


def test_sm_copied_groups_follow_the_merged_chunks(dmuon_lib):
    groups = [(4, 1, 1.6, 117 * MB, 0), (2, 1, 1.3, 33.5 * MB, 0), (512, 512, 0.05, 32 * 1024, 1)]
    pieces = dmuon_lib.dmuon_debug_io_order(groups, cached=True)
    covers_every_matrix_once(groups, pieces)
    assert [p[0] for p in pieces[:6]] == [0, 1, 0, 0, 1, 0]
    assert pieces[6:] == [(2, 0, 384), (2, 384, 128)]  # after the merge, its last quarter split off


def test_single_chunk_call_splits_both_ends(dmuon_lib):
    groups = [(16, 16, 0.2, 2 * MB, 0)]
    assert dmuon_lib.dmuon_debug_io_order(groups, cached=True) == [(0, 0, 3), (0, 3, 9), (0, 12, 4)]
    assert dmuon_lib.dmuon_debug_io_order([(1, 4, 0.2, 2 * MB, 0)], cached=True) == [(0, 0, 1)]


def test_random_descriptions_cover_every_matrix_once(dmuon_lib):
    rng = random.Random(7)
    for _ in range(200):
        groups = [(rng.randint(1, 40), rng.randint(1, 12), rng.uniform(0.01, 3.0), rng.uniform(1e4, 2e8),
                   rng.random() < 0.2) for _ in range(rng.randint(1, 5))]
        for cached in (False, True):
            pieces = dmuon_lib.dmuon_debug_io_order(groups, cached=cached)
            covers_every_matrix_once(groups, pieces)
            for g, first, cnt in pieces:
                assert cnt <= groups[g][1]  # no piece exceeds its group's chunk (its scratch)


def test_bad_descriptions_are_rejected(dmuon_lib):
    with pytest.raises(dmuon_lib.DmuonError):
        dmuon_lib.dmuon_debug_io_order([(4, 0, 1.0, 1.0, 0)], cached=True)
    with pytest.raises(dmuon_lib.DmuonError):
        dmuon_lib.dmuon_debug_io_order([(4, 2, float("nan"), 1.0, 0)], cached=True)
    assert dmuon_lib.dmuon_debug_io_order([], cached=True) == []
