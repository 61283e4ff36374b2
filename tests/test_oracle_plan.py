"""Pins for the oracle's tile plan (CPU only).

The plan is recounted tile by tile and bit by bit with Python loops on small
ragged masks, inverted back into the mask it came from, and checked against the
closed-form tile counts of the causal and BSR workloads.
"""

import numpy as np
import pytest

from oracle import masks as om
from oracle import plan as op


def _brute_plan(M, BM, BN):
    Sq, Sk = M.shape
    nqt, nkt = -(-Sq // BM), -(-Sk // BN)
    cls = np.zeros((nqt, nkt), dtype=np.uint8)
    fine = {}
    for qt in range(nqt):
        for kt in range(nkt):
            n_in, n_on = 0, 0
            words = np.zeros((BM, BN // 32), dtype=np.uint64)
            for r in range(BM):
                for c in range(BN):
                    i, j = qt * BM + r, kt * BN + c
                    if i < Sq and j < Sk:
                        n_in += 1
                        if M[i, j]:
                            n_on += 1
                            words[r, c // 32] |= np.uint64(1) << np.uint64(c % 32)
            cls[qt, kt] = 0 if n_on == 0 else (2 if n_on == n_in else 1)
            if cls[qt, kt] == 1:
                fine[(qt, kt)] = words.astype(np.uint32)
    return cls, fine


@pytest.mark.parametrize("shape,BM,BN,density", [
    ((70, 90), 32, 32, 0.5),
    ((64, 64), 32, 32, 0.97),
    ((33, 130), 32, 64, 0.2),
    ((300, 200), 128, 128, 0.0005),
])
def test_plan_matches_brute_force(shape, BM, BN, density):
    rng = np.random.default_rng(sum(shape))
    M = rng.random(shape) < density
    # plant an all-True and an all-False in-range tile so every class occurs
    M[:BM, :BN] = True
    M[BM:2 * BM, :BN] = False
    cls_ref, fine_ref = _brute_plan(M, BM, BN)
    P = op.plan_masks([M], BM, BN)
    np.testing.assert_array_equal(P["cls"][0], cls_ref)
    e = 0
    p = 0
    for qt in range(cls_ref.shape[0]):
        kts = [kt for kt in range(cls_ref.shape[1]) if cls_ref[qt, kt] != 0]
        assert list(P["kv_tile"][P["row_ptr"][qt]:P["row_ptr"][qt + 1]]) == kts
        for kt in kts:
            assert P["partial"][e] == (cls_ref[qt, kt] == 1)
            if cls_ref[qt, kt] == 1:
                np.testing.assert_array_equal(P["fine"][p], fine_ref[(qt, kt)])
                p += 1
            e += 1
    assert p == P["fine"].shape[0] == len(fine_ref)


@pytest.mark.parametrize("seed", range(4))
def test_expand_plan_reproduces_mask(seed):
    rng = np.random.default_rng(100 + seed)
    shapes = [(int(rng.integers(1, 400)), int(rng.integers(1, 400))) for _ in range(3)]
    masks = []
    for (a, b) in shapes:
        M = rng.random((a, b)) < rng.choice([0.001, 0.3, 0.999])
        M[: a // 3] = rng.random((a // 3, b)) < 0.5
        masks.append(M)
    P = op.plan_masks(masks)
    for M, R in zip(masks, op.expand_plan(P, shapes)):
        np.testing.assert_array_equal(M, R)


def test_lpt_order_properties():
    rng = np.random.default_rng(1)
    counts = rng.integers(0, 6, size=200)
    order = op.lpt_order(counts)
    assert sorted(order.tolist()) == list(range(200))          # a permutation
    c = counts[order]
    assert np.all(np.diff(c) <= 0)                             # longest first
    for a, b in zip(order[:-1], order[1:]):
        if counts[a] == counts[b]:
            assert a < b                                       # stable ties


def test_causal_8192_tile_counts_closed_form():
    N, T = 8192, 128
    M = om.positional_dense(N, N, causal=True)
    cls = op.tile_classes(M)
    n = N // T
    assert int((cls == 2).sum()) == n * (n - 1) // 2 == 2016
    assert int((cls == 1).sum()) == n == 64
    assert int((cls == 0).sum()) == n * (n - 1) // 2
    assert np.all(np.diag(cls) == 1)
    assert int(M.sum()) == N * (N + 1) // 2 == 33558528


def test_bsr_workload_tile_counts_closed_form():
    from workloads import bsr_routing
    nb, T = 128, 128
    indptr, indices = bsr_routing(1, 1, nb, 1234)
    M = om.bsr_dense(indptr, indices, nb * T, nb * T, T, T, causal=True)[0, 0]
    cls = op.tile_classes(M)
    assert int((cls == 2).sum()) == sum(i // 4 for i in range(nb)) == 1984
    assert int((cls == 1).sum()) == nb
    assert int(M.sum()) == 1984 * T * T + nb * T * (T + 1) // 2 == 33562624


def test_block_ids_tail_tile_classes():
    """Ragged tail: a tile is classified over its in-range pairs only."""
    M = np.ones((130, 129), dtype=bool)
    cls = op.tile_classes(M)
    assert cls.shape == (2, 2) and np.all(cls == 2)
    M[129, 128] = False
    assert op.tile_classes(M)[1, 1] == 1
    w = op.pack_tile(M, 1, 1)
    assert w.shape == (128, 4)
    assert w[0, 0] == 1 and w[1, 0] == 0 and np.all(w[2:] == 0) and np.all(w[:, 1:] == 0)


def test_plan_stats_cover_grid():
    rng = np.random.default_rng(2)
    masks = [rng.random((257, 300)) < 0.01, np.zeros((10, 10), bool)]
    P = op.plan_masks(masks)
    assert sum(op.plan_stats(P)) == 3 * 3 + 1
    assert P["counts"][-1] == 0 and P["row_ptr"][-1] == P["kv_tile"].size


@pytest.mark.parametrize("seed", [0, 1])
def test_transposed_plan_lists_the_same_tiles_as_the_rows(seed):
    rng = np.random.default_rng(seed)
    masks = [rng.random((300, 420)) < 0.002, np.tril(np.ones((260, 260), dtype=bool)), rng.random((129, 77)) < 0.5]
    plan = op.plan_masks(masks)
    tp = op.transpose_plan(plan["cls"])
    # brute force: column c of group g lists every query tile holding an attended pair of key tile kt
    c = 0
    r0 = 0
    rows_pairs, cols_pairs = set(), set()
    for g, M in enumerate(masks):
        nqt, nkt = -(-M.shape[0] // 128), -(-M.shape[1] // 128)
        for kt in range(nkt):
            want = [qt for qt in range(nqt) if M[qt * 128:(qt + 1) * 128, kt * 128:(kt + 1) * 128].any()]
            got = tp["q_tile"][tp["col_ptr"][c]:tp["col_ptr"][c + 1]].tolist()
            assert got == want and tp["col_group"][c] == g and tp["col_kt"][c] == kt
            for e, qt in enumerate(got):
                blk = M[qt * 128:(qt + 1) * 128, kt * 128:(kt + 1) * 128]
                assert tp["partial"][tp["col_ptr"][c] + e] == (0 if blk.all() else 1)
                cols_pairs.add((g, qt, kt))
            c += 1
        for qt in range(nqt):
            for e in range(plan["row_ptr"][r0 + qt], plan["row_ptr"][r0 + qt + 1]):
                rows_pairs.add((g, qt, int(plan["kv_tile"][e])))
        r0 += nqt
    assert rows_pairs == cols_pairs
    assert np.array_equal(tp["order"], np.lexsort((np.arange(len(tp["counts"])), -tp["counts"])))


def _brute_pairs(masks, BM=128, BN=128):
    """Work pairs recomputed from the masks with plain loops: inside each group,
    query tiles (2i, 2i + 1) form a pair, the last tile of an odd group stands
    alone (stored as ~row); a pair costs the non-empty key tiles of its rows; the
    order is longest first, ties by pair index (insertion sort, stable)."""
    pair_row, cost = [], []
    r0 = 0
    for M in masks:
        Sq, Sk = M.shape
        nqt, nkt = -(-Sq // BM), -(-Sk // BN)
        counts = []
        for qt in range(nqt):
            n = 0
            for kt in range(nkt):
                if M[qt * BM:(qt + 1) * BM, kt * BN:(kt + 1) * BN].any():
                    n += 1
            counts.append(n)
        i = 0
        while i < nqt:
            if i + 1 < nqt:
                pair_row.append(r0 + i)
                cost.append(counts[i] + counts[i + 1])
            else:
                pair_row.append(-(r0 + i) - 1)
                cost.append(counts[i])
            i += 2
        r0 += nqt
    order = []
    for p in range(len(cost)):
        pos = len(order)
        while pos > 0 and cost[order[pos - 1]] < cost[p]:
            pos -= 1
        order.insert(pos, p)
    return pair_row, order


@pytest.mark.parametrize("seed", range(3))
def test_work_pairs_match_brute_force(seed):
    rng = np.random.default_rng(300 + seed)
    masks = [
        rng.random((5 * 128 + 17, 700)) < 0.004,        # odd tile count with a ragged last tile
        np.tril(np.ones((128, 128), dtype=bool)),       # a group of one tile
        np.zeros((0, 256), dtype=bool),                 # an empty group (no query tiles)
        np.zeros((300, 260), dtype=bool),               # rows with nothing listed
        rng.random((4 * 128, 3 * 128 + 5)) < 0.5,       # even tile count
        np.tril(np.ones((3 * 128 - 1, 3 * 128 - 1), dtype=bool)),
    ]
    masks[3][200, 5] = True                            # one attended pair in the middle row
    P = op.plan_masks(masks)
    pair_row, order = _brute_pairs(masks)
    np.testing.assert_array_equal(P["pair_row"], np.array(pair_row, dtype=np.int32))
    np.testing.assert_array_equal(P["pair_order"], np.array(order, dtype=np.int32))
    # the pairs cover every row exactly once, in group order
    rows = []
    for pr in pair_row:
        rows += [pr, pr + 1] if pr >= 0 else [~pr]
    r0, want = 0, []
    for M in masks:
        nqt = -(-M.shape[0] // 128)
        want += list(range(r0, r0 + nqt))
        r0 += nqt
    assert rows == want


def test_work_pairs_of_the_causal_grid_closed_form():
    """Causal 8192: pair i holds tiles 2i, 2i + 1 with 2i + 1 + 2i + 2 listed tiles,
    so the longest-first order is the pairs in reverse."""
    n = 64
    M = np.tril(np.ones((n * 128, n * 128), dtype=bool))
    P = op.plan_masks([M])
    assert P["counts"].tolist() == list(range(1, n + 1))
    assert P["pair_row"].tolist() == list(range(0, n, 2))
    assert P["pair_order"].tolist() == list(range(n // 2 - 1, -1, -1))
