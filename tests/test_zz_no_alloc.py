"""The dense planner that allocates nothing, called through the C ABI.

Some callers cannot let a library allocate device memory -- a serving process
whose memory manager has reserved the whole GPU up front, or code that must keep
a fixed device-memory footprint.  ``bfa_plan_dense_noalloc`` computes the same
plan as ``bfa_plan_dense`` into buffers the caller owns, using a scratch array
that lives inside the library.  This test calls it twice in a row (two different
masks, so the shared scratch is reused) and compares each result with the plan of
the allocating entry point, bit for bit.  It runs last so that a failure here
never hides the rest of the suite.
"""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

bfa = pytest.importorskip("mask_skipping_flashattention_b200")

TILE = 128
MAX_ROWS, MAX_KV_TILES = 4096, 16384  # BFA_NOALLOC_MAX_ROWS, BFA_NOALLOC_MAX_KV_TILES in include/bfa.h


def _noalloc_plan(mask):
    """Call the C entry point with caller-owned torch buffers; return host copies."""
    lib = bfa._L
    Sq, Sk = mask.shape
    nqt, nkt = -(-Sq // TILE), -(-Sk // TILE)
    dev = mask.device
    classes = torch.full((nqt * nkt,), 255, dtype=torch.uint8, device=dev)
    row_ptr = torch.full((nqt + 1,), -7, dtype=torch.int32, device=dev)
    kv_tile = torch.full((nqt * nkt,), -7, dtype=torch.int32, device=dev)
    part = torch.full((nqt * nkt,), -7, dtype=torch.int32, device=dev)
    fine = torch.zeros((nqt * nkt, TILE, 4), dtype=torch.int32, device=dev)
    order = torch.full((nqt,), -7, dtype=torch.int32, device=dev)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = lib.bfa_plan_dense_noalloc(P(mask), mask.stride(0), Sq, Sk, P(classes), P(row_ptr), P(kv_tile), P(part),
                                    P(fine), P(order), st)
    assert rc == 0, lib.bfa_last_error().decode()
    torch.cuda.synchronize()
    rp = row_ptr.cpu().numpy()
    nnz = int(rp[-1])
    prt = part.cpu().numpy()[:nnz]
    fine_h = fine.cpu().numpy().view(np.uint32)
    partial = (prt >= 0).astype(np.uint8)
    fine_list = fine_h[prt[prt >= 0]] if (prt >= 0).any() else np.zeros((0, TILE, 4), np.uint32)
    return dict(classes=classes.cpu().numpy(), row_ptr=rp, kv_tile=kv_tile.cpu().numpy()[:nnz], partial=partial,
                fine=fine_list, order=order.cpu().numpy())


def _masks():
    rng = np.random.default_rng(2024)
    a = rng.random((1000, 1300)) < 0.05
    a[:128, :128] = True
    a[128:256] = False
    a[300:700, 200:900] |= np.tril(np.ones((400, 700), bool))
    b = np.tril(np.ones((8192, 8192), dtype=bool))
    return [a, b]


def test_noalloc_matches_allocating_planner_twice():
    for M in _masks():
        m = torch.from_numpy(M).cuda()
        got = _noalloc_plan(m)
        ref = bfa.plan_dense(m).export()
        for key in ("classes", "row_ptr", "kv_tile", "partial", "fine", "order"):
            np.testing.assert_array_equal(got[key], ref[key], err_msg=f"{key} differs for {M.shape}")


def test_noalloc_rejects_sizes_beyond_its_limit():
    """One tile past either limit is refused before anything is launched (the
    dummy buffers are never touched)."""
    lib = bfa._L
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    P = ctypes.c_void_p(dummy.data_ptr())
    too_many_rows = (MAX_ROWS + 1) * TILE
    rc = lib.bfa_plan_dense_noalloc(P, 1, too_many_rows, 1, P, P, P, P, P, P, None)
    assert bfa._lib.STATUS[rc] == "BFA_ERR_CAPACITY"
    assert "limit" in lib.bfa_last_error().decode()
    too_many_keys = (MAX_KV_TILES + 1) * TILE
    rc = lib.bfa_plan_dense_noalloc(P, too_many_keys, 1, too_many_keys, P, P, P, P, P, P, None)
    assert bfa._lib.STATUS[rc] == "BFA_ERR_CAPACITY"
    assert "limit" in lib.bfa_last_error().decode()


def test_noalloc_accepts_exactly_the_largest_query_tile_count():
    """Sq = 4096 query tiles (the limit itself) is planned, and equals the
    allocating planner's plan."""
    Sq, Sk = MAX_ROWS * TILE, 40
    rng = np.random.default_rng(7)
    M = rng.random((Sq, Sk)) < 0.3
    M[:TILE] = True
    M[TILE:2 * TILE] = False
    M[-1, :] = True
    m = torch.from_numpy(M).cuda()
    got = _noalloc_plan(m)
    ref = bfa.plan_dense(m).export()
    for key in ("classes", "row_ptr", "kv_tile", "partial", "fine", "order"):
        np.testing.assert_array_equal(got[key], ref[key], err_msg=f"{key} differs at the query-tile limit")


def test_noalloc_leaves_free_device_memory_unchanged():
    """After a first call (which looks up the scratch array and loads the planner
    kernels), further calls do not change the device's free memory."""
    lib = bfa._L
    Sq, Sk = 2000, 3000
    m = torch.from_numpy(np.tril(np.ones((Sq, Sk), dtype=bool))).cuda()
    nqt, nkt = -(-Sq // TILE), -(-Sk // TILE)
    bufs = [torch.empty(nqt * nkt, dtype=torch.uint8, device="cuda"),
            torch.empty(nqt + 1, dtype=torch.int32, device="cuda"),
            torch.empty(nqt * nkt, dtype=torch.int32, device="cuda"),
            torch.empty(nqt * nkt, dtype=torch.int32, device="cuda"),
            torch.empty(nqt * nkt * TILE * 4, dtype=torch.int32, device="cuda"),
            torch.empty(nqt, dtype=torch.int32, device="cuda")]
    args = [ctypes.c_void_p(t.data_ptr()) for t in bufs]
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        rc = lib.bfa_plan_dense_noalloc(ctypes.c_void_p(m.data_ptr()), Sk, Sq, Sk, *args, st)
        assert rc == 0, lib.bfa_last_error().decode()

    call()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
