"""The tile plan that a dense mask defines.

Oracle (test infrastructure only).  The plan restates BinFlash's preprocessing
(BinFlash, "Efficiently Dispatching FlashAttention For Partially Filled Attention
Masks"): the (N, N) bool mask is reduced to a coarse (N/BM x N/BN) block mask with
three tile classes -- all-True ("full"), mixed ("partial") and all-False
("empty") -- with the partial tiles' bits packed 32 to a word, and each row of
query tiles gets its non-empty key tiles as a sorted list.

Readings fixed here (the pages leave them open):

* tiles are BM = BN = 128; a tile on the ragged edge is classified over its
  in-range (query, key) pairs only;
* fine-mask encoding: per partial tile, BM rows of BN/32 uint32 words, row-major;
  bit ``b`` of word ``w`` of row ``r`` is the mask at (row ``r``, column
  ``32 w + b``) of the tile, least significant bit first; out-of-range bits are 0;
* the key-tile list of a row is ascending;
* the work order of rows is longest-first: a stable sort on (-count, row index),
  count = number of non-empty tiles of the row;
* work pairs: inside each group, query tiles (2i, 2i+1) form one pair (the last
  tile alone when the group has an odd number); pairs are listed group by group,
  stored as their first row (bit-inverted, ~row, for a single-row pair), and
  ordered longest-first by the pair's total listed tiles, ties by pair index;
* a plan over several groups (batches, sequences, or BSR head groups) is the
  concatenation of the groups' rows in group order.

Classes: 0 = empty, 1 = partial, 2 = full.
"""

from __future__ import annotations

import numpy as np

EMPTY, PARTIAL, FULL = 0, 1, 2


def tile_classes(M, BM=128, BN=128):
    """Class of every (query tile, key tile) of a (Sq, Sk) bool mask."""
    M = np.asarray(M, dtype=bool)
    Sq, Sk = M.shape
    nqt, nkt = -(-Sq // BM), -(-Sk // BN)
    cls = np.zeros((nqt, nkt), dtype=np.uint8)
    for qt in range(nqt):
        q0, q1 = qt * BM, min(Sq, (qt + 1) * BM)
        band = M[q0:q1]
        # pad columns to whole tiles; padded positions are out of range and False
        padded = np.zeros((q1 - q0, nkt * BN), dtype=bool)
        padded[:, :Sk] = band
        cnt = padded.reshape(q1 - q0, nkt, BN).sum(axis=(0, 2))
        ncols = np.minimum(BN, Sk - np.arange(nkt) * BN)
        in_range = (q1 - q0) * ncols
        cls[qt] = np.where(cnt == 0, EMPTY, np.where(cnt == in_range, FULL, PARTIAL))
    return cls


def pack_tile(M, qt, kt, BM=128, BN=128):
    """Fine mask words (BM, BN // 32) uint32 of one tile, LSB-first, zero outside."""
    M = np.asarray(M, dtype=bool)
    Sq, Sk = M.shape
    t = np.zeros((BM, BN), dtype=bool)
    q0, k0 = qt * BM, kt * BN
    blk = M[q0:min(Sq, q0 + BM), k0:min(Sk, k0 + BN)]
    t[:blk.shape[0], :blk.shape[1]] = blk
    by = np.packbits(t, axis=1, bitorder="little")          # (BM, BN/8) bytes
    return by.view("<u4").astype(np.uint32).reshape(BM, BN // 32)


def plan_group(M, BM=128, BN=128):
    """Plan of one group's (Sq, Sk) mask: classes, per-row CSR, packed partial tiles."""
    cls = tile_classes(M, BM, BN)
    row_lists, row_part, fine = [], [], []
    for qt in range(cls.shape[0]):
        kts = np.nonzero(cls[qt] != EMPTY)[0]
        row_lists.append(kts.astype(np.int32))
        part = (cls[qt, kts] == PARTIAL).astype(np.uint8)
        row_part.append(part)
        for kt, p in zip(kts, part):
            if p:
                fine.append(pack_tile(M, qt, int(kt), BM, BN))
    return cls, row_lists, row_part, fine


def lpt_order(counts):
    """Row order: stable sort on (-count, row index)."""
    counts = np.asarray(counts, dtype=np.int64)
    return np.array(sorted(range(len(counts)), key=lambda r: (-counts[r], r)), dtype=np.int32)


def plan_masks(masks, BM=128, BN=128):
    """Plan of a sequence of group masks (each (Sq_g, Sk_g) bool), groups in order."""
    return combine_groups([plan_group(M, BM, BN) for M in masks], BM, BN)


def combine_groups(group_plans, BM=128, BN=128):
    """The plan of several groups from each group's own plan (``plan_group``), in
    group order: the groups' rows concatenated, then the row order and the work
    pairs over all rows.  Lets a caller build a large plan one group's mask at a
    time."""
    cls_all, lists, parts, fines = [], [], [], []
    for cls, rl, rp, fn in group_plans:
        cls_all.append(cls)
        lists += rl
        parts += rp
        fines += fn
    counts = np.array([len(x) for x in lists], dtype=np.int32)
    pair_row, pair_cost = [], []
    r0 = 0
    for cls in cls_all:
        nqt = cls.shape[0]
        for i in range(0, nqt, 2):
            two = i + 1 < nqt
            pair_row.append(r0 + i if two else ~(r0 + i))
            pair_cost.append(int(counts[r0 + i]) + (int(counts[r0 + i + 1]) if two else 0))
        r0 += nqt
    row_ptr = np.zeros(len(lists) + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum(counts)
    kv_tile = np.concatenate(lists).astype(np.int32) if lists else np.zeros(0, np.int32)
    partial = np.concatenate(parts).astype(np.uint8) if parts else np.zeros(0, np.uint8)
    fine = (np.stack(fines).astype(np.uint32) if fines
            else np.zeros((0, BM, BN // 32), dtype=np.uint32))
    return {
        "cls": cls_all,
        "row_ptr": row_ptr,
        "kv_tile": kv_tile,
        "partial": partial,
        "fine": fine,
        "counts": counts,
        "order": lpt_order(counts),
        "pair_row": np.array(pair_row, dtype=np.int32),
        "pair_order": lpt_order(pair_cost),
    }


def transpose_plan(cls_groups):
    """Key-tile columns of a plan: the work lists of the backward's key-tile pass.

    BinFlash (its backward runs dK/dV over key blocks and dQ over query blocks,
    from the same gathered block lists): the dK/dV pass visits, for every key
    tile, the query tiles whose tile is not empty.  Column c enumerates the
    groups in order and, inside a group, the key tiles ascending; its list holds
    the query tiles qt with class(qt, kt) != empty, ascending, with a partial flag;
    columns are ordered longest first, ties by column index (the row order's rule).
    """
    q_tile, partial, counts, col_group, col_kt = [], [], [], [], []
    for g, cls in enumerate(cls_groups):
        nqt, nkt = cls.shape
        for kt in range(nkt):
            qs = [qt for qt in range(nqt) if cls[qt, kt] != EMPTY]
            q_tile += qs
            partial += [1 if cls[qt, kt] == PARTIAL else 0 for qt in qs]
            counts.append(len(qs))
            col_group.append(g)
            col_kt.append(kt)
    counts = np.array(counts, dtype=np.int32)
    col_ptr = np.zeros(len(counts) + 1, dtype=np.int32)
    col_ptr[1:] = np.cumsum(counts)
    return {
        "col_ptr": col_ptr,
        "q_tile": np.array(q_tile, dtype=np.int32),
        "partial": np.array(partial, dtype=np.uint8),
        "counts": counts,
        "order": lpt_order(counts),
        "col_group": np.array(col_group, dtype=np.int32),
        "col_kt": np.array(col_kt, dtype=np.int32),
    }


def expand_plan(plan, shapes, BM=128, BN=128):
    """Inverse check: rebuild every group's dense mask from a plan.

    Full tiles become all-True over their in-range pairs, partial tiles take the
    unpacked fine bits, tiles absent from a row's list are all-False.  ``shapes``
    is the list of (Sq, Sk) per group.
    """
    out = []
    r = 0
    pidx = 0
    for (Sq, Sk) in shapes:
        M = np.zeros((Sq, Sk), dtype=bool)
        nqt = -(-Sq // BM)
        for qt in range(nqt):
            for e in range(plan["row_ptr"][r], plan["row_ptr"][r + 1]):
                kt = int(plan["kv_tile"][e])
                q0, q1 = qt * BM, min(Sq, (qt + 1) * BM)
                k0, k1 = kt * BN, min(Sk, (kt + 1) * BN)
                if plan["partial"][e]:
                    words = plan["fine"][pidx]
                    pidx += 1
                    bits = np.unpackbits(words.astype("<u4").view(np.uint8).reshape(BM, -1),
                                         axis=1, bitorder="little").astype(bool)
                    M[q0:q1, k0:k1] = bits[:q1 - q0, :k1 - k0]
                else:
                    M[q0:q1, k0:k1] = True
            r += 1
        out.append(M)
    return out


def plan_stats(plan):
    """(n_full, n_partial, n_empty) over all groups' tile grids."""
    n_full = sum(int((c == FULL).sum()) for c in plan["cls"])
    n_part = sum(int((c == PARTIAL).sum()) for c in plan["cls"])
    n_empty = sum(int((c == EMPTY).sum()) for c in plan["cls"])
    return n_full, n_part, n_empty
