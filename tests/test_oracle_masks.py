"""Pins for the oracle's mask builders (CPU only).

Each check compares the oracle against something other than itself: per-element
brute-force loops over the rule the pages state, printed examples from the pages
(``tests/golden``), or special cases with a known answer.
"""

import os

import numpy as np
import pytest

from oracle import masks as om

INT32_MIN = np.iinfo(np.int32).min


def _brute_block_ids(pad, att, n_cross=None, cpad=None):
    """Running counter of opened blocks, written as an explicit loop."""
    B, N = att.shape
    q_blk = np.zeros((B, N), dtype=np.int64)
    for b in range(B):
        cur = 0
        for i in range(N):
            if att[b, i]:
                cur += 1
            q_blk[b, i] = cur
    if n_cross is None:
        return q_blk, q_blk.copy(), pad.copy(), pad.copy()
    k_blk = np.zeros((B, n_cross + N), dtype=np.int64)
    k_valid = np.zeros((B, n_cross + N), dtype=bool)
    for b in range(B):
        for j in range(n_cross):
            k_blk[b, j] = INT32_MIN
            k_valid[b, j] = cpad[b, j]
        for j in range(N):
            k_blk[b, n_cross + j] = q_blk[b, j]
            k_valid[b, n_cross + j] = pad[b, j]
    return q_blk, k_blk, pad.copy(), k_valid


def _brute_dense(q_blk, k_blk, q_valid, k_valid):
    B, Sq = q_blk.shape
    Sk = k_blk.shape[1]
    M = np.zeros((B, Sq, Sk), dtype=bool)
    for b in range(B):
        for i in range(Sq):
            for j in range(Sk):
                M[b, i, j] = bool(q_valid[b, i]) and bool(k_valid[b, j]) and int(k_blk[b, j]) <= int(q_blk[b, i])
    return M


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("cross", [None, 3])
def test_block_ids_match_brute_force(seed, cross):
    rng = np.random.default_rng(seed)
    B, N = 2, 13
    att = (rng.random((B, N)) < 0.3).astype(np.uint8)
    if seed % 2:
        att[:, 0] = 1
    pad = rng.random((B, N)) < 0.8
    cpad = None if cross is None else rng.random((B, cross)) < 0.7
    got = om.make_att_block_ids(pad, att, cross, cpad)
    ref = _brute_block_ids(pad, att, cross, cpad)
    for g, r in zip(got, ref):
        np.testing.assert_array_equal(np.asarray(g).astype(np.int64), np.asarray(r).astype(np.int64))
    np.testing.assert_array_equal(om.blockid_dense(*got), _brute_dense(*ref))


def test_block_ids_before_first_open_are_zero():
    att = np.array([[0, 0, 1, 0, 1, 1, 0]], dtype=np.uint8)
    pad = np.ones_like(att, dtype=bool)
    q_blk, k_blk, _, _ = om.make_att_block_ids(pad, att)
    np.testing.assert_array_equal(q_blk[0], [0, 0, 1, 1, 2, 3, 3])


def test_block_causal_structure():
    """Inside one block every pair attends both ways; later blocks see earlier ones only."""
    att = np.zeros((1, 12), dtype=np.uint8)
    att[0, [0, 5, 9]] = 1                      # blocks [0,5) [5,9) [9,12)
    pad = np.ones((1, 12), dtype=bool)
    M = om.blockid_dense(*om.make_att_block_ids(pad, att))[0]
    blocks = [range(0, 5), range(5, 9), range(9, 12)]
    for bi, rows in enumerate(blocks):
        for bj, cols in enumerate(blocks):
            sub = M[np.ix_(list(rows), list(cols))]
            assert sub.all() if bj <= bi else not sub.any()


def test_cross_columns_always_attended_unless_padded():
    rng = np.random.default_rng(7)
    B, N, C = 3, 10, 5
    att = (rng.random((B, N)) < 0.4).astype(np.uint8)
    pad = rng.random((B, N)) < 0.7
    cpad = rng.random((B, C)) < 0.6
    M = om.blockid_dense(*om.make_att_block_ids(pad, att, C, cpad))
    for b in range(B):
        for i in range(N):
            if pad[b, i]:
                np.testing.assert_array_equal(M[b, i, :C], cpad[b])
            else:
                assert not M[b, i].any()


def test_missing_cross_pad_is_an_error():
    with pytest.raises(ValueError):
        om.make_att_block_ids(np.ones((1, 4), bool), np.ones((1, 4), np.uint8), 2, None)


def test_causal_equals_lower_triangle():
    for Sq, Sk in [(1, 1), (7, 7), (33, 33), (5, 9)]:
        ref = np.array([[j <= i for j in range(Sk)] for i in range(Sq)])
        np.testing.assert_array_equal(om.positional_dense(Sq, Sk, causal=True), ref)
    np.testing.assert_array_equal(om.positional_dense(4, 6, causal=False), np.ones((4, 6), bool))


@pytest.mark.parametrize("W", [1, 2, 5, 17, 64, 100])
def test_window_matches_direct_loop(W):
    N = 64
    ref = np.zeros((N, N), dtype=bool)
    for i in range(N):
        for j in range(N):
            ref[i, j] = (i - j >= 0) and (i - j < W)
    np.testing.assert_array_equal(om.positional_dense(N, N, causal=True, window=W), ref)


def _read_golden_window(path):
    rows = []
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        rows.append([int(x) for x in line.split()])
    return rows


def test_window_example_from_the_page(golden_dir):
    rows = _read_golden_window(os.path.join(golden_dir, "omni_causal_window4_16.txt"))
    M_pos = om.positional_dense(16, 16, causal=True, window=4)
    M_pred = om.create_mask(om.and_masks(om.causal, om.window(4)), 1, 1, 16, 16)[0, 0]
    np.testing.assert_array_equal(M_pos, M_pred)
    for qi, first, last, n in rows:
        att = np.nonzero(M_pos[qi])[0]
        assert att[0] == first and att[-1] == last and att.size == n
        assert att.size == last - first + 1


def test_predicate_algebra():
    a = om.create_mask(om.causal, 1, 1, 9, 9)[0, 0]
    w = om.create_mask(om.window(3), 1, 1, 9, 9)[0, 0]
    np.testing.assert_array_equal(om.create_mask(om.and_masks(om.causal, om.window(3)), 1, 1, 9, 9)[0, 0], a & w)
    np.testing.assert_array_equal(om.create_mask(om.or_masks(om.causal, om.window(3)), 1, 1, 9, 9)[0, 0], a | w)
    assert om.create_mask(om.noop_mask, 2, 2, 3, 5).all()
    assert om.create_mask(om.and_masks(), 1, 1, 2, 2).all()
    assert not om.create_mask(om.or_masks(), 1, 1, 2, 2).any()


def test_varlen_example_from_the_page(golden_dir):
    vals = {}
    for line in open(os.path.join(golden_dir, "varlen_packed_example.txt")):
        if line.startswith("#") or not line.strip():
            continue
        key, *rest = line.split()
        vals[key] = [int(x) for x in rest]
    cu = np.array(vals["cu_seqlens"], dtype=np.int32)
    assert list(np.diff(cu)) == vals["lengths"] and cu[-1] == vals["total"][0]
    M = om.varlen_dense(cu, cu, causal=True)
    assert M.shape == (16, 16)
    # keys of another sequence are never attended
    assert not M[:5, 5:].any() and not M[5:, :5].any()
    np.testing.assert_array_equal(M[:5, :5], np.tril(np.ones((5, 5), bool)))
    np.testing.assert_array_equal(M[5:, 5:], np.tril(np.ones((11, 11), bool)))


def test_varlen_window_and_unequal_lengths():
    cq = np.array([0, 3, 10, 10, 14], dtype=np.int32)   # includes an empty sequence
    ck = np.array([0, 4, 9, 12, 20], dtype=np.int32)
    M = om.varlen_dense(cq, ck, causal=True, window=2)
    ref = np.zeros((14, 20), dtype=bool)
    for s in range(4):
        for i in range(cq[s], cq[s + 1]):
            for j in range(ck[s], ck[s + 1]):
                li, lj = i - cq[s], j - ck[s]
                ref[i, j] = 0 <= li - lj < 2
    np.testing.assert_array_equal(M, ref)


def test_varlen_with_block_ids():
    cu = np.array([0, 4, 9], dtype=np.int32)
    qb = np.array([0, 0, 1, 1, 0, 1, 1, 2, 2], dtype=np.int32)
    M = om.varlen_dense(cu, cu, q_blk=qb, k_blk=qb)
    ref = np.zeros((9, 9), dtype=bool)
    for s in range(2):
        for i in range(cu[s], cu[s + 1]):
            for j in range(cu[s], cu[s + 1]):
                ref[i, j] = qb[j] <= qb[i]
    np.testing.assert_array_equal(M, ref)


def _brute_bsr(indptr, indices, Sq, Skv, qb, kb, causal):
    B, H, _ = indptr.shape
    M = np.zeros((B, H, Sq, Skv), dtype=bool)
    for b in range(B):
        for h in range(H):
            for i in range(Sq):
                r = i // qb
                sel = set(int(x) for x in indices[indptr[b, h, r]:indptr[b, h, r + 1]])
                for j in range(Skv):
                    M[b, h, i, j] = (j // kb in sel) and (not causal or j <= i)
    return M


@pytest.mark.parametrize("causal", [False, True])
def test_bsr_expand_matches_brute_force(causal):
    rng = np.random.default_rng(11)
    B, H, Sq, Skv, qb, kb = 2, 2, 19, 23, 4, 5
    nqb, nkb = -(-Sq // qb), -(-Skv // kb)
    indptr = np.zeros((B, H, nqb + 1), dtype=np.int32)
    idx = []
    pos = 0
    for b in range(B):
        for h in range(H):
            indptr[b, h, 0] = pos
            for r in range(nqb):
                row = np.sort(rng.choice(nkb, size=rng.integers(0, nkb + 1), replace=False))
                idx.append(row)
                pos += row.size
                indptr[b, h, r + 1] = pos
    indices = np.concatenate(idx).astype(np.int32)
    got = om.bsr_dense(indptr, indices, Sq, Skv, qb, kb, causal=causal)
    np.testing.assert_array_equal(got, _brute_bsr(indptr, indices, Sq, Skv, qb, kb, causal))
    assert om.bsr_is_canonical(indptr, indices, nkb)


def test_bsr_canonical_checks():
    indptr = np.array([[[0, 2, 3]]], dtype=np.int32)
    assert om.bsr_is_canonical(indptr, np.array([0, 1, 1], np.int32), 2)
    assert not om.bsr_is_canonical(indptr, np.array([1, 0, 1], np.int32), 2)       # unsorted
    assert not om.bsr_is_canonical(indptr, np.array([1, 1, 1], np.int32), 2)       # duplicate
    assert not om.bsr_is_canonical(indptr, np.array([0, 1, 2], np.int32), 2)       # out of range
    assert not om.bsr_is_canonical(np.array([[[0, 3, 2]]], np.int32), np.array([0, 1, 1], np.int32), 2)
    assert not om.bsr_is_canonical(np.array([[[0, 2, 4]]], np.int32), np.array([0, 1, 1], np.int32), 2)


def _pack_bits(sel):
    """bool (..., n) -> uint32 words LSB-first, written as an explicit loop."""
    *lead, n = sel.shape
    words = -(-n // 32)
    out = np.zeros((*lead, words), dtype=np.uint32)
    for idx in np.ndindex(*lead):
        for j in range(n):
            if sel[idx + (j,)]:
                out[idx + (j // 32,)] |= np.uint32(1) << np.uint32(j % 32)
    return out


@pytest.mark.parametrize("qb,kb,causal", [(4, 8, False), (3, 5, True), (16, 16, True)])
def test_block_bits_expand_matches_brute_force(qb, kb, causal):
    rng = np.random.default_rng(qb * 10 + kb)
    B, H, Sq, Skv = 2, 2, 37, 45
    nqb, nkb = -(-Sq // qb), -(-Skv // kb)
    sel = rng.random((B, H, nqb, nkb)) < 0.4
    valid = rng.random((B, Skv)) < 0.8
    got = om.block_bits_dense(_pack_bits(sel), Sq, Skv, qb, kb, causal=causal, kv_valid_bits=_pack_bits(valid))
    ref = np.zeros((B, H, Sq, Skv), dtype=bool)
    for b in range(B):
        for h in range(H):
            for i in range(Sq):
                for j in range(Skv):
                    ref[b, h, i, j] = sel[b, h, i // qb, j // kb] and valid[b, j] and (not causal or j <= i)
    np.testing.assert_array_equal(got, ref)


def test_bsr_and_block_bits_select_the_same_mask():
    from workloads import bsr_routing
    indptr, indices = bsr_routing(1, 2, 6, 5)
    bits = om.bsr_to_block_bits(indptr, indices, 6)
    for causal in (False, True):
        np.testing.assert_array_equal(om.bsr_dense(indptr, indices, 6 * 7, 6 * 9, 7, 9, causal=causal),
                                      om.block_bits_dense(bits, 6 * 7, 6 * 9, 7, 9, causal=causal))


def _brute_terms(terms, Sq, Sk):
    M = np.zeros((Sq, Sk), dtype=bool)
    for i in range(Sq):
        for j in range(Sk):
            for t in terms:
                ok = True
                for key, test in (("diag_lo", lambda v: i - j >= v), ("diag_hi", lambda v: i - j <= v),
                                  ("q_lo", lambda v: i >= v), ("q_hi", lambda v: i < v),
                                  ("k_lo", lambda v: j >= v), ("k_hi", lambda v: j < v)):
                    if t.get(key) is not None and not test(t[key]):
                        ok = False
                if ok:
                    M[i, j] = True
                    break
    return M


PREDICATES = {
    "causal": [om.term(diag_lo=0)],
    "window5": [om.term(diag_lo=0, diag_hi=4)],
    "prefix_lm7": [om.term(diag_lo=0), om.term(k_hi=7)],
    "global3_window4": [om.term(diag_lo=0, diag_hi=3), om.term(q_hi=3), om.term(k_hi=3)],
    "two_bands": [om.term(diag_lo=-2, diag_hi=2), om.term(diag_lo=10, diag_hi=12, q_lo=5, q_hi=20)],
    "noop": [om.term()],
    "none": [],
}


@pytest.mark.parametrize("name", sorted(PREDICATES))
def test_predicate_terms_match_brute_force(name):
    terms = PREDICATES[name]
    np.testing.assert_array_equal(om.predicate_dense(terms, 23, 29), _brute_terms(terms, 23, 29))


def test_predicate_terms_match_the_page_algebra():
    """causal / window terms equal the omni_attention predicates built with and_masks / or_masks."""
    np.testing.assert_array_equal(om.predicate_dense([om.term(diag_lo=0, diag_hi=3)], 16, 16),
                                  om.create_mask(om.and_masks(om.causal, om.window(4)), 1, 1, 16, 16)[0, 0])
    glob = lambda b, h, qi, ki: (qi < 3) | (ki < 3)
    alg = om.create_mask(om.or_masks(om.and_masks(om.causal, om.window(4)), glob), 1, 1, 20, 20)[0, 0]
    np.testing.assert_array_equal(om.predicate_dense(PREDICATES["global3_window4"], 20, 20), alg)
    assert om.predicate_dense(PREDICATES["noop"], 4, 6).all()
    assert not om.predicate_dense([], 4, 6).any()


def test_gqa_packed_rows_hand_example_and_brute_force():
    # two positions, two keys, two heads per kv head: each position's row appears
    # once per head, position-major (row t = position t // 2, head t % 2)
    M = np.array([[1, 0], [0, 1]], dtype=bool)
    np.testing.assert_array_equal(om.gqa_packed_rows(M, 2),
                                  np.array([[1, 0], [1, 0], [0, 1], [0, 1]], dtype=bool))
    rng = np.random.default_rng(3)
    A = rng.random((37, 53)) < 0.4
    for G in (1, 2, 4, 8):
        P = om.gqa_packed_rows(A, G)
        assert P.shape == (37 * G, 53)
        for t in range(P.shape[0]):
            np.testing.assert_array_equal(P[t], A[t // G])
    np.testing.assert_array_equal(om.gqa_packed_rows(A, 1), A)


def test_gqa_packed_rows_of_a_bsr_routing_follow_the_routing():
    # packed rows of a BSR mask: row t attends key j exactly when position t // G's
    # BSR row lists j's block (checked against the routing directly, not via bsr_dense)
    indptr = np.array([[[0, 2, 3, 5]]], dtype=np.int32)
    indices = np.array([0, 2, 1, 0, 3], dtype=np.int32)
    Sq, Skv, qb, kb, G = 12, 32, 4, 8, 4
    packed = om.gqa_packed_rows(om.bsr_dense(indptr, indices, Sq, Skv, qb, kb)[0, 0], G)
    for t in range(Sq * G):
        r = (t // G) // qb
        blocks = set(indices[indptr[0, 0, r]:indptr[0, 0, r + 1]].tolist())
        for j in range(Skv):
            assert packed[t, j] == (j // kb in blocks)


def test_short_row_bsr_routing_is_canonical_and_follows_its_rule():
    # the 16-token-row routing of the packed-tile workload: canonical rows, each the key
    # block of its first token plus floor(d / 4) distinct earlier blocks
    import workloads
    Sq, qb, kb = 1000, 16, 128
    ip, ix = workloads.bsr_rows_routing(2, 3, Sq, qb, kb, 11)
    assert ip.shape == (2, 3, -(-Sq // qb) + 1)
    assert om.bsr_is_canonical(ip, ix, -(-Sq // kb))
    for b in range(2):
        for h in range(3):
            for r in range(ip.shape[2] - 1):
                row = ix[ip[b, h, r]:ip[b, h, r + 1]]
                d = (r * qb) // kb
                assert row[-1] == d and row.size == d // 4 + 1 and (row[:-1] < d).all()
