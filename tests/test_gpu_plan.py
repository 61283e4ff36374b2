"""GPU planner parity: every plan is compared bit for bit with the oracle's plan.

The oracle plan of any mask form is the plan of its dense mask (built by the
oracle's own builders); the GPU planners get the compact forms (dense bytes,
block ids, positions, BSR routing, exact-block bitmaps) through the C ABI.
"""

import numpy as np
import pytest
import torch

import workloads
from helpers import assert_plan_equal, oracle_plan_for_groups
from oracle import masks as om

pytestmark = pytest.mark.gpu

bfa = pytest.importorskip("mask_skipping_flashattention_b200")


def _cuda(x, dtype=None):
    t = torch.as_tensor(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


# ---------------------------------------------------------------- dense plans
@pytest.mark.parametrize("shape,density", [
    ((1, 1), 1.0), ((1, 1), 0.0), ((5, 300), 0.5), ((128, 128), 0.999), ((129, 257), 0.3),
    ((300, 200), 0.001), ((1000, 1300), 0.05), ((513, 129), 1.0), ((2048, 2048), 0.0),
])
def test_dense_plan_random(shape, density):
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    M = rng.random(shape) < density
    if shape[0] >= 256 and shape[1] >= 256:
        M[:128, :128] = True         # a full tile
        M[128:256, 128:256] = False  # an empty tile
    got = bfa.plan_dense(_cuda(M)).export()
    assert_plan_equal(got, oracle_plan_for_groups([M]))


def test_dense_plan_strided_and_uint8_mask():
    rng = np.random.default_rng(3)
    big = rng.random((300, 512)) < 0.2
    t = _cuda(big)[:, :333]                    # row stride 512 bytes, 333 columns
    got = bfa.plan_dense(t).export()
    assert_plan_equal(got, oracle_plan_for_groups([big[:, :333]]))
    t2 = _cuda(big.astype(np.uint8) * 7)[:, 1:300]   # nonzero bytes, unaligned base
    got = bfa.plan_dense(t2).export()
    assert_plan_equal(got, oracle_plan_for_groups([big[:, 1:300]]))
    # aligned rows of bytes other than 0 / 1 (any nonzero byte attends), mixed with
    # bool-like 16-byte runs: both ways of packing the bits on the vector path
    vals = rng.integers(1, 256, size=big.shape).astype(np.uint8)
    vals[:, :256] = 1
    t3 = _cuda(np.where(big, vals, 0).astype(np.uint8))
    got = bfa.plan_dense(t3).export()
    assert_plan_equal(got, oracle_plan_for_groups([big]))


def test_dense_plan_tiny_blockcausal():
    w = workloads.tiny_blockcausal()
    ids = om.make_att_block_ids(w["pad_masks"], w["att_masks"])
    M = om.blockid_dense(*ids)[0]
    assert_plan_equal(bfa.plan_dense(_cuda(M)).export(), oracle_plan_for_groups([M]))


def test_dense_plan_causal_8192():
    w = workloads.causal_8192(with_qkv=False)
    P = bfa.plan_dense(w["mask"].cuda())
    assert P.stats() == (2016, 64, 2016)
    assert_plan_equal(P.export(), oracle_plan_for_groups([w["mask"].numpy()]))


def test_dense_plan_union_16384():
    w = workloads.union_16384(with_qkv=False)
    M = w["mask"]
    P = bfa.plan_dense(M.cuda())
    assert_plan_equal(P.export(), oracle_plan_for_groups([M.numpy()]))


# ---------------------------------------------------------------- block ids
def test_make_block_ids_matches_oracle():
    w = workloads.blockcausal_gqa()
    ref = om.make_att_block_ids(w["pad_masks"], w["att_masks"], w["n_cross"], w["cross_pad_masks"])
    got = bfa.make_att_block_ids(_cuda(w["pad_masks"]), _cuda(w["att_masks"]), w["n_cross"],
                                 _cuda(w["cross_pad_masks"]))
    for g, r in zip(got, ref):
        np.testing.assert_array_equal(g.cpu().numpy().astype(np.int64), np.asarray(r).astype(np.int64))


@pytest.mark.parametrize("name", ["tiny_blockcausal", "blockcausal_gqa"])
def test_blockid_plan_matches_dense_oracle(name):
    w = workloads.get(name)
    nc = w.get("n_cross")
    ref_ids = om.make_att_block_ids(w["pad_masks"], w["att_masks"], nc, w.get("cross_pad_masks"))
    dense = om.blockid_dense(*ref_ids)
    ids = bfa.make_att_block_ids(_cuda(w["pad_masks"]), _cuda(w["att_masks"]), nc,
                                 _cuda(w["cross_pad_masks"]) if nc else None)
    P = bfa.plan_blockids(*ids)
    assert P.kind == "blockids"
    ref = oracle_plan_for_groups(list(dense))
    assert_plan_equal(P.export(), ref)
    # the block-id planner's classes equal the dense planner's on the materialised mask
    for b in range(dense.shape[0]):
        Pd = bfa.plan_dense(_cuda(dense[b])).export()
        nq, nk = ref["cls"][b].shape
        np.testing.assert_array_equal(P.export()["classes"][b * nq * nk:(b + 1) * nq * nk], Pd["classes"])


@pytest.mark.parametrize("seed", range(4))
def test_blockid_plan_random_ragged(seed):
    rng = np.random.default_rng(40 + seed)
    B, Sq, Sk = 3, int(rng.integers(1, 700)), int(rng.integers(1, 900))
    qb = np.sort(rng.integers(0, 6, size=(B, Sq)), axis=1).astype(np.int32)
    kb = rng.integers(-3, 8, size=(B, Sk)).astype(np.int32)
    kb[:, : min(5, Sk)] = np.iinfo(np.int32).min
    qv = rng.random((B, Sq)) < (0.9 if seed % 2 else 1.0)
    kv = rng.random((B, Sk)) < 0.8
    P = bfa.plan_blockids(_cuda(qb), _cuda(kb), _cuda(qv), _cuda(kv))
    dense = om.blockid_dense(qb, kb, qv, kv)
    assert_plan_equal(P.export(), oracle_plan_for_groups(list(dense)))


def test_positional_batched_plan():
    P = bfa.plan_blockids(B=2, Sq=1000, Sk=1000)
    assert P.kind == "positional"
    M = om.positional_dense(1000, 1000, causal=True)
    assert_plan_equal(P.export(), oracle_plan_for_groups([M, M]))


def test_positional_with_validity_uses_predicate_plan():
    rng = np.random.default_rng(5)
    qv = rng.random((2, 300)) < 0.9
    P = bfa.plan_blockids(q_valid=_cuda(qv), k_valid=_cuda(np.ones((2, 300), bool)), B=2, Sq=300, Sk=300)
    assert P.kind == "blockids"
    masks = [om.positional_dense(300, 300) & qv[b][:, None] for b in range(2)]
    assert_plan_equal(P.export(), oracle_plan_for_groups(masks))


# ---------------------------------------------------------------- varlen
def _varlen_oracle(cu_q, cu_k, window):
    masks = []
    for s in range(len(cu_q) - 1):
        lq, lk = int(cu_q[s + 1] - cu_q[s]), int(cu_k[s + 1] - cu_k[s])
        masks.append(om.positional_dense(lq, lk, causal=True, window=window))
    return masks


@pytest.mark.parametrize("window", [-1, 1024])
def test_varlen_plan_workload(window):
    w = workloads.varlen_16()
    cu = _cuda(w["cu_seqlens"])
    P = bfa.plan_blockids(cu_seqlens_q=cu, cu_seqlens_k=cu, max_q=w["max_len"], max_k=w["max_len"],
                          window_left=window)
    assert P.info["varlen"] == 1 and P.info["n_groups"] == 16
    assert_plan_equal(P.export(), oracle_plan_for_groups(_varlen_oracle(w["cu_seqlens"], w["cu_seqlens"], window)))


@pytest.mark.parametrize("window", [-1, 1, 7, 200])
def test_varlen_plan_ragged_unequal(window):
    cq = np.array([0, 3, 3, 260, 900, 901], dtype=np.int32)     # includes an empty sequence
    ck = np.array([0, 130, 131, 131, 700, 1000], dtype=np.int32)
    P = bfa.plan_blockids(cu_seqlens_q=_cuda(cq), cu_seqlens_k=_cuda(ck), max_q=640, max_k=600,
                          window_left=window)
    assert_plan_equal(P.export(), oracle_plan_for_groups(_varlen_oracle(cq, ck, window)))


def test_varlen_understated_max_is_an_error():
    cu = _cuda(np.array([0, 100, 300], dtype=np.int32))
    with pytest.raises(bfa.BfaError) as e:
        bfa.plan_blockids(cu_seqlens_q=cu, cu_seqlens_k=cu, max_q=150, max_k=300)
    assert e.value.status == "BFA_ERR_INVALID_ARG"


# ---------------------------------------------------------------- BSR
def _bsr_oracle(indptr, indices, S, causal):
    D = om.bsr_dense(indptr, indices, S, S, 128, 128, causal=causal)
    return [D[b, h] for b in range(D.shape[0]) for h in range(D.shape[1])]


@pytest.mark.parametrize("causal", [False, True])
def test_bsr_plan_small(causal):
    indptr, indices = workloads.bsr_routing(2, 3, 9, 77)
    S = 9 * 128 - 50                       # ragged last block
    P = bfa.plan_bsr(_cuda(indptr), _cuda(indices), S, S, causal=causal)
    assert_plan_equal(P.export(), oracle_plan_for_groups(_bsr_oracle(indptr, indices, S, causal)))


def test_bsr_plan_workload_full_size_every_group():
    """The BSR 16384 workload's plan, bit for bit on all 16 (batch, kv head) groups:
    the oracle plan is built one group's 16384 x 16384 mask at a time and the groups
    are combined (rows concatenated, then the row order and the work pairs over all
    rows).  The same routing in the exact-block bitmask form gives the same plan
    (with its packed fine words)."""
    from oracle import plan as op
    w = workloads.bsr_16384(with_qkv=False)
    ip, ix, S = w["block_indptr"], w["block_indices"], w["S"]
    B, Hkv, _ = ip.shape
    P = bfa.plan_bsr(_cuda(ip), _cuda(ix), S, S, causal=True)
    n_full, n_part, n_empty = P.stats()
    assert n_part == B * Hkv * 128 and n_full == B * Hkv * 1984
    groups = []
    for b in range(B):
        for h in range(Hkv):
            groups.append(op.plan_group(_bsr_oracle(ip[b:b + 1, h:h + 1], ix, S, True)[0]))
    ref = op.combine_groups(groups)
    assert_plan_equal(P.export(), ref)
    bits = om.bsr_to_block_bits(ip, ix, -(-S // 128))
    P2 = bfa.plan_block_bits(_cuda(bits.view(np.int32)), S, S, causal=True)
    assert_plan_equal(P2.export(), ref)


def test_bsr_noncanonical_rejected():
    indptr = np.array([[[0, 2, 3]]], dtype=np.int32)
    for bad in ([1, 0, 1], [1, 1, 1], [0, 1, 2]):
        with pytest.raises(bfa.BfaError) as e:
            bfa.plan_bsr(_cuda(indptr), _cuda(np.array(bad, np.int32)), 256, 256)
        assert e.value.status == "BFA_ERR_NONCANONICAL_BSR"
    with pytest.raises(bfa.BfaError) as e:
        bfa.plan_bsr(_cuda(np.array([[[0, 3, 2]]], np.int32)), _cuda(np.array([0, 1, 1], np.int32)), 256, 256)
    assert e.value.status == "BFA_ERR_NONCANONICAL_BSR"


def test_plan_rejects_host_memory():
    with pytest.raises(bfa.BfaError) as e:
        bfa.plan_dense(torch.ones(8, 8, dtype=torch.bool))
    assert e.value.status == "BFA_ERR_NOT_DEVICE"


# ---------------------------------------------------------------- general block sparsity
def _routing(B, H, nqb, nkb, seed, density=0.35):
    rng = np.random.default_rng(seed)
    indptr = np.zeros((B, H, nqb + 1), dtype=np.int32)
    idx, pos = [], 0
    for b in range(B):
        for h in range(H):
            indptr[b, h, 0] = pos
            for r in range(nqb):
                row = np.sort(rng.choice(nkb, size=int(rng.binomial(nkb, density)), replace=False))
                idx.append(row)
                pos += row.size
                indptr[b, h, r + 1] = pos
    return indptr, np.concatenate(idx).astype(np.int32)


def _valid_bits(B, Skv, seed):
    rng = np.random.default_rng(seed)
    valid = rng.random((B, Skv)) < 0.9
    words = -(-Skv // 32)
    out = np.zeros((B, words), dtype=np.uint32)
    for b in range(B):
        for j in np.nonzero(valid[b])[0]:
            out[b, j // 32] |= np.uint32(1) << np.uint32(j % 32)
    return out


@pytest.mark.parametrize("qb,kb,causal,valid", [
    (64, 64, True, False), (32, 8, False, True), (100, 192, True, True), (128, 16, False, False),
    (128, 128, True, True), (7, 32, True, False),
])
def test_general_block_sparse_plans(qb, kb, causal, valid):
    B, H, Sq, Skv = 2, 2, 450, 600
    nqb, nkb = -(-Sq // qb), -(-Skv // kb)
    indptr, indices = _routing(B, H, nqb, nkb, qb * 1000 + kb)
    kvb = _valid_bits(B, Skv, kb) if valid else None
    P = bfa.plan_bsr(_cuda(indptr), _cuda(indices), Sq, Skv, qb, kb, causal=causal,
                     kv_valid_bits=_cuda(kvb.view(np.int32)) if valid else None)
    assert P.info["packed_fine"] == 1
    D = om.block_bits_dense(om.bsr_to_block_bits(indptr, indices, nkb), Sq, Skv, qb, kb, causal=causal,
                            kv_valid_bits=kvb)
    ref = oracle_plan_for_groups([D[b, h] for b in range(B) for h in range(H)])
    assert_plan_equal(P.export(), ref)
    # the bitmask format selects the same mask
    bits = om.bsr_to_block_bits(indptr, indices, nkb)
    P2 = bfa.plan_block_bits(_cuda(bits.view(np.int32)), Sq, Skv, qb, kb, causal=causal,
                             kv_valid_bits=_cuda(kvb.view(np.int32)) if valid else None)
    assert_plan_equal(P2.export(), ref)


def test_general_block_sparse_rejects_bad_blocks():
    indptr, indices = _routing(1, 1, 4, 10, 3)
    for kb in (0, 24, 48, 100):
        with pytest.raises(bfa.BfaError) as e:
            bfa.plan_bsr(_cuda(indptr), _cuda(indices), 256, 640, 64, kb)
        assert e.value.status == "BFA_ERR_INVALID_ARG"


# ---------------------------------------------------------------- position-term predicates
PRED_CASES = {
    "causal": [om.term(diag_lo=0)],
    "window100": [om.term(diag_lo=0, diag_hi=99)],
    "prefix_lm": [om.term(diag_lo=0), om.term(k_hi=300)],
    "global64_window256": [om.term(diag_lo=0, diag_hi=255), om.term(q_hi=64), om.term(k_hi=64)],
    "two_bands": [om.term(diag_lo=-20, diag_hi=20), om.term(diag_lo=400, diag_hi=412, q_lo=450, q_hi=700)],
    "noop": [om.term()],
    "none": [],
}


@pytest.mark.parametrize("name", sorted(PRED_CASES))
def test_predicate_plan_batched(name):
    terms = PRED_CASES[name]
    P = bfa.plan_predicate(terms, B=2, Sq=700, Sk=650)
    assert P.kind == "predicate"
    M = om.predicate_dense(terms, 700, 650)
    assert_plan_equal(P.export(), oracle_plan_for_groups([M, M]))


def test_predicate_plan_varlen_seqused():
    terms = PRED_CASES["prefix_lm"]
    cq = np.array([0, 500, 501, 1300], dtype=np.int32)
    ck = np.array([0, 400, 900, 1700], dtype=np.int32)
    used = np.array([400, 350, 790], dtype=np.int32)
    P = bfa.plan_predicate(terms, cu_seqlens_q=_cuda(cq), cu_seqlens_k=_cuda(ck), seqused_k=_cuda(used),
                           max_q=800, max_k=800)
    masks = []
    for s in range(3):
        lq, lk = int(cq[s + 1] - cq[s]), int(min(ck[s + 1] - ck[s], used[s]))
        masks.append(om.predicate_dense(terms, lq, lk))
    assert_plan_equal(P.export(), oracle_plan_for_groups(masks))


# ---------------------------------------------------------------- transposed lists (backward)
def _assert_cols_equal(P, masks):
    from oracle import plan as op
    ref = op.transpose_plan(op.plan_masks(masks)["cls"])
    got = P.export_cols()
    np.testing.assert_array_equal(got["col_ptr"], ref["col_ptr"], err_msg="col_ptr")
    np.testing.assert_array_equal(got["q_tile"], ref["q_tile"], err_msg="q_tile")
    np.testing.assert_array_equal((got["tpart"] >= 0).astype(np.uint8), ref["partial"], err_msg="partial flags")
    np.testing.assert_array_equal(got["col_order"], ref["order"], err_msg="column order")


@pytest.mark.parametrize("shape,density", [((1, 1), 1.0), ((300, 420), 0.01), ((1000, 700), 0.3), ((513, 129), 1.0)])
def test_transposed_lists_dense(shape, density):
    rng = np.random.default_rng(shape[0] + shape[1])
    M = rng.random(shape) < density
    _assert_cols_equal(bfa.plan_dense(_cuda(M)), [M])


def test_transposed_lists_causal_8192_and_blockids():
    M = np.tril(np.ones((8192, 8192), dtype=bool))
    _assert_cols_equal(bfa.plan_dense(_cuda(M)), [M])
    P = bfa.plan_blockids(B=2, Sq=700, Sk=650, window_left=100)
    M2 = om.positional_dense(700, 650, True, 100)
    _assert_cols_equal(P, [M2, M2])


def test_transposed_lists_block_bits_and_predicates():
    B, H, Sq, Skv, qb, kb = 2, 2, 450, 600, 32, 8
    nqb, nkb = -(-Sq // qb), -(-Skv // kb)
    indptr, indices = _routing(B, H, nqb, nkb, 77)
    P = bfa.plan_bsr(_cuda(indptr), _cuda(indices), Sq, Skv, qb, kb, causal=True)
    D = om.block_bits_dense(om.bsr_to_block_bits(indptr, indices, nkb), Sq, Skv, qb, kb, causal=True)
    _assert_cols_equal(P, [D[b, h] for b in range(B) for h in range(H)])
    terms = PRED_CASES["global64_window256"]
    Pp = bfa.plan_predicate(terms, B=2, Sq=700, Sk=650)
    Mp = om.predicate_dense(terms, 700, 650)
    _assert_cols_equal(Pp, [Mp, Mp])


# ---------------------------------------------------------------- GQA-packed BSR plans
@pytest.mark.parametrize("qb,kb,G,causal,valid", [
    (16, 128, 8, False, False), (16, 64, 8, True, True), (32, 128, 4, True, False), (64, 32, 2, False, True),
    (8, 16, 16, True, False), (100, 128, 2, False, False),
])
def test_bsr_packed_plans(qb, kb, G, causal, valid):
    # the plan of each (batch, kv head) group over its packed rows (position-major,
    # every head of the kv head), bit for bit against the oracle's plan of the same rows
    B, Hkv, Sq, Skv = 2, 2, 300, 520
    nqb, nkb = -(-Sq // qb), -(-Skv // kb)
    indptr, indices = _routing(B, Hkv, nqb, nkb, qb * 100 + kb + G)
    kvb = _valid_bits(B, Skv, G) if valid else None
    P = bfa.plan_bsr_packed(_cuda(indptr), _cuda(indices), Sq, Skv, G, qb, kb, causal=causal,
                            kv_valid_bits=_cuda(kvb.view(np.int32)) if valid else None)
    assert P.info["heads_per_kv"] == G and P.info["sq"] == Sq
    M = om.block_bits_dense(om.bsr_to_block_bits(indptr, indices, nkb), Sq, Skv, qb, kb, causal=causal,
                            kv_valid_bits=kvb)
    ref = oracle_plan_for_groups([om.gqa_packed_rows(M[b, h], G) for b in range(B) for h in range(Hkv)])
    assert_plan_equal(P.export(), ref)


def test_bsr_packed_rejects_bad_packing():
    indptr, indices = _routing(1, 1, 4, 4, 5)
    for qb, G in ((64, 3), (64, 256), (3, 2), (64, 0)):
        with pytest.raises(bfa.BfaError) as e:
            bfa.plan_bsr_packed(_cuda(indptr), _cuda(indices), 4 * qb, 512, G, qb, 128)
        assert e.value.status == "BFA_ERR_INVALID_ARG"
