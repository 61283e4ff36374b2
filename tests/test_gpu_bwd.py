"""GPU backward parity: dQ, dK, dV against the float64 oracle (oracle.backward).

The library's forward supplies out and lse (bf16 / fp32), as a training step
would; the oracle differentiates the exact forward definition in float64 on the
same bf16 inputs.  Tolerance: the kernel rounds P and dS to bf16 before their
products (relative 2^-9 each), uses the bf16 output for D = dO . O and rounds
the gradients to bf16; per gradient tensor the max-abs error must stay below
1e-2 of the tensor's largest magnitude plus 1e-3 (bf16 N(0, 1) inputs at the
default scale).  Rows that attend nothing and keys that no query attends get
exact zeros.
"""

import numpy as np
import pytest
import torch

import workloads
from oracle import backward as ob
from oracle import masks as om

pytestmark = pytest.mark.gpu

bfa = pytest.importorskip("mask_skipping_flashattention_b200")

REL = 1e-2
ABS = 1e-3


def _cuda(x):
    return torch.as_tensor(np.ascontiguousarray(x)).cuda()


def _close(got, ref, name):
    got = np.asarray(got.float().cpu(), dtype=np.float64)
    assert np.all(np.isfinite(got)), f"non-finite {name}"
    err = np.abs(got - ref).max() if ref.size else 0.0
    bound = REL * (np.abs(ref).max() if ref.size else 0.0) + ABS
    assert err <= bound, f"{name}: max-abs {err:.3e} > {bound:.3e}"
    return err


def _run_bshd(P, q, k, v, do, mask_for, scale=None):
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    out, lse = bfa.fwd(P, qc, kc, vc, scale=scale)
    dq, dk, dv = bfa.bwd(P, qc, kc, vc, out, dc, lse, scale=scale)
    torch.cuda.synchronize()
    P.device_status()
    rq, rk, rv = ob.attention_bwd_bshd(q, k, v, do, mask_for, scale)
    return (_close(dq, rq, "dq"), _close(dk, rk, "dk"), _close(dv, rv, "dv")), (dq, dk, dv)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("shape,density", [((300, 300), 0.3), ((129, 257), 0.9), ((512, 512), 0.02)])
def test_dense_random_masks(D, shape, density):
    Sq, Sk = shape
    rng = np.random.default_rng(Sq * 3 + Sk + D)
    M = rng.random((Sq, Sk)) < density
    M[:, 0] |= rng.random(Sq) < 0.5
    B, H = 1, 2
    q = workloads.randn_bf16((B, Sq, H, D), 11)
    k = workloads.randn_bf16((B, Sk, H, D), 12)
    v = workloads.randn_bf16((B, Sk, H, D), 13)
    do = workloads.randn_bf16((B, Sq, H, D), 14)
    _run_bshd(bfa.plan_dense(_cuda(M)), q, k, v, do, lambda b, h: M)


def test_dense_causal_gqa_two_batches():
    B, H, Hkv, N, D = 2, 4, 2, 384, 128
    M = np.tril(np.ones((N, N), dtype=bool))
    q = workloads.randn_bf16((B, N, H, D), 21)
    k = workloads.randn_bf16((B, N, Hkv, D), 22)
    v = workloads.randn_bf16((B, N, Hkv, D), 23)
    do = workloads.randn_bf16((B, N, H, D), 24)
    _run_bshd(bfa.plan_dense(_cuda(M)), q, k, v, do, lambda b, h: M, scale=0.1)


def test_blockids_with_padding_and_cross_columns():
    w = workloads.tiny_blockcausal()
    ids_ref = om.make_att_block_ids(w["pad_masks"], w["att_masks"])
    M = om.blockid_dense(*ids_ref)[0]
    P = bfa.plan_blockids(*bfa.make_att_block_ids(_cuda(w["pad_masks"]), _cuda(w["att_masks"])))
    do = workloads.randn_bf16(tuple(w["q"].shape), 31)
    errs, (dq, dk, dv) = _run_bshd(P, w["q"], w["k"], w["v"], do, lambda b, h: M, w["scale"])
    # padded query rows attend nothing; padded keys are attended by nothing
    assert torch.all(dq[0, 240:] == 0)
    assert torch.all(dk[0, 240:] == 0) and torch.all(dv[0, 240:] == 0)


def test_blockids_unsorted_and_sorted_key_tiles():
    # arbitrary key-id order on some key tiles, non-decreasing on others: both forms
    # of the block-id mask in the dQ pass (rows) and the dK/dV pass (columns)
    rng = np.random.default_rng(77)
    B, Sq, Sk, H, D = 1, 300, 400, 2, 64
    qb = np.sort(rng.integers(0, 9, size=(B, Sq)), axis=1).astype(np.int32)
    kb = rng.integers(-2, 10, size=(B, Sk)).astype(np.int32)
    kb[:, 128:256] = np.sort(kb[:, 128:256], axis=1)
    qv = rng.random((B, Sq)) < 0.9
    kv = rng.random((B, Sk)) < 0.85
    P = bfa.plan_blockids(_cuda(qb), _cuda(kb), _cuda(qv), _cuda(kv))
    M = om.blockid_dense(qb, kb, qv, kv)
    q = workloads.randn_bf16((B, Sq, H, D), 91)
    k = workloads.randn_bf16((B, Sk, H, D), 92)
    v = workloads.randn_bf16((B, Sk, H, D), 93)
    do = workloads.randn_bf16((B, Sq, H, D), 94)
    _run_bshd(P, q, k, v, do, lambda b, h: M[b])


def test_positional_window_batched():
    B, H, Sq, Sk, D, W = 2, 2, 700, 650, 64, 100
    P = bfa.plan_blockids(B=B, Sq=Sq, Sk=Sk, window_left=W)
    M = om.positional_dense(Sq, Sk, True, W)
    q = workloads.randn_bf16((B, Sq, H, D), 41)
    k = workloads.randn_bf16((B, Sk, H, D), 42)
    v = workloads.randn_bf16((B, Sk, H, D), 43)
    do = workloads.randn_bf16((B, Sq, H, D), 44)
    _run_bshd(P, q, k, v, do, lambda b, h: M)


def test_predicate_terms():
    terms = [om.term(diag_lo=0, diag_hi=255), om.term(q_hi=64), om.term(k_hi=64)]
    B, H, Sq, Sk, D = 1, 2, 600, 600, 128
    P = bfa.plan_predicate(terms, B=B, Sq=Sq, Sk=Sk)
    M = om.predicate_dense(terms, Sq, Sk)
    q = workloads.randn_bf16((B, Sq, H, D), 51)
    k = workloads.randn_bf16((B, Sk, H, D), 52)
    v = workloads.randn_bf16((B, Sk, H, D), 53)
    do = workloads.randn_bf16((B, Sq, H, D), 54)
    _run_bshd(P, q, k, v, do, lambda b, h: M)


def test_general_block_sparse_with_validity():
    B, H, Hkv, Sq, Skv, qb, kb, D = 1, 4, 2, 450, 600, 32, 8, 128
    nqb, nkb = -(-Sq // qb), -(-Skv // kb)
    rng = np.random.default_rng(5)
    indptr = np.zeros((B, Hkv, nqb + 1), dtype=np.int32)
    idx, pos = [], 0
    for b in range(B):
        for h in range(Hkv):
            indptr[b, h, 0] = pos
            for r in range(nqb):
                row = np.sort(rng.choice(nkb, size=int(rng.binomial(nkb, 0.3)), replace=False))
                idx.append(row)
                pos += row.size
                indptr[b, h, r + 1] = pos
    indices = np.concatenate(idx).astype(np.int32)
    valid = rng.random((B, Skv)) < 0.9
    kvb = np.zeros((B, -(-Skv // 32)), dtype=np.uint32)
    for b in range(B):
        for j in np.nonzero(valid[b])[0]:
            kvb[b, j // 32] |= np.uint32(1) << np.uint32(j % 32)
    P = bfa.plan_bsr(_cuda(indptr), _cuda(indices), Sq, Skv, qb, kb, causal=True,
                     kv_valid_bits=_cuda(kvb.view(np.int32)))
    Dm = om.block_bits_dense(om.bsr_to_block_bits(indptr, indices, nkb), Sq, Skv, qb, kb, causal=True,
                             kv_valid_bits=kvb)
    q = workloads.randn_bf16((B, Sq, H, D), 61)
    k = workloads.randn_bf16((B, Skv, Hkv, D), 62)
    v = workloads.randn_bf16((B, Skv, Hkv, D), 63)
    do = workloads.randn_bf16((B, Sq, H, D), 64)
    _run_bshd(P, q, k, v, do, lambda b, h: Dm[b, h // (H // Hkv)])


def test_varlen_causal_packed():
    cu = np.array([0, 5, 300, 300, 777], dtype=np.int32)  # includes an empty sequence
    T, H, Hkv, D = int(cu[-1]), 4, 2, 64
    P = bfa.plan_blockids(cu_seqlens_q=_cuda(cu), cu_seqlens_k=_cuda(cu), max_q=512, max_k=512)
    M = np.zeros((T, T), dtype=bool)
    for s in range(len(cu) - 1):
        a, z = cu[s], cu[s + 1]
        M[a:z, a:z] = np.tril(np.ones((z - a, z - a), dtype=bool))
    q = workloads.randn_bf16((T, H, D), 71)
    k = workloads.randn_bf16((T, Hkv, D), 72)
    v = workloads.randn_bf16((T, Hkv, D), 73)
    do = workloads.randn_bf16((T, H, D), 74)
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    out, lse = bfa.fwd(P, qc, kc, vc)
    dq, dk, dv = bfa.bwd(P, qc, kc, vc, out, dc, lse)
    torch.cuda.synchronize()
    P.device_status()
    rq, rk, rv = ob.attention_bwd_thd(q, k, v, do, M)
    _close(dq, rq, "dq")
    _close(dk, rk, "dk")
    _close(dv, rv, "dv")


def test_all_false_mask_gives_zero_gradients():
    M = np.zeros((200, 300), dtype=bool)
    q = workloads.randn_bf16((1, 200, 1, 64), 81).cuda()
    k = workloads.randn_bf16((1, 300, 1, 64), 82).cuda()
    v = workloads.randn_bf16((1, 300, 1, 64), 83).cuda()
    do = workloads.randn_bf16((1, 200, 1, 64), 84).cuda()
    P = bfa.plan_dense(_cuda(M))
    out, lse = bfa.fwd(P, q, k, v)
    dq, dk, dv = bfa.bwd(P, q, k, v, out, do, lse)
    torch.cuda.synchronize()
    assert torch.all(dq == 0) and torch.all(dk == 0) and torch.all(dv == 0)


def test_bwd_rejects_bad_arguments():
    M = np.ones((128, 128), dtype=bool)
    q = workloads.randn_bf16((1, 128, 1, 64), 91).cuda()
    P = bfa.plan_dense(_cuda(M))
    out, lse = bfa.fwd(P, q, q, q)
    with pytest.raises(TypeError):
        bfa.bwd(P, q, q, q, out, q, None)
    with pytest.raises(bfa.BfaError) as e:
        bfa.bwd(P, q.cpu(), q, q, out, q, lse)
    assert e.value.status == "BFA_ERR_NOT_DEVICE"


def test_blockcausal_gqa_cross_columns_one_batch():
    # the block-causal GQA workload (H=16 over Hkv=4, 256 cross columns, padding): all heads of one batch
    w = workloads.blockcausal_gqa(B=2)
    ids = bfa.make_att_block_ids(_cuda(w["pad_masks"]), _cuda(w["att_masks"]), w["n_cross"],
                                 _cuda(w["cross_pad_masks"]))
    P = bfa.plan_blockids(*ids)
    dense = om.blockid_dense(*om.make_att_block_ids(w["pad_masks"], w["att_masks"], w["n_cross"],
                                                    w["cross_pad_masks"]))
    do = workloads.randn_bf16(tuple(w["q"].shape), 101)
    qc, kc, vc, dc = w["q"].cuda(), w["k"].cuda(), w["v"].cuda(), do.cuda()
    out, lse = bfa.fwd(P, qc, kc, vc)
    dq, dk, dv = bfa.bwd(P, qc, kc, vc, out, dc, lse)
    torch.cuda.synchronize()
    P.device_status()
    b = 1
    rq, rk, rv = ob.attention_bwd_bshd(w["q"][b:b + 1], w["k"][b:b + 1], w["v"][b:b + 1], do[b:b + 1],
                                       lambda _b, h: dense[b])
    _close(dq[b:b + 1], rq, "dq")
    _close(dk[b:b + 1], rk, "dk")
    _close(dv[b:b + 1], rv, "dv")


def test_causal_8192_bench_workload_sampled_heads():
    # the bench's workload (B=4, H=32, N=8192, D=128) in the bench's launch; the oracle
    # differentiates two (batch, head) pairs in full
    w = workloads.causal_8192()
    M = w["mask"].numpy()
    do = workloads.randn_bf16(tuple(w["q"].shape), 4242)
    qc, kc, vc, dc = w["q"].cuda(), w["k"].cuda(), w["v"].cuda(), do.cuda()
    P = bfa.plan_dense(w["mask"].cuda())
    out, lse = bfa.fwd(P, qc, kc, vc)
    dq, dk, dv = bfa.bwd(P, qc, kc, vc, out, dc, lse)
    torch.cuda.synchronize()
    P.device_status()
    for (b, h) in [(0, 0), (3, 31)]:
        rq, rk, rv, _ = ob.masked_attention_bwd(w["q"][b, :, h], w["k"][b, :, h], w["v"][b, :, h], M,
                                                do[b, :, h], w["scale"])
        _close(dq[b, :, h], rq, f"dq {b},{h}")
        _close(dk[b, :, h], rk, f"dk {b},{h}")
        _close(dv[b, :, h], rv, f"dv {b},{h}")


# ---------------------------------------------------------------- full-size workloads
def _group_bwd_check(dq, dk, dv, q, k, v, do, M, g, rep, scale, rows, where):
    """Oracle gradients of kv head g (all `rep` query heads that read it) on the row range
    `rows` of packed (T, H, D) tensors, compared with the library's."""
    a, z = rows
    rk = np.zeros((z - a, k.shape[-1]))
    rv = np.zeros((z - a, v.shape[-1]))
    for h in range(g * rep, (g + 1) * rep):
        rq, k_, v_, _ = ob.masked_attention_bwd(q[a:z, h], k[a:z, g], v[a:z, g], M, do[a:z, h], scale)
        _close(dq[a:z, h], rq, f"{where} dq head {h}")
        rk += k_
        rv += v_
    _close(dk[a:z, g], rk, f"{where} dk kv head {g}")
    _close(dv[a:z, g], rv, f"{where} dv kv head {g}")


@pytest.mark.parametrize("window", [-1, 1024])
def test_varlen_workload_sampled_sequences(window):
    # the varlen workload (16 sequences of 512-4096 tokens, H=32 / Hkv=8, packed) in full on
    # the GPU; the oracle differentiates the first, the longest and the last sequence for the
    # first and the last kv-head group (the four query heads of a group sum into its dK / dV)
    w = workloads.varlen_16()
    cu = w["cu_seqlens"]
    P = bfa.plan_blockids(cu_seqlens_q=_cuda(cu), cu_seqlens_k=_cuda(cu), max_q=w["max_len"],
                          max_k=w["max_len"], window_left=window)
    do = workloads.randn_bf16(tuple(w["q"].shape), 4343)
    qc, kc, vc, dc = w["q"].cuda(), w["k"].cuda(), w["v"].cuda(), do.cuda()
    out, lse = bfa.fwd(P, qc, kc, vc)
    dq, dk, dv = bfa.bwd(P, qc, kc, vc, out, dc, lse)
    torch.cuda.synchronize()
    P.device_status()
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    rep = w["H"] // w["Hkv"]
    for s in sorted({0, int(np.argmax(w["lens"])), len(w["lens"]) - 1}):
        a, z = int(cu[s]), int(cu[s + 1])
        M = om.positional_dense(z - a, z - a, True, window)
        for g in (0, w["Hkv"] - 1):
            _group_bwd_check(dq, dk, dv, w["q"], w["k"], w["v"], do, M, g, rep, w["scale"], (a, z),
                             f"varlen seq {s} window {window}")


def test_bsr_workload_one_kv_group():
    # the BSR workload (B=2, S=16384, H=32 / Hkv=8, causal inside the routed blocks) in full on
    # the GPU; the oracle differentiates kv head 5 of batch 1 with its four query heads
    w = workloads.bsr_16384()
    P = bfa.plan_bsr(_cuda(w["block_indptr"]), _cuda(w["block_indices"]), w["S"], w["S"], causal=True)
    do = workloads.randn_bf16(tuple(w["q"].shape), 4444)
    qc, kc, vc, dc = w["q"].cuda(), w["k"].cuda(), w["v"].cuda(), do.cuda()
    out, lse = bfa.fwd(P, qc, kc, vc)
    dq, dk, dv = bfa.bwd(P, qc, kc, vc, out, dc, lse)
    torch.cuda.synchronize()
    P.device_status()
    b, g = 1, 5
    M = om.bsr_dense(w["block_indptr"][b:b + 1, g:g + 1], w["block_indices"], w["S"], w["S"], 128, 128,
                     causal=True)[0, 0]
    _group_bwd_check(dq[b].cpu(), dk[b].cpu(), dv[b].cpu(), w["q"][b], w["k"][b], w["v"][b], do[b], M, g,
                     w["H"] // w["Hkv"], w["scale"], (0, w["S"]), "bsr")


class _two_pass:
    """Backward in the two-pass (bitwise reproducible) form inside the block."""

    def __enter__(self):
        bfa.set_bwd_deterministic(True)

    def __exit__(self, *exc):
        bfa.set_bwd_deterministic(False)


@pytest.mark.parametrize("case", ["dense_ragged_gqa", "varlen_window", "varlen_single_row_tiles",
                                  "varlen_cross_full_tiles"])
def test_fused_and_two_pass_forms_agree(case):
    # D = 128: the fused pass (default) and the two-pass form both match the
    # oracle; dK and dV are made by the same products in the same order in both
    # forms (bit-identical); dQ differs only by the order of its fp32 sums.  The
    # packed cases put other sequences' tokens in the rows past a sequence's last
    # key tile: the fused pass sums dQ over every key row of a tile, so those rows
    # must not count (one valid query and one valid key make a full diagonal tile;
    # non-causal cross lengths make full tiles that run past their keys).
    D = 128
    if case == "dense_ragged_gqa":
        rng = np.random.default_rng(5)
        B, H, Hkv, Sq, Sk = 2, 4, 2, 300, 389
        M = rng.random((Sq, Sk)) < 0.4
        M[:, :3] = True
        P = bfa.plan_dense(_cuda(M))
        q = workloads.randn_bf16((B, Sq, H, D), 51)
        k = workloads.randn_bf16((B, Sk, Hkv, D), 52)
        v = workloads.randn_bf16((B, Sk, Hkv, D), 53)
        do = workloads.randn_bf16((B, Sq, H, D), 54)
        rq, rk, rv = ob.attention_bwd_bshd(q, k, v, do, lambda b, h: M, None)
    else:
        H, Hkv = 4, 2
        if case == "varlen_cross_full_tiles":
            cq = np.array([0, 100, 357, 400], dtype=np.int32)
            ck = np.array([0, 150, 389, 529], dtype=np.int32)
            # one block id for every token: each query attends all keys of its sequence
            ids = dict(q_blk=_cuda(np.zeros(cq[-1], np.int32)), k_blk=_cuda(np.zeros(ck[-1], np.int32)))
            P = bfa.plan_blockids(**ids, cu_seqlens_q=_cuda(cq), cu_seqlens_k=_cuda(ck), max_q=512, max_k=512)
            M = om.varlen_dense(cq, ck, False, -1)
        else:
            cq = ck = (np.array([0, 130, 515, 772, 836], dtype=np.int32) if case == "varlen_window"
                       else np.array([0, 1, 130, 259], dtype=np.int32))
            W = 200 if case == "varlen_window" else -1
            P = bfa.plan_blockids(cu_seqlens_q=_cuda(cq), cu_seqlens_k=_cuda(ck), max_q=512, max_k=512,
                                  window_left=W)
            M = om.varlen_dense(cq, ck, True, W)
        Tq, Tk = int(cq[-1]), int(ck[-1])
        q = workloads.randn_bf16((Tq, H, D), 61)
        k = workloads.randn_bf16((Tk, Hkv, D), 62)
        v = workloads.randn_bf16((Tk, Hkv, D), 63)
        do = workloads.randn_bf16((Tq, H, D), 64)
        rq, rk, rv = ob.attention_bwd_thd(q, k, v, do, M)
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    out, lse = bfa.fwd(P, qc, kc, vc)
    fused = bfa.bwd(P, qc, kc, vc, out, dc, lse)
    with _two_pass():
        two = bfa.bwd(P, qc, kc, vc, out, dc, lse)
    torch.cuda.synchronize()
    P.device_status()
    for grads in (fused, two):
        _close(grads[0], rq, "dq")
        _close(grads[1], rk, "dk")
        _close(grads[2], rv, "dv")
    assert torch.equal(fused[1], two[1]) and torch.equal(fused[2], two[2])
    dq_diff = (fused[0].float() - two[0].float()).abs().max().item()
    assert dq_diff <= 2 ** -7 * two[0].float().abs().max().item() + 1e-3


def test_two_pass_form_is_bitwise_reproducible():
    # the deterministic form repeats itself bit for bit; the fused form repeats
    # dK and dV bit for bit (its dQ sums may come in another order)
    B, H, Hkv, N, D = 1, 4, 2, 640, 128
    M = np.tril(np.ones((N, N), dtype=bool))
    P = bfa.plan_dense(_cuda(M))
    q, k, v, do = (workloads.randn_bf16(s, 70 + i).cuda() for i, s in
                   enumerate([(B, N, H, D), (B, N, Hkv, D), (B, N, Hkv, D), (B, N, H, D)]))
    out, lse = bfa.fwd(P, q, k, v)
    with _two_pass():
        a = bfa.bwd(P, q, k, v, out, do, lse)
        b = bfa.bwd(P, q, k, v, out, do, lse)
    f1 = bfa.bwd(P, q, k, v, out, do, lse)
    f2 = bfa.bwd(P, q, k, v, out, do, lse)
    torch.cuda.synchronize()
    P.device_status()
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert torch.equal(f1[1], f2[1]) and torch.equal(f1[2], f2[2])


@pytest.mark.parametrize("qb,kb,G,causal,D,form", [
    (16, 128, 8, False, 128, "fused"), (32, 64, 4, True, 128, "fused"), (32, 64, 4, True, 128, "two_pass"),
    (16, 128, 8, True, 64, "two_pass"),
])
def test_bsr_packed_backward(qb, kb, G, causal, D, form):
    # GQA-packed plans: a tile's rows are positions x every head of a kv head; the
    # gradients against the oracle per head, dK / dV summing the group's heads
    from test_gpu_plan import _routing, _valid_bits
    B, Hkv, Sq, Skv = 2, 2, 300, 520
    H = Hkv * G
    nqb, nkb = -(-Sq // qb), -(-Skv // kb)
    indptr, indices = _routing(B, Hkv, nqb, nkb, 900 + qb + G)
    kvb = _valid_bits(B, Skv, 13)
    P = bfa.plan_bsr_packed(_cuda(indptr), _cuda(indices), Sq, Skv, G, qb, kb, causal=causal,
                            kv_valid_bits=_cuda(kvb.view(np.int32)))
    M = om.block_bits_dense(om.bsr_to_block_bits(indptr, indices, nkb), Sq, Skv, qb, kb, causal=causal,
                            kv_valid_bits=kvb)
    q = workloads.randn_bf16((B, Sq, H, D), 81)
    k = workloads.randn_bf16((B, Skv, Hkv, D), 82)
    v = workloads.randn_bf16((B, Skv, Hkv, D), 83)
    do = workloads.randn_bf16((B, Sq, H, D), 84)
    if form == "two_pass":
        with _two_pass():
            _run_bshd(P, q, k, v, do, lambda b, h: M[b, h // G])
    else:
        _run_bshd(P, q, k, v, do, lambda b, h: M[b, h // G])
