"""GPU forward parity: outputs and LSE against the float64 oracle.

Tolerance (bf16 N(0, 1) inputs, fp32 accumulation): output max-abs 1e-2, LSE
max-abs 1e-3, and -inf LSE exactly where a row attends no key.  Small workloads
are compared on every output; the full-size workloads on sampled rows of
sampled heads, in the same call the bench times.
"""

import math

import numpy as np
import pytest
import torch

import workloads
from helpers import check_bshd, compare_rows, peaked_bound, sample_rows
from oracle import attention as oa
from oracle import masks as om

pytestmark = pytest.mark.gpu

bfa = pytest.importorskip("mask_skipping_flashattention_b200")


def _cuda(x):
    return torch.as_tensor(np.ascontiguousarray(x)).cuda()


def _rand(shape, seed):
    return workloads.randn_bf16(shape, seed)


# ---------------------------------------------------------------- tiny / block-causal
@pytest.mark.parametrize("form", ["dense", "blockids"])
def test_tiny_blockcausal(form):
    w = workloads.tiny_blockcausal()
    ids_ref = om.make_att_block_ids(w["pad_masks"], w["att_masks"])
    M = om.blockid_dense(*ids_ref)[0]
    if form == "dense":
        P = bfa.plan_dense(_cuda(M))
    else:
        P = bfa.plan_blockids(*bfa.make_att_block_ids(_cuda(w["pad_masks"]), _cuda(w["att_masks"])))
    out, lse = bfa.fwd(P, w["q"].cuda(), w["k"].cuda(), w["v"].cuda(), scale=w["scale"])
    torch.cuda.synchronize()
    P.device_status()
    pairs = [(0, 0), (0, 1)]
    check_bshd(out.cpu(), lse.cpu(), w["q"], w["k"], w["v"], lambda b, h: M, w["scale"], pairs, where=form)
    # padded query rows attend nothing: output 0 and LSE -inf
    assert torch.all(out[0, 240:] == 0) and torch.all(torch.isneginf(lse[0, :, 240:]))


def test_blockcausal_gqa_cross_columns():
    w = workloads.blockcausal_gqa()
    ids = bfa.make_att_block_ids(_cuda(w["pad_masks"]), _cuda(w["att_masks"]), w["n_cross"],
                                 _cuda(w["cross_pad_masks"]))
    P = bfa.plan_blockids(*ids)
    out, lse = bfa.fwd(P, w["q"].cuda(), w["k"].cuda(), w["v"].cuda())
    torch.cuda.synchronize()
    dense = om.blockid_dense(*om.make_att_block_ids(w["pad_masks"], w["att_masks"], w["n_cross"],
                                                    w["cross_pad_masks"]))
    pairs = [(b, h) for b in range(w["B"]) for h in range(w["H"])]
    check_bshd(out.cpu(), lse.cpu(), w["q"], w["k"], w["v"], lambda b, h: dense[b], None, pairs, where="cfg3")


@pytest.mark.parametrize("seed", range(2))
def test_blockids_unsorted_and_sorted_key_tiles(seed):
    # key ids in arbitrary order on some key tiles (every key compared) and
    # non-decreasing on others (one binary search per row): both forms of the
    # block-id mask against the dense mask the ids define
    rng = np.random.default_rng(70 + seed)
    B, Sq, Sk, H, D = 2, 300, 520, 2, 64
    qb = np.sort(rng.integers(0, 9, size=(B, Sq)), axis=1).astype(np.int32)
    kb = rng.integers(-2, 10, size=(B, Sk)).astype(np.int32)
    kb[:, 128:384] = np.sort(kb[:, 128:384], axis=1)      # key tiles 1 and 2 in order
    kb[:, :7] = np.iinfo(np.int32).min
    qv = rng.random((B, Sq)) < 0.9
    kv = rng.random((B, Sk)) < 0.85
    P = bfa.plan_blockids(_cuda(qb), _cuda(kb), _cuda(qv), _cuda(kv))
    dense = om.blockid_dense(qb, kb, qv, kv)
    q = _rand((B, Sq, H, D), 81 + seed)
    k = _rand((B, Sk, H, D), 83 + seed)
    v = _rand((B, Sk, H, D), 85 + seed)
    out, lse = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    pairs = [(b, h) for b in range(B) for h in range(H)]
    check_bshd(out.cpu(), lse.cpu(), q, k, v, lambda b, h: dense[b], None, pairs, where="unsorted ids")


# ---------------------------------------------------------------- causal 8192
def test_causal_8192_reduced_heads_all_rows():
    w = workloads.causal_8192(B=1, H=2)
    P = bfa.plan_dense(w["mask"].cuda())
    out, lse = bfa.fwd(P, w["q"].cuda(), w["k"].cuda(), w["v"].cuda())
    torch.cuda.synchronize()
    M = w["mask"].numpy()
    check_bshd(out.cpu(), lse.cpu(), w["q"], w["k"], w["v"], lambda b, h: M, None, [(0, 0), (0, 1)],
               where="causal full rows")


def test_causal_8192_full_size_sampled():
    """The bench workload (B=4, H=32, N=8192) in the bench's launch; sampled rows."""
    w = workloads.causal_8192()
    mask = w["mask"].cuda()
    q, k, v = w["q"].cuda(), w["k"].cuda(), w["v"].cuda()
    P = bfa.plan_dense(mask)
    out, lse = bfa.fwd(P, q, k, v)
    torch.cuda.synchronize()
    P.device_status()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    rows = sample_rows(8192, 48, 7, must=(0, 1, 127, 128, 4095, 8191))
    M = w["mask"].numpy()
    pairs = [(0, 0), (1, 17), (2, 31), (3, 5)]
    check_bshd(out.cpu(), lse.cpu(), w["q"], w["k"], w["v"], lambda b, h: M, None, pairs, rows=rows,
               where="causal full size")


# ---------------------------------------------------------------- varlen
def _varlen_check(out, lse, w, window, heads, rows_per_seq=None):
    cu = w["cu_seqlens"]
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        M = om.positional_dense(b - a, b - a, causal=True, window=window)
        rows = None if rows_per_seq is None else sample_rows(b - a, rows_per_seq, s, must=(0, b - a - 1))
        for h in heads:
            g = h // (w["H"] // w["Hkv"])
            qq = w["q"][a:b, h]
            MM = M
            if rows is not None:
                qq, MM = qq[rows], M[rows]
            O, L = oa.masked_attention(qq, w["k"][a:b, g], w["v"][a:b, g], MM)
            og = out[a:b, h] if rows is None else out[a:b, h][rows]
            lg = lse[h, a:b] if rows is None else lse[h, a:b][rows]
            compare_rows(og, lg, O, L, where=f"varlen seq {s} head {h} window {window}")


@pytest.mark.parametrize("window", [-1, 1024])
def test_varlen_workload(window):
    w = workloads.varlen_16()
    cu = _cuda(w["cu_seqlens"])
    P = bfa.plan_blockids(cu_seqlens_q=cu, cu_seqlens_k=cu, max_q=w["max_len"], max_k=w["max_len"],
                          window_left=window)
    out, lse = bfa.fwd(P, w["q"].cuda(), w["k"].cuda(), w["v"].cuda())
    torch.cuda.synchronize()
    _varlen_check(out.cpu(), lse.cpu(), w, window, heads=[0, 13, 31], rows_per_seq=96)


def test_varlen_small_all_rows():
    rng = np.random.default_rng(2)
    lens = [1, 127, 128, 129, 300, 0, 5]
    cu = np.zeros(len(lens) + 1, np.int32)
    cu[1:] = np.cumsum(lens)
    T, H, Hkv, D = int(cu[-1]), 4, 2, 64
    w = dict(cu_seqlens=cu, H=H, Hkv=Hkv, q=_rand((T, H, D), 11), k=_rand((T, Hkv, D), 12),
             v=_rand((T, Hkv, D), 13))
    for window in (-1, 3):
        P = bfa.plan_blockids(cu_seqlens_q=_cuda(cu), cu_seqlens_k=_cuda(cu), max_q=300, max_k=300,
                              window_left=window)
        out, lse = bfa.fwd(P, w["q"].cuda(), w["k"].cuda(), w["v"].cuda())
        torch.cuda.synchronize()
        _varlen_check(out.cpu(), lse.cpu(), w, window, heads=range(H))


# ---------------------------------------------------------------- BSR and dense union
def test_bsr_workload_sampled():
    w = workloads.bsr_16384()
    P = bfa.plan_bsr(_cuda(w["block_indptr"]), _cuda(w["block_indices"]), w["S"], w["S"], causal=True)
    out, lse = bfa.fwd(P, w["q"].cuda(), w["k"].cuda(), w["v"].cuda())
    torch.cuda.synchronize()
    rows = sample_rows(w["S"], 40, 3, must=(0, 127, 128, 16383))
    pairs = [(0, 0), (0, 9), (1, 31)]
    out_c, lse_c = out.cpu(), lse.cpu()
    for (b, h) in pairs:
        g = h // 4
        M = om.bsr_dense(w["block_indptr"][b:b + 1, g:g + 1], w["block_indices"], w["S"], w["S"], 128, 128,
                         causal=True)[0, 0]
        check_bshd(out_c, lse_c, w["q"], w["k"], w["v"], lambda bb, hh: M, None, [(b, h)], rows=rows,
                   where="bsr")


def test_union_workload_sampled():
    w = workloads.union_16384()
    P = bfa.plan_dense(w["mask"].cuda())
    out, lse = bfa.fwd(P, w["q"].cuda(), w["k"].cuda(), w["v"].cuda())
    torch.cuda.synchronize()
    M = w["mask"].numpy()
    rows = sample_rows(w["S"], 40, 4, must=(0, 63, 64, 2047, 16383))
    check_bshd(out.cpu(), lse.cpu(), w["q"], w["k"], w["v"], lambda b, h: M, None, [(0, 0), (1, 30)],
               rows=rows, where="union")


# ---------------------------------------------------------------- edge cases
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Sq,Sk", [(1, 1), (77, 300), (300, 77), (256, 256), (129, 1000)])
def test_dense_ragged_gqa(D, Sq, Sk):
    rng = np.random.default_rng(Sq * 13 + Sk + D)
    B, H, Hkv = 2, 4, 2
    M = rng.random((Sq, Sk)) < 0.6
    M[0] = False                      # a fully masked row
    if Sq > 3:
        M[3] = False
        M[3, Sk - 1] = True           # a single attended key, at the edge
    q, k, v = _rand((B, Sq, H, D), 1), _rand((B, Sk, Hkv, D), 2), _rand((B, Sk, Hkv, D), 3)
    P = bfa.plan_dense(_cuda(M))
    out, lse = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    pairs = [(b, h) for b in range(B) for h in range(H)]
    check_bshd(out.cpu(), lse.cpu(), q, k, v, lambda b, h: M, None, pairs, where=f"ragged D={D}")
    assert torch.all(out[:, 0] == 0) and torch.all(torch.isneginf(lse[:, :, 0]))
    if Sq > 3:   # the single attended key is copied exactly
        assert torch.equal(out[:, 3].cpu(), v[:, Sk - 1].repeat_interleave(H // Hkv, dim=1))


@pytest.mark.parametrize("D", [64, 128])
def test_peaked_softmax_within_bf16_bound(D):
    """scale = 0.3 makes the softmax far peakier than D^-0.5; compare with the
    worst-case bf16 rounding bound instead of the default-scale tolerance."""
    rng = np.random.default_rng(D)
    B, H, Hkv, Sq, Sk = 2, 4, 2, 300, 517
    M = rng.random((Sq, Sk)) < 0.6
    q, k, v = _rand((B, Sq, H, D), 31), _rand((B, Sk, Hkv, D), 32), _rand((B, Sk, Hkv, D), 33)
    P = bfa.plan_dense(_cuda(M))
    out, lse = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda(), scale=0.3)
    torch.cuda.synchronize()
    Os, Ls = oa.attention_bshd(q, k, v, lambda b, h: M, 0.3)
    for (b, h), O in Os.items():
        g = h // (H // Hkv)
        vmax = float(v[b, :, g].float().abs().max())
        err = np.abs(out[b, :, h].float().cpu().numpy() - O)
        assert np.all(err <= peaked_bound(O, vmax)), f"b={b} h={h} max err {err.max():.3e}"
        np.testing.assert_allclose(lse[b, h].cpu().numpy(), Ls[(b, h)], atol=1e-3)


def test_all_true_and_empty_masks():
    B, H, S, D = 1, 2, 384, 128
    q, k, v = _rand((B, S, H, D), 4), _rand((B, S, H, D), 5), _rand((B, S, H, D), 6)
    for M in (np.ones((S, S), bool), np.zeros((S, S), bool)):
        P = bfa.plan_dense(_cuda(M))
        out, lse = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda())
        torch.cuda.synchronize()
        check_bshd(out.cpu(), lse.cpu(), q, k, v, lambda b, h: M, None, [(0, 0), (0, 1)], where="all/none")
    assert torch.all(out == 0)


def test_bhsd_strides_and_out_buffer():
    B, H, S, D = 2, 3, 200, 128
    qh = _rand((B, H, S, D), 7).cuda()
    kh = _rand((B, H, S, D), 8).cuda()
    vh = _rand((B, H, S, D), 9).cuda()
    q, k, v = (t.transpose(1, 2) for t in (qh, kh, vh))      # BSHD views of BHSD storage
    M = om.positional_dense(S, S, causal=True)
    P = bfa.plan_dense(_cuda(M))
    big = torch.zeros((B, S, H, 2 * D), dtype=torch.bfloat16, device="cuda")
    out = big[..., D:]
    bfa.fwd(P, q, k, v, out=out, return_lse=False)
    torch.cuda.synchronize()
    assert torch.all(big[..., :D] == 0)
    pairs = [(b, h) for b in range(B) for h in range(H)]
    check_bshd(out.cpu(), None, q.cpu(), k.cpu(), v.cpu(), lambda b, h: M, None, pairs, where="bhsd")


def test_default_scale_matches_explicit():
    B, H, S, D = 1, 1, 256, 64
    q, k, v = _rand((B, S, H, D), 21).cuda(), _rand((B, S, H, D), 22).cuda(), _rand((B, S, H, D), 23).cuda()
    P = bfa.plan_dense(_cuda(om.positional_dense(S, S)))
    o1, l1 = bfa.fwd(P, q, k, v)
    o2, l2 = bfa.fwd(P, q, k, v, scale=1.0 / math.sqrt(D))
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_error_paths():
    B, H, S, D = 1, 4, 128, 128
    q, k, v = _rand((B, S, H, D), 1).cuda(), _rand((B, S, 3, D), 2).cuda(), _rand((B, S, 3, D), 3).cuda()
    P = bfa.plan_dense(_cuda(np.ones((S, S), bool)))
    with pytest.raises(bfa.BfaError) as e:
        bfa.fwd(P, q, k, v)                                   # H % Hkv != 0
    assert e.value.status == "BFA_ERR_INVALID_ARG"
    q96 = torch.zeros((B, S, H, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bfa.BfaError) as e:
        bfa.fwd(P, q96, q96, q96)
    assert e.value.status == "BFA_ERR_UNSUPPORTED"
    qc = torch.zeros((B, S, H, D), dtype=torch.bfloat16)
    with pytest.raises(bfa.BfaError) as e:
        bfa.fwd(P, qc, qc, qc, out=torch.zeros_like(qc.cuda()))
    assert e.value.status == "BFA_ERR_NOT_DEVICE"
    Pb = bfa.plan_blockids(B=2, Sq=S, Sk=S)
    qq = torch.zeros((3, S, H, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bfa.BfaError) as e:
        bfa.fwd(Pb, qq, qq, qq)                               # batch mismatch
    assert e.value.status == "BFA_ERR_INVALID_ARG"


def test_bounded_wait_reports_timeout_and_context_survives():
    bfa.set_wait_timeout_ns(50_000_000)
    try:
        assert bfa.selftest_wait_timeout() == "BFA_ERR_TIMEOUT"
    finally:
        bfa.set_wait_timeout_ns(0)
    # the context is still usable
    test_default_scale_matches_explicit()


def test_max_jump_in_a_later_key_tile():
    """Scores of some key tiles far above the earlier ones: a row's running max
    grows by much more than 2^8 after its first tile, so the forward must move
    its reference max and rescale the O it has accumulated."""
    B, H, N, D = 1, 4, 1024, 128
    q, k, v = (_rand((B, N, H, D), 9300 + i) for i in range(3))
    k = k.float()
    k[:, 5 * 128:6 * 128] *= 12.0          # key tile 5: scores about 12 x larger
    k[:, 700:704] *= 20.0                  # and a few keys of tile 5 larger still
    k = k.to(torch.bfloat16)
    M = np.tril(np.ones((N, N), dtype=bool))
    P = bfa.plan_dense(_cuda(M))
    out, lse = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    P.device_status()
    check_bshd(out.cpu(), lse.cpu(), q, k, v, lambda b, h: M, None, [(0, h) for h in range(H)], where="max jump")


def test_forward_and_backward_give_up_on_a_short_wait_bound():
    """The kernels' own failure path: with the shortest loop-wait bound (1 us) the
    first wait of a block for its scores outlasts the bound (the copies of Q and K
    alone take longer), so blocks stop their work, drain the copies and products
    they issued, release tensor memory and report BFA_ERR_TIMEOUT through the plan
    (forward, fused backward, two-pass backward).  Afterwards the default bound
    gives oracle-exact results on the same plan."""
    B, H, N, D = 2, 8, 2048, 128
    M = np.tril(np.ones((N, N), dtype=bool))
    q, k, v = (_rand((B, N, H, D), 9100 + i) for i in range(3))
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    P = bfa.plan_dense(_cuda(M))
    bfa.set_wait_timeout_ns(1)  # clamped to the minimum, 1 us
    try:
        out, lse = bfa.fwd(P, qc, kc, vc)
        torch.cuda.synchronize()
        with pytest.raises(bfa.BfaError) as e:
            P.device_status()
        assert e.value.status == "BFA_ERR_TIMEOUT"
        dout = _rand((B, N, H, D), 9199).cuda()
        for deterministic in (False, True):  # the fused pass, then the two passes
            bfa.set_bwd_deterministic(deterministic)
            bfa.bwd(P, qc, kc, vc, out, dout, lse)
            torch.cuda.synchronize()
            with pytest.raises(bfa.BfaError) as e:
                P.device_status()
            assert e.value.status == "BFA_ERR_TIMEOUT"
    finally:
        bfa.set_wait_timeout_ns(0)
        bfa.set_bwd_deterministic(False)
    out, lse = bfa.fwd(P, qc, kc, vc)
    torch.cuda.synchronize()
    P.device_status()
    rows = sample_rows(N, 48, 5, must=(0, N - 1))
    check_bshd(out.cpu(), lse.cpu(), q, k, v, lambda b, h: M, None, [(0, 0), (1, H - 1)], rows=rows,
               where="after the timeout")


@pytest.mark.parametrize("qb,kb,causal", [(64, 32, True), (100, 192, False)])
def test_general_block_sparse_forward(qb, kb, causal):
    from test_gpu_plan import _routing, _valid_bits
    B, H, Hkv, Sq, Skv, D = 2, 4, 2, 300, 500, 128
    nqb, nkb = -(-Sq // qb), -(-Skv // kb)
    indptr, indices = _routing(B, Hkv, nqb, nkb, 77 + qb)
    kvb = _valid_bits(B, Skv, 5)
    P = bfa.plan_bsr(_cuda(indptr), _cuda(indices), Sq, Skv, qb, kb, causal=causal,
                     kv_valid_bits=_cuda(kvb.view(np.int32)))
    q, k, v = _rand((B, Sq, H, D), 41), _rand((B, Skv, Hkv, D), 42), _rand((B, Skv, Hkv, D), 43)
    out, lse = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    M = om.block_bits_dense(om.bsr_to_block_bits(indptr, indices, nkb), Sq, Skv, qb, kb, causal=causal,
                            kv_valid_bits=kvb)
    pairs = [(b, h) for b in range(B) for h in range(H)]
    check_bshd(out.cpu(), lse.cpu(), q, k, v, lambda b, h: M[b, h // (H // Hkv)], None, pairs, where="general bsr")


# ---------------------------------------------------------------- paged keys / values, seqused_k
def _paged_cache(lens, page_size, Hkv, D, seed):
    """Scatter per-sequence K/V into randomly placed pages; returns caches, table, gathered K/V."""
    rng = np.random.default_rng(seed)
    n_pages_seq = [-(-L // page_size) for L in lens]
    pages_per_seq = max(max(n_pages_seq), 1) + 1
    num_pages = sum(n_pages_seq) + 5
    perm = rng.permutation(num_pages)
    kc = _rand((num_pages, page_size, Hkv, D), seed + 1)
    vc = _rand((num_pages, page_size, Hkv, D), seed + 2)
    table = np.full((len(lens), pages_per_seq), -1, dtype=np.int32)
    ks, vs, pos = [], [], 0
    for s, L in enumerate(lens):
        pages = perm[pos:pos + n_pages_seq[s]]
        pos += n_pages_seq[s]
        table[s, :len(pages)] = pages
        rows_k = torch.cat([kc[int(p_)] for p_ in pages], dim=0)[:L] if len(pages) else kc[:0, 0]
        rows_v = torch.cat([vc[int(p_)] for p_ in pages], dim=0)[:L] if len(pages) else vc[:0, 0]
        ks.append(rows_k)
        vs.append(rows_v)
    return kc, vc, table, ks, vs


@pytest.mark.parametrize("page_size", [16, 64, 128, 256])
def test_paged_kv_varlen(page_size):
    lens = [100, 300, 129, 257, 1]
    H, Hkv, D = 4, 2, 128
    cu = np.zeros(len(lens) + 1, np.int32)
    cu[1:] = np.cumsum(lens)
    T = int(cu[-1])
    q = _rand((T, H, D), 61)
    kc, vc, table, ks, vs = _paged_cache(lens, page_size, Hkv, D, 70 + page_size)
    P = bfa.plan_blockids(cu_seqlens_q=_cuda(cu), cu_seqlens_k=_cuda(cu), max_q=max(lens), max_k=max(lens))
    out, lse = bfa.fwd_paged(P, q.cuda(), kc.cuda(), vc.cuda(), _cuda(table))
    torch.cuda.synchronize()
    P.device_status()
    for s, L in enumerate(lens):
        a, b = int(cu[s]), int(cu[s + 1])
        M = om.positional_dense(L, L, causal=True)
        for h in range(H):
            g = h // (H // Hkv)
            O, Ls = oa.masked_attention(q[a:b, h], ks[s][:, g], vs[s][:, g], M)
            compare_rows(out[a:b, h].cpu(), lse[h, a:b].cpu(), O, Ls, where=f"paged {page_size} seq {s} h {h}")


def test_paged_kv_batched_dense_plan():
    B, H, Hkv, S, D, page_size = 2, 2, 2, 300, 64, 32
    q = _rand((B, S, H, D), 81)
    kc, vc, table, ks, vs = _paged_cache([S] * B, page_size, Hkv, D, 90)
    M = om.positional_dense(S, S, causal=True)
    P = bfa.plan_dense(_cuda(M))
    out, lse = bfa.fwd_paged(P, q.cuda(), kc.cuda(), vc.cuda(), _cuda(table))
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(H):
            O, Ls = oa.masked_attention(q[b, :, h], ks[b][:, h], vs[b][:, h], M)
            compare_rows(out[b, :, h].cpu(), lse[b, h].cpu(), O, Ls, where=f"paged dense b {b} h {h}")


def test_seqused_k_bounds_the_keys():
    lens = [300, 200, 129]
    used = np.array([250, 0, 129], dtype=np.int32)       # a sequence with no usable key
    H, Hkv, D = 2, 1, 64
    cu = np.zeros(len(lens) + 1, np.int32)
    cu[1:] = np.cumsum(lens)
    T = int(cu[-1])
    q, k, v = _rand((T, H, D), 91), _rand((T, Hkv, D), 92), _rand((T, Hkv, D), 93)
    P = bfa.plan_blockids(cu_seqlens_q=_cuda(cu), cu_seqlens_k=_cuda(cu), seqused_k=_cuda(used), max_q=300,
                          max_k=300)
    out, lse = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    for s, L in enumerate(lens):
        a, b = int(cu[s]), int(cu[s + 1])
        M = om.positional_dense(L, L, causal=True)
        M[:, used[s]:] = False
        for h in range(H):
            O, Ls = oa.masked_attention(q[a:b, h], k[a:b, 0], v[a:b, 0], M)
            compare_rows(out[a:b, h].cpu(), lse[h, a:b].cpu(), O, Ls, where=f"seqused seq {s} h {h}")


@pytest.mark.parametrize("name", ["prefix_lm", "global64_window256", "two_bands"])
def test_predicate_forward(name):
    from test_gpu_plan import PRED_CASES
    terms = PRED_CASES[name]
    B, H, Hkv, Sq, Sk, D = 2, 4, 2, 700, 650, 128
    q, k, v = _rand((B, Sq, H, D), 51), _rand((B, Sk, Hkv, D), 52), _rand((B, Sk, Hkv, D), 53)
    P = bfa.plan_predicate(terms, B=B, Sq=Sq, Sk=Sk)
    out, lse = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    M = om.predicate_dense(terms, Sq, Sk)
    pairs = [(b, h) for b in range(B) for h in range(H)]
    check_bshd(out.cpu(), lse.cpu(), q, k, v, lambda b, h: M, None, pairs, where=name)


def test_predicate_union_workload_sampled():
    """The union workload's window and global tokens as terms (no dense mask), N=16384."""
    terms = [om.term(diag_lo=0, diag_hi=2047), om.term(q_hi=64), om.term(k_hi=64)]
    w = workloads.union_16384(with_qkv=True)
    P = bfa.plan_predicate(terms, B=w["B"], Sq=w["S"], Sk=w["S"])
    out, lse = bfa.fwd(P, w["q"].cuda(), w["k"].cuda(), w["v"].cuda())
    torch.cuda.synchronize()
    rows = sample_rows(w["S"], 32, 8, must=(0, 63, 64, 2047, 2048, 16383))
    M = om.predicate_dense(terms, w["S"], w["S"])
    check_bshd(out.cpu(), lse.cpu(), w["q"], w["k"], w["v"], lambda b, h: M, None, [(0, 3), (1, 17)], rows=rows,
               where="union terms")


def _near_far_inputs(B, S, H, Hkv, D, seed):
    """Even key tiles score about +6, odd ones about -6 (natural units) for every
    query; odd tiles carry values of 1e4, so their e^-12 weights still move the
    exact output by ~0.06 while the approximation drops them."""
    g = torch.Generator().manual_seed(seed)
    u = (torch.randint(0, 2, (D,), generator=g) * 2 - 1).float() * 0.73
    q = (u + 0.1 * torch.randn(B, S, H, D, generator=g)).to(torch.bfloat16)
    sign = torch.ones(S)
    for t in range(S // 128):
        if t % 2:
            sign[t * 128:(t + 1) * 128] = -1.0
    k = (sign[None, :, None, None] * u + 0.1 * torch.randn(B, S, Hkv, D, generator=g)).to(torch.bfloat16)
    v = torch.randn(B, S, Hkv, D, generator=g)
    v[:, sign < 0] = 1e4
    return q, k, v.to(torch.bfloat16), sign > 0


@pytest.mark.parametrize("H,Hkv", [(2, 2), (4, 2)])
def test_block_skipping_drops_far_tiles(H, Hkv):
    B, S, D = 1, 1024, 128
    q, k, v, near = _near_far_inputs(B, S, H, Hkv, D, 7)
    P = bfa.plan_dense(_cuda(np.ones((S, S), bool)))
    exact, lse_e = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda())
    approx, lse_a = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda(), softmax_threshold=8.0)
    torch.cuda.synchronize()
    full = np.ones((S, S), bool)
    near_only = np.broadcast_to(near.numpy()[None, :], (S, S))
    pairs = [(0, h) for h in range(H)]
    Of, _ = oa.attention_bshd(q, k, v, lambda b, h: full, None, heads=pairs)
    On, _ = oa.attention_bshd(q, k, v, lambda b, h: near_only, None, heads=pairs)
    assert max(np.abs(Of[p] - On[p]).max() for p in pairs) > 0.03   # the far tiles matter exactly
    check_bshd(exact.cpu(), lse_e.cpu(), q, k, v, lambda b, h: full, None, pairs, where="exact")
    check_bshd(approx.cpu(), None, q, k, v, lambda b, h: near_only, None, pairs, where="approx = near keys")
    # LSE moves by at most n_dropped * exp(-threshold)
    assert float((lse_a - lse_e).abs().max()) <= 512 * math.exp(-8.0) + 1e-3


def test_block_skipping_with_huge_threshold_is_exact():
    B, S, H, D = 1, 512, 2, 64
    q, k, v = _rand((B, S, H, D), 5), _rand((B, S, H, D), 6), _rand((B, S, H, D), 7)
    P = bfa.plan_dense(_cuda(om.positional_dense(S, S)))
    o1, l1 = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda())
    o2, l2 = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda(), softmax_threshold=1e9)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    with pytest.raises(bfa.BfaError):
        bfa.fwd(P, q.cuda(), k.cuda(), v.cuda(), softmax_threshold=-1.0)


# ---------------------------------------------------------------- GQA-packed BSR query tiles
@pytest.mark.parametrize("qb,kb,G,causal,D", [
    (16, 128, 8, False, 128), (16, 64, 8, True, 128), (32, 128, 4, True, 128), (64, 32, 2, False, 128),
    (16, 128, 8, True, 64),
])
def test_bsr_packed_forward(qb, kb, G, causal, D):
    # a tile holds 128 / G positions of every head of a kv head; outputs and LSE
    # against the oracle per head, and the unpacked plan of the same routing agrees
    from test_gpu_plan import _routing, _valid_bits
    B, Hkv, Sq, Skv = 2, 2, 300, 520
    H = Hkv * G
    nqb, nkb = -(-Sq // qb), -(-Skv // kb)
    indptr, indices = _routing(B, Hkv, nqb, nkb, 500 + qb + G)
    kvb = _valid_bits(B, Skv, 11)
    P = bfa.plan_bsr_packed(_cuda(indptr), _cuda(indices), Sq, Skv, G, qb, kb, causal=causal,
                            kv_valid_bits=_cuda(kvb.view(np.int32)))
    q, k, v = _rand((B, Sq, H, D), 61), _rand((B, Skv, Hkv, D), 62), _rand((B, Skv, Hkv, D), 63)
    out, lse = bfa.fwd(P, q.cuda(), k.cuda(), v.cuda())
    Pu = bfa.plan_bsr(_cuda(indptr), _cuda(indices), Sq, Skv, qb, kb, causal=causal,
                      kv_valid_bits=_cuda(kvb.view(np.int32)))
    out_u, lse_u = bfa.fwd(Pu, q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    P.device_status()
    M = om.block_bits_dense(om.bsr_to_block_bits(indptr, indices, nkb), Sq, Skv, qb, kb, causal=causal,
                            kv_valid_bits=kvb)
    pairs = [(b, h) for b in range(B) for h in range(H)]
    check_bshd(out.cpu(), lse.cpu(), q, k, v, lambda b, h: M[b, h // G], None, pairs, where="packed bsr")
    assert (out.float() - out_u.float()).abs().max().item() <= 2e-2
    fin = torch.isfinite(lse_u)
    assert torch.equal(fin, torch.isfinite(lse)) and (lse - lse_u)[fin].abs().max().item() <= 2e-3


def test_bsr_packed_plans_reject_other_head_counts():
    from test_gpu_plan import _routing
    B, Hkv, Sq, Skv, D, G = 1, 2, 256, 256, 128, 4
    indptr, indices = _routing(B, Hkv, Sq // 32, Skv // 128, 9)
    P = bfa.plan_bsr_packed(_cuda(indptr), _cuda(indices), Sq, Skv, G, 32, 128)
    k, v = _rand((B, Skv, Hkv, D), 2).cuda(), _rand((B, Skv, Hkv, D), 3).cuda()
    with pytest.raises(bfa.BfaError) as e:   # H / Hkv = 2 against the plan's 4
        bfa.fwd(P, _rand((B, Sq, 2 * Hkv, D), 1).cuda(), k, v)
    assert e.value.status == "BFA_ERR_INVALID_ARG"
    q = _rand((B, Sq, G * Hkv, D), 1).cuda()
    out, lse = bfa.fwd(P, q, k, v)
    q2 = _rand((B, Sq, 2 * Hkv, D), 4).cuda()
    with pytest.raises(bfa.BfaError) as e:
        bfa.bwd(P, q2, k, v, q2, q2, lse)
    assert e.value.status == "BFA_ERR_INVALID_ARG"


@pytest.mark.parametrize("page_size", [16, 128])
def test_bsr_packed_paged_and_approximate(page_size):
    # packed tiles with keys / values in a paged cache give the contiguous result bit
    # for bit, and the approximate mode with a threshold that drops nothing gives the
    # exact result bit for bit
    from test_gpu_plan import _routing
    B, Hkv, G, Sq, Skv, D, qb, kb = 2, 2, 4, 256, 384, 128, 32, 64
    H = Hkv * G
    indptr, indices = _routing(B, Hkv, -(-Sq // qb), -(-Skv // kb), 41)
    P = bfa.plan_bsr_packed(_cuda(indptr), _cuda(indices), Sq, Skv, G, qb, kb, causal=True)
    q = _rand((B, Sq, H, D), 91).cuda()
    kc, vc, table, ks, vs = _paged_cache([Skv] * B, page_size, Hkv, D, 95 + page_size)
    k, v = torch.stack(ks).cuda(), torch.stack(vs).cuda()
    o1, l1 = bfa.fwd(P, q, k, v)
    o2, l2 = bfa.fwd_paged(P, q, kc.cuda(), vc.cuda(), _cuda(table))
    o3, l3 = bfa.fwd(P, q, k, v, softmax_threshold=1e9)
    torch.cuda.synchronize()
    P.device_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(o1, o3) and torch.equal(l1, l3)
