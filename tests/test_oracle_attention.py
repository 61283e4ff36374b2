"""Pins for the oracle's masked attention (CPU only).

The oracle is checked against per-element brute force, torch's CPU
``scaled_dot_product_attention`` in float64 on the special cases that reduce to
it (all-True mask, causal), and closed forms.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import masks as om


def _brute(q, k, v, M, scale):
    Sq, D = q.shape
    Sk = k.shape[0]
    O = np.zeros((Sq, v.shape[1]))
    L = np.zeros(Sq)
    for i in range(Sq):
        s = [scale * sum(q[i, d] * k[j, d] for d in range(D)) for j in range(Sk)]
        att = [j for j in range(Sk) if M[i, j]]
        if not att:
            O[i] = 0.0
            L[i] = -math.inf
            continue
        mx = max(s[j] for j in att)
        w = {j: math.exp(s[j] - mx) for j in att}
        tot = sum(w.values())
        for d in range(v.shape[1]):
            O[i, d] = sum(w[j] * v[j, d] for j in att) / tot
        L[i] = mx + math.log(tot)
    return O, L


@pytest.mark.parametrize("seed", range(5))
def test_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    Sq, Sk, D = 9, 13, 4
    q, k, v = rng.standard_normal((Sq, D)), rng.standard_normal((Sk, D)), rng.standard_normal((Sk, 5))
    M = rng.random((Sq, Sk)) < 0.5
    M[3] = False                         # a fully masked row
    scale = 0.7
    O, L = oa.masked_attention(q, k, v, M, scale)
    Ob, Lb = _brute(q, k, v, M, scale)
    np.testing.assert_allclose(O, Ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(np.isinf(L), np.isinf(Lb))
    fin = np.isfinite(Lb)
    np.testing.assert_allclose(L[fin], Lb[fin], rtol=1e-12, atol=1e-12)


def _sdpa64(q, k, v, is_causal=False):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), is_causal=is_causal)[0, 0].numpy()


def test_all_true_equals_unmasked_sdpa():
    rng = np.random.default_rng(3)
    Sq, Sk, D = 37, 41, 16
    q, k, v = (rng.standard_normal((n, D)) for n in (Sq, Sk, Sk))
    O, L = oa.masked_attention(q, k, v, np.ones((Sq, Sk), bool))
    np.testing.assert_allclose(O, _sdpa64(q, k, v), rtol=1e-10, atol=1e-12)
    # LSE against its definition computed by a library log-sum-exp
    S = (q @ k.T) / math.sqrt(D)
    np.testing.assert_allclose(L, torch.logsumexp(torch.from_numpy(S), dim=1).numpy(), rtol=1e-12)


def test_causal_equals_sdpa_is_causal():
    rng = np.random.default_rng(4)
    N, D = 50, 8
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    O, _ = oa.masked_attention(q, k, v, om.positional_dense(N, N, causal=True))
    np.testing.assert_allclose(O, _sdpa64(q, k, v, is_causal=True), rtol=1e-10, atol=1e-12)


def test_gqa_head_mapping_against_repeated_kv():
    rng = np.random.default_rng(5)
    B, S, H, Hkv, D = 2, 12, 6, 2, 4
    q = rng.standard_normal((B, S, H, D))
    k = rng.standard_normal((B, S, Hkv, D))
    v = rng.standard_normal((B, S, Hkv, D))
    Os, Ls = oa.attention_bshd(q, k, v, lambda b, h: np.ones((S, S), bool))
    kr = np.repeat(k, H // Hkv, axis=2)      # head h reads kv head h // (H // Hkv)
    vr = np.repeat(v, H // Hkv, axis=2)
    for b in range(B):
        for h in range(H):
            ref = _sdpa64(q[b, :, h], kr[b, :, h], vr[b, :, h])
            np.testing.assert_allclose(Os[(b, h)], ref, rtol=1e-10, atol=1e-12)
    with pytest.raises(ValueError):
        oa.kv_head(0, 5, 2)


def test_closed_forms():
    rng = np.random.default_rng(6)
    Sq, Sk, D = 20, 30, 8
    M = rng.random((Sq, Sk)) < 0.3
    M[0] = False
    M[1] = False
    M[1, 7] = True                                    # a single attended key
    k, v = rng.standard_normal((Sk, D)), rng.standard_normal((Sk, D))
    # Q = 0: uniform weights over the attended keys, LSE = log(count)
    O, L = oa.masked_attention(np.zeros((Sq, D)), k, v, M)
    for i in range(Sq):
        n = M[i].sum()
        if n == 0:
            assert np.all(O[i] == 0) and L[i] == -np.inf
        else:
            np.testing.assert_allclose(O[i], v[M[i]].mean(axis=0), rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(L[i], math.log(n), rtol=1e-12, atol=1e-14)
    # V constant: output constant on rows with an attended key
    q = rng.standard_normal((Sq, D))
    O, _ = oa.masked_attention(q, k, np.full((Sk, D), 2.5), M)
    assert np.all(O[M.any(1)] == pytest.approx(2.5, abs=1e-12))
    # single attended key: output = that value row, LSE = scale * q.k
    O, L = oa.masked_attention(q, k, v, M, scale=0.3)
    np.testing.assert_allclose(O[1], v[7], rtol=1e-12)
    np.testing.assert_allclose(L[1], 0.3 * q[1] @ k[7], rtol=1e-12)


def test_fully_masked_rows_are_zero_and_minus_inf():
    rng = np.random.default_rng(8)
    O, L = oa.masked_attention(rng.standard_normal((5, 4)), rng.standard_normal((6, 4)),
                               rng.standard_normal((6, 4)), np.zeros((5, 6), bool))
    assert np.all(O == 0.0) and np.all(L == -np.inf)


def test_default_scale_and_chunking():
    rng = np.random.default_rng(9)
    Sq, Sk, D = 23, 17, 16
    q, k, v = (rng.standard_normal((n, D)) for n in (Sq, Sk, Sk))
    M = rng.random((Sq, Sk)) < 0.6
    O1, L1 = oa.masked_attention(q, k, v, M)
    O2, L2 = oa.masked_attention(q, k, v, M, scale=1 / math.sqrt(D), chunk=4)
    np.testing.assert_allclose(O1, O2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(L1[np.isfinite(L1)], L2[np.isfinite(L2)], rtol=1e-13)


def test_bf16_inputs_upcast_exactly():
    g = torch.Generator().manual_seed(0)
    q = torch.randn(6, 8, generator=g).to(torch.bfloat16)
    k = torch.randn(7, 8, generator=g).to(torch.bfloat16)
    v = torch.randn(7, 8, generator=g).to(torch.bfloat16)
    M = np.ones((6, 7), bool)
    O, _ = oa.masked_attention(q, k, v, M)
    Od, _ = oa.masked_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), M)
    np.testing.assert_array_equal(O, Od)


def test_thd_matches_per_sequence():
    rng = np.random.default_rng(10)
    cu = np.array([0, 5, 16], dtype=np.int32)
    H, Hkv, D = 4, 2, 8
    q = rng.standard_normal((16, H, D))
    k = rng.standard_normal((16, Hkv, D))
    v = rng.standard_normal((16, Hkv, D))
    M = om.varlen_dense(cu, cu, causal=True)
    Os, Ls = oa.attention_thd(q, k, v, M)
    for h in range(H):
        g = h // (H // Hkv)
        for s in range(2):
            a, b = cu[s], cu[s + 1]
            ref = _sdpa64(q[a:b, h], k[a:b, g], v[a:b, g], is_causal=True)
            np.testing.assert_allclose(Os[h][a:b], ref, rtol=1e-10, atol=1e-12)
