"""Pins of oracle.backward: gradients of the forward definition.

Independent checks: central finite differences of the forward oracle (float64),
torch autograd in float64 on the CPU, closed forms, and the identity
D_i = dO_i . O_i against the forward oracle."""

import numpy as np
import pytest

from oracle import attention as oa
from oracle import backward as ob

torch = pytest.importorskip("torch")


def _case(seed, Sq=5, Sk=7, D=3, Dv=4, dead_row=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((Sq, D))
    k = rng.standard_normal((Sk, D))
    v = rng.standard_normal((Sk, Dv))
    mask = rng.random((Sq, Sk)) < 0.6
    mask[0, :] = False if dead_row else mask[0, :]
    mask[1, :] = True
    g = rng.standard_normal((Sq, Dv))  # upstream gradient of sum(O * g)
    return q, k, v, mask, g


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_matches_central_finite_differences(seed):
    q, k, v, mask, g = _case(seed)
    scale = 0.7
    dQ, dK, dV, _ = ob.masked_attention_bwd(q, k, v, mask, g, scale)

    def loss(q_, k_, v_):
        O, _ = oa.masked_attention(q_, k_, v_, mask, scale)
        return float((O * g).sum())

    h = 1e-6
    for X, dX, which in ((q, dQ, 0), (k, dK, 1), (v, dV, 2)):
        num = np.zeros_like(X)
        for idx in np.ndindex(*X.shape):
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += h
            Xm[idx] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which] = Xp
            args_m[which] = Xm
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        assert np.allclose(dX, num, atol=1e-7, rtol=1e-6), (which, np.abs(dX - num).max())


def test_matches_torch_autograd_float64_with_gqa():
    rng = np.random.default_rng(7)
    B, Sq, Sk, H, Hkv, D = 2, 9, 11, 4, 2, 5
    q = rng.standard_normal((B, Sq, H, D))
    k = rng.standard_normal((B, Sk, Hkv, D))
    v = rng.standard_normal((B, Sk, Hkv, D))
    do = rng.standard_normal((B, Sq, H, D))
    masks = rng.random((B, H, Sq, Sk)) < 0.5
    masks[:, :, :, 0] = True  # every row attends something
    scale = 0.45
    dQ, dK, dV = ob.attention_bwd_bshd(q, k, v, do, lambda b, h: masks[b, h], scale)

    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k, requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    rep = H // Hkv
    kk = tk.repeat_interleave(rep, dim=2)  # (B, Sk, H, D)
    vv = tv.repeat_interleave(rep, dim=2)
    S = scale * torch.einsum("bqhd,bkhd->bhqk", tq, kk)
    S = S.masked_fill(~torch.tensor(masks), float("-inf"))
    O = torch.einsum("bhqk,bkhd->bqhd", torch.softmax(S, dim=-1), vv)
    (O * torch.tensor(do)).sum().backward()
    assert np.allclose(dQ, tq.grad.numpy(), atol=1e-12)
    assert np.allclose(dK, tk.grad.numpy(), atol=1e-12)
    assert np.allclose(dV, tv.grad.numpy(), atol=1e-12)


def test_constant_values_give_zero_query_and_key_gradients():
    q, k, v, mask, g = _case(3, dead_row=False)
    v[:] = 2.5
    dQ, dK, dV, _ = ob.masked_attention_bwd(q, k, v, mask, g, 0.9)
    assert np.abs(dQ).max() < 1e-13 and np.abs(dK).max() < 1e-13
    P = ob.softmax_probs(q, k, mask, 0.9)
    assert np.allclose(dV, P.T @ g, atol=1e-14)


def test_single_attended_key_per_row():
    rng = np.random.default_rng(4)
    Sq, Sk, D = 6, 6, 4
    q, k, v = (rng.standard_normal((n, D)) for n in (Sq, Sk, Sk))
    g = rng.standard_normal((Sq, D))
    mask = np.zeros((Sq, Sk), dtype=bool)
    cols = rng.integers(0, Sk, Sq)
    mask[np.arange(Sq), cols] = True
    dQ, dK, dV, _ = ob.masked_attention_bwd(q, k, v, mask, g, 0.5)
    assert np.abs(dQ).max() < 1e-14 and np.abs(dK).max() < 1e-14
    want = np.zeros_like(v)
    np.add.at(want, cols, g)
    assert np.allclose(dV, want, atol=1e-14)


def test_dvec_is_dout_dot_out_and_dead_rows_are_inert():
    q, k, v, mask, g = _case(5)
    O, _ = oa.masked_attention(q, k, v, mask, 0.8)
    dQ, dK, dV, Dvec = ob.masked_attention_bwd(q, k, v, mask, g, 0.8)
    assert np.allclose(Dvec, (g * O).sum(axis=1), atol=1e-13)
    assert np.all(dQ[0] == 0.0) and Dvec[0] == 0.0
    # the dead row contributes nothing: removing it leaves dK and dV unchanged
    _, dK2, dV2, _ = ob.masked_attention_bwd(q[1:], k, v, mask[1:], g[1:], 0.8)
    assert np.allclose(dK, dK2, atol=1e-14) and np.allclose(dV, dV2, atol=1e-14)


def test_thd_matches_per_sequence_blocks():
    rng = np.random.default_rng(9)
    H, Hkv, D = 2, 1, 4
    lens = [3, 5]
    T = sum(lens)
    q, do = rng.standard_normal((T, H, D)), rng.standard_normal((T, H, D))
    k, v = rng.standard_normal((T, Hkv, D)), rng.standard_normal((T, Hkv, D))
    M = np.zeros((T, T), dtype=bool)
    o = 0
    for L in lens:
        M[o:o + L, o:o + L] = np.tril(np.ones((L, L), dtype=bool))
        o += L
    dQ, dK, dV = ob.attention_bwd_thd(q, k, v, do, M, 0.6)
    o = 0
    for L in lens:
        sl = slice(o, o + L)
        dq, dk, dv = ob.attention_bwd_bshd(q[None, sl], k[None, sl], v[None, sl], do[None, sl],
                                           lambda b, h: np.tril(np.ones((L, L), dtype=bool)), 0.6)
        assert np.allclose(dQ[sl], dq[0]) and np.allclose(dK[sl], dk[0]) and np.allclose(dV[sl], dv[0])
        o += L
