"""Gradients of masked softmax attention, float64, one head at a time.

Oracle (test infrastructure only).

The pages ship a forward and a backward (BinFlash runs the backward as two
passes, dK/dV over key blocks and dQ over query blocks, and its usage example
back-propagates ``out.sum()`` into q, k and v; opentau fuses both directions;
tensorplay varlen returns the log-sum-exp so that the backward can use it again).  What the backward computes is the gradient of the
forward's definition (``oracle.attention``) with respect to q, k and v, for an
upstream gradient dO of the output.  Written out (the softmax Jacobian):

    S  = scale * Q K^T, masked entries -inf          P = softmax_rows(S)
    dV = P^T dO
    dP = dO V^T
    dS = P * (dP - D),   D_i = sum_j P_ij dP_ij  (= dO_i . O_i)
    dQ = scale * dS K
    dK = scale * dS^T Q

Masked pairs have P = 0 and so contribute nothing; a row that attends nothing
has P = 0 everywhere (output 0, the forward's reading) and gets dQ = 0.  Under
GQA a key/value head's gradient is the sum over the query heads that read it.
Rows are processed in chunks only to bound memory.
"""

from __future__ import annotations

import numpy as np

from .attention import _f64, default_scale, kv_head


def softmax_probs(q, k, mask, scale):
    """P (Sq, Sk) of one head: row softmax of the scaled, masked scores (0 where masked)."""
    S = scale * (q @ k.T)
    S = np.where(mask, S, -np.inf)
    any_row = mask.any(axis=1)
    m = np.where(any_row, S.max(axis=1, initial=-np.inf), 0.0)
    E = np.where(mask, np.exp(S - m[:, None]), 0.0)
    l = E.sum(axis=1)
    return E / np.where(any_row, l, 1.0)[:, None]


def masked_attention_bwd(q, k, v, mask, do, scale=None, chunk=512):
    """One head: q (Sq, D), k (Sk, D), v (Sk, Dv), mask (Sq, Sk) bool, do (Sq, Dv).

    Returns (dQ (Sq, D), dK (Sk, D), dV (Sk, Dv), Dvec (Sq,)) in float64, where
    Dvec_i = sum_j P_ij dP_ij.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    mask = np.asarray(mask, dtype=bool)
    Sq, D = q.shape
    if scale is None:
        scale = default_scale(D)
    dQ = np.zeros_like(q)
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    Dvec = np.zeros((Sq,), dtype=np.float64)
    for r0 in range(0, Sq, chunk):
        r1 = min(Sq, r0 + chunk)
        P = softmax_probs(q[r0:r1], k, mask[r0:r1], scale)
        dP = do[r0:r1] @ v.T
        Dr = (P * dP).sum(axis=1)
        dS = P * (dP - Dr[:, None])
        dV += P.T @ do[r0:r1]
        dQ[r0:r1] = scale * (dS @ k)
        dK += scale * (dS.T @ q[r0:r1])
        Dvec[r0:r1] = Dr
    return dQ, dK, dV, Dvec


def attention_bwd_bshd(q, k, v, do, mask_for, scale=None):
    """Batched BSHD gradients: q, do (B, Sq, H, D); k, v (B, Sk, Hkv, D).

    ``mask_for(b, h)`` returns the (Sq, Sk) bool mask of query head ``h`` in batch
    ``b``.  Returns dQ (B, Sq, H, D), dK and dV (B, Sk, Hkv, D) in float64; the kv
    gradients sum over the query heads of each GQA group.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Sq, H, D = q.shape
    Hkv = k.shape[2]
    dQ = np.zeros_like(q)
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            g = kv_head(h, H, Hkv)
            dq, dk, dv, _ = masked_attention_bwd(q[b, :, h], k[b, :, g], v[b, :, g],
                                                 np.asarray(mask_for(b, h), dtype=bool), do[b, :, h], scale)
            dQ[b, :, h] = dq
            dK[b, :, g] += dk
            dV[b, :, g] += dv
    return dQ, dK, dV


def attention_bwd_thd(q, k, v, do, mask, scale=None):
    """Packed THD gradients: q, do (Tq, H, D); k, v (Tk, Hkv, D); mask (Tq, Tk) shared by heads."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    Tq, H, D = q.shape
    Hkv = k.shape[1]
    M = np.asarray(mask, dtype=bool)
    dQ = np.zeros_like(q)
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    for h in range(H):
        g = kv_head(h, H, Hkv)
        dq, dk, dv, _ = masked_attention_bwd(q[:, h], k[:, g], v[:, g], M, do[:, h], scale)
        dQ[:, h] = dq
        dK[:, g] += dk
        dV[:, g] += dv
    return dQ, dK, dV
