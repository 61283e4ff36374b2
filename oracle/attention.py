"""Masked softmax attention with log-sum-exp, float64, one head at a time.

Oracle (test infrastructure only).

Definition restated from the pages:

* output = softmax(scale * Q K^T + mask) V with a boolean mask, True = attend
  (BinFlash "Inputs": mask is (N, N) bool, True = attend; opentau
  ``flash_attn_blockmask``), masked scores are -inf before the softmax;
* without an explicit ``scale`` the scores are multiplied by D^(-1/2) (BinFlash "Inputs" ``sm_scale``; tensorplay varlen
  keyword ``scale``; flashinfer ``sm_scale``);
* LSE is the natural-log log-sum-exp of the scaled attended scores of a row
  (tensorplay omni_attention, "Outputs", ``return_lse``);
* GQA: query head ``h`` reads key/value head ``h // (H // Hkv)``, ``H % Hkv == 0``
  (opentau ``flash_attn_blockmask`` parameter ``k``; contiguous grouping is the
  reading taken where the pages only state divisibility);
* a row with no attended key has output 0 and LSE -inf (the pages are silent;
  this is the reading taken).

Rows are processed in chunks only to bound memory: each chunk is the same
formula on a subset of rows, nothing is reordered or fused.
"""

from __future__ import annotations

import math

import numpy as np


def _f64(x):
    """Exact upcast of a bf16/fp32 torch tensor or array to float64 NumPy."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def default_scale(D):
    """1 / sqrt(D)."""
    return 1.0 / math.sqrt(D)


def masked_attention(q, k, v, mask, scale=None, chunk=512):
    """One head: q (Sq, D), k (Sk, D), v (Sk, Dv), mask (Sq, Sk) bool.

    Returns (O (Sq, Dv) float64, LSE (Sq,) float64).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    mask = np.asarray(mask, dtype=bool)
    Sq, D = q.shape
    Sk = k.shape[0]
    if mask.shape != (Sq, Sk):
        raise ValueError(f"mask shape {mask.shape} != {(Sq, Sk)}")
    if scale is None:
        scale = default_scale(D)
    O = np.zeros((Sq, v.shape[1]), dtype=np.float64)
    L = np.full((Sq,), -np.inf, dtype=np.float64)
    for r0 in range(0, Sq, chunk):
        r1 = min(Sq, r0 + chunk)
        S = scale * (q[r0:r1] @ k.T)
        M = mask[r0:r1]
        S = np.where(M, S, -np.inf)
        any_row = M.any(axis=1)
        m = np.where(any_row, S.max(axis=1, initial=-np.inf), 0.0)
        P = np.where(M, np.exp(S - m[:, None]), 0.0)
        l = P.sum(axis=1)
        safe_l = np.where(any_row, l, 1.0)
        O[r0:r1] = np.where(any_row[:, None], (P @ v) / safe_l[:, None], 0.0)
        L[r0:r1] = np.where(any_row, m + np.log(safe_l), -np.inf)
    return O, L


def kv_head(h, H, Hkv):
    """Query head -> key/value head under contiguous GQA grouping."""
    if H % Hkv != 0:
        raise ValueError("H must be a multiple of Hkv")
    return h // (H // Hkv)


def attention_bshd(q, k, v, mask_for, scale=None, heads=None, rows=None):
    """Batched BSHD attention: q (B, Sq, H, D), k/v (B, Sk, Hkv, D).

    ``mask_for(b, h)`` returns the (Sq, Sk) bool mask of query head ``h`` in batch
    ``b``.  ``heads`` optionally restricts the (b, h) pairs computed; ``rows``
    optionally restricts the query rows (an index array) -- each output row only
    depends on its own query row, so a subset is the same formula on fewer rows.
    Returns dicts keyed by (b, h): O (n_rows, D) and LSE (n_rows,).
    """
    B, Sq, H, D = q.shape
    Hkv = k.shape[2]
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    outO, outL = {}, {}
    for (b, h) in pairs:
        g = kv_head(h, H, Hkv)
        M = np.asarray(mask_for(b, h), dtype=bool)
        qq = q[b, :, h, :]
        if rows is not None:
            qq = qq[rows]
            M = M[rows]
        O, L = masked_attention(qq, k[b, :, g, :], v[b, :, g, :], M, scale)
        outO[(b, h)] = O
        outL[(b, h)] = L
    return outO, outL


def attention_thd(q, k, v, mask, scale=None, heads=None, rows=None):
    """Packed THD attention: q (Tq, H, D), k/v (Tk, Hkv, D), mask (Tq, Tk) shared by heads.

    Returns dicts keyed by h.
    """
    Tq, H, D = q.shape
    Hkv = k.shape[1]
    hs = heads if heads is not None else range(H)
    outO, outL = {}, {}
    M = np.asarray(mask, dtype=bool)
    for h in hs:
        g = kv_head(h, H, Hkv)
        qq = q[:, h, :]
        MM = M
        if rows is not None:
            qq = qq[rows]
            MM = M[rows]
        O, L = masked_attention(qq, k[:, g, :], v[:, g, :], MM, scale)
        outO[h] = O
        outL[h] = L
    return outO, outL
