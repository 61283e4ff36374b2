"""Dense boolean attention masks, True = attend, built from each mask form.

Oracle (test infrastructure only).  Every builder returns plain NumPy bool
arrays; nothing is tiled, packed or fused here.

Readings of the pages that these builders fix (each is also listed in the
design notes):

* block id of a token = inclusive running count of ``att_masks`` ones up to and
  including the token; tokens before the first 1 have id 0
  (opentau ``make_att_block_ids``: a 1 starts a new block, a 0 extends the current one).
* cross-attention key columns are prepended with block id INT32_MIN and their own
  padding mask, and they are still gated by the query's padding
  (opentau module docstring and ``make_att_block_ids`` parameters).
* causal is top-left aligned, ``kv_idx <= q_idx``
  (tensorplay omni_attention, "Block masks", the ``causal`` predicate).
* sliding window keeps keys with ``0 <= q_idx - kv_idx < W``
  (tensorplay omni_attention, "Block masks", the ``window`` predicate, where the
  printed example limits every query to its own key and the three before it,
  written ``q_idx - kv_idx < 4``).
* varlen: sequences packed along the token axis, delimited by ``cu_seqlens``
  starting at 0; positions are local to each sequence and keys of another
  sequence are never attended (tensorplay varlen, "Packed layout").
* BSR: query block ``i`` of head group ``(b, hkv)`` attends the KV blocks listed
  in ``block_indices[block_indptr[b, hkv, i] : block_indptr[b, hkv, i + 1]]``;
  ``mask_type="causal"`` further applies ``kv_idx <= q_idx`` on absolute
  positions inside the selected blocks (flashinfer ``block_sparse_attention``,
  parameters ``block_indptr``, ``block_indices``, ``mask_type``).
"""

from __future__ import annotations

import numpy as np

INT32_MIN = np.iinfo(np.int32).min


# --------------------------------------------------------------------------
# block-id form (opentau.policies.flash_attn_cuda)
# --------------------------------------------------------------------------

def make_att_block_ids(pad_masks, att_masks, n_cross_att_tokens=None, cross_att_pad_masks=None):
    """Compact block-id representation of a block-causal mask.

    Follows opentau ``make_att_block_ids``: returns ``(q_blk, k_blk, q_valid,
    k_valid)``; ``q_blk`` int32 (B, N) is the inclusive running count of
    ``att_masks`` ones, ``k_blk`` is the same ids with ``n_cross_att_tokens``
    columns of INT32_MIN prepended, ``q_valid = pad_masks`` and ``k_valid`` is
    ``cross_att_pad_masks`` followed by ``pad_masks``.
    """
    pad = np.asarray(pad_masks).astype(bool)
    att = np.asarray(att_masks).astype(np.int64)
    if pad.shape != att.shape or pad.ndim != 2:
        raise ValueError("pad_masks and att_masks must both be (B, N)")
    ids = np.cumsum(att != 0, axis=1).astype(np.int32)
    q_blk = ids
    q_valid = pad.copy()
    if n_cross_att_tokens is None:
        if cross_att_pad_masks is not None:
            raise ValueError("cross_att_pad_masks given without n_cross_att_tokens")
        return q_blk, ids.copy(), q_valid, pad.copy()
    if cross_att_pad_masks is None:
        raise ValueError("cross_att_pad_masks is required when n_cross_att_tokens is set")
    cpad = np.asarray(cross_att_pad_masks).astype(bool)
    B = pad.shape[0]
    if cpad.shape != (B, n_cross_att_tokens):
        raise ValueError("cross_att_pad_masks must be (B, n_cross_att_tokens)")
    cross_ids = np.full((B, n_cross_att_tokens), INT32_MIN, dtype=np.int32)
    k_blk = np.concatenate([cross_ids, ids], axis=1)
    k_valid = np.concatenate([cpad, pad], axis=1)
    return q_blk, k_blk, q_valid, k_valid


def blockid_dense(q_blk, k_blk, q_valid, k_valid):
    """attend(i, j) = q_valid[i] & k_valid[j] & (k_blk[j] <= q_blk[i]), per batch.

    The reconstruction rule stated for opentau ``make_att_block_ids`` /
    ``flash_attn_blockmask``.  Inputs (B, Sq) and (B, Sk); returns (B, Sq, Sk).
    The comparison is done in int64 so INT32_MIN needs no special case.
    """
    qb = np.asarray(q_blk).astype(np.int64)
    kb = np.asarray(k_blk).astype(np.int64)
    qv = np.asarray(q_valid).astype(bool)
    kv = np.asarray(k_valid).astype(bool)
    return qv[:, :, None] & kv[:, None, :] & (kb[:, None, :] <= qb[:, :, None])


def positional_dense(Sq, Sk, causal=True, window=-1):
    """Position predicate on one sequence: causal ``j <= i`` and optional window.

    ``window < 0`` disables the window ((-1, -1) disables it on the tensorplay
    varlen page); otherwise a key is kept iff ``0 <= i - j < window`` (the
    omni_attention ``window`` predicate with ``causal``).  ``causal=False`` with
    no window is the allow-everything ``noop_mask``.
    """
    i = np.arange(Sq)[:, None]
    j = np.arange(Sk)[None, :]
    m = np.ones((Sq, Sk), dtype=bool)
    if causal:
        m &= j <= i
    if window is not None and window >= 0:
        m &= (0 <= i - j) & (i - j < window)
    return m


def varlen_dense(cu_seqlens_q, cu_seqlens_k, causal=True, window=-1, q_blk=None, k_blk=None,
                 q_valid=None, k_valid=None):
    """Block-diagonal mask over packed sequences (tensorplay varlen, "Packed layout").

    Sequence ``s`` owns query rows ``cu_q[s]:cu_q[s+1]`` and key rows
    ``cu_k[s]:cu_k[s+1]``; inside the block the predicate uses positions local to
    the sequence (causal / window as in ``positional_dense``) or, when per-token
    block ids are given (indexed by packed token), the block-id rule.
    Returns (total_q, total_k).
    """
    cq = np.asarray(cu_seqlens_q, dtype=np.int64)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64)
    if cq.ndim != 1 or cq.shape != ck.shape or cq[0] != 0 or ck[0] != 0:
        raise ValueError("cu_seqlens must be 1-D, equal length, starting at 0")
    if np.any(np.diff(cq) < 0) or np.any(np.diff(ck) < 0):
        raise ValueError("cu_seqlens must be non-decreasing")
    M = np.zeros((int(cq[-1]), int(ck[-1])), dtype=bool)
    for s in range(len(cq) - 1):
        q0, q1, k0, k1 = int(cq[s]), int(cq[s + 1]), int(ck[s]), int(ck[s + 1])
        if q_blk is not None:
            qb = np.asarray(q_blk)[q0:q1][None]
            kb = np.asarray(k_blk)[k0:k1][None]
            qv = np.ones_like(qb, dtype=bool) if q_valid is None else np.asarray(q_valid)[q0:q1][None]
            kv = np.ones_like(kb, dtype=bool) if k_valid is None else np.asarray(k_valid)[k0:k1][None]
            blk = blockid_dense(qb, kb, qv, kv)[0]
        else:
            blk = positional_dense(q1 - q0, k1 - k0, causal=causal, window=window)
            if q_valid is not None:
                blk &= np.asarray(q_valid)[q0:q1].astype(bool)[:, None]
            if k_valid is not None:
                blk &= np.asarray(k_valid)[k0:k1].astype(bool)[None, :]
        M[q0:q1, k0:k1] = blk
    return M


def bsr_dense(block_indptr, block_indices, Sq, Skv, q_block_size, kv_block_size, causal=False):
    """Expand BSR routing into (B, Hkv, Sq, Skv) bool (flashinfer block_sparse_attention).

    ``block_indptr`` is (B, Hkv, ceil(Sq/q_block_size) + 1) with absolute offsets
    into ``block_indices``; each listed id selects a ``kv_block_size``-wide block of
    keys for the ``q_block_size`` query rows of that BSR row.  With ``causal`` the
    selected blocks are further restricted to ``kv_idx <= q_idx`` (``mask_type``).
    """
    indptr = np.asarray(block_indptr, dtype=np.int64)
    idx = np.asarray(block_indices, dtype=np.int64)
    B, Hkv, nrows1 = indptr.shape
    nqb = -(-Sq // q_block_size)
    if nrows1 != nqb + 1:
        raise ValueError("block_indptr last dim must be ceil(Sq/q_block_size)+1")
    M = np.zeros((B, Hkv, Sq, Skv), dtype=bool)
    for b in range(B):
        for h in range(Hkv):
            for r in range(nqb):
                q0, q1 = r * q_block_size, min(Sq, (r + 1) * q_block_size)
                for kb in idx[indptr[b, h, r]:indptr[b, h, r + 1]]:
                    k0, k1 = int(kb) * kv_block_size, min(Skv, (int(kb) + 1) * kv_block_size)
                    M[b, h, q0:q1, k0:k1] = True
    if causal:
        M &= positional_dense(Sq, Skv, causal=True)[None, None]
    return M


def block_bits_dense(block_bits, Sq, Skv, q_block_size, kv_block_size, causal=False, kv_valid_bits=None):
    """Expand an exact-block bitmap into (B, Hkv, Sq, Skv) bool (flashinfer
    block_sparse_attention, ``sparse_format="bitmask"`` with ``exact_block_bits``).

    Reading: ``block_bits`` is (B, Hkv, ceil(Sq/q_block_size), ceil(nkb/32)) uint32;
    bit ``j`` of word ``w`` in row ``i`` selects KV block ``32 w + j`` for query block
    ``i`` (least significant bit first).  ``kv_valid_bits`` (B, ceil(Skv/32)) uint32
    marks valid key tokens the same way (``kv_valid_bits``); invalid keys are never
    attended.  ``causal`` applies ``kv_idx <= q_idx`` (``mask_type``).
    """
    bits = np.asarray(block_bits, dtype=np.uint32)
    B, H, nqb, _ = bits.shape
    nkb = -(-Skv // kv_block_size)
    sel = np.unpackbits(bits.view(np.uint8), axis=-1, bitorder="little").astype(bool)[..., :nkb]
    rows = np.arange(Sq) // q_block_size
    cols = np.arange(Skv) // kv_block_size
    M = sel[:, :, rows][:, :, :, cols]
    if causal:
        M &= positional_dense(Sq, Skv, causal=True)[None, None]
    if kv_valid_bits is not None:
        kv = np.unpackbits(np.asarray(kv_valid_bits, dtype=np.uint32).view(np.uint8), axis=-1,
                           bitorder="little").astype(bool)[:, :Skv]
        M &= kv[:, None, None, :]
    return M


def gqa_packed_rows(M, heads_per_kv):
    """Rows of one (batch, kv head) mask in GQA-packed order (flashinfer
    block_sparse_attention, ``q_block_size``: one physical query tile holds the
    query tokens of a BSR row for every query head that shares the kv head, which
    is why the page asks ``q_block_size * Hq / Hkv`` to be a multiple of 8).

    ``M`` is the (Sq, Skv) mask of the kv head.  The result has Sq * heads_per_kv
    rows; row ``t`` is query position ``t // heads_per_kv`` of the group's query
    head ``t % heads_per_kv``, and every head of the group attends with the kv
    head's routing, so row ``t`` is ``M[t // heads_per_kv]``.
    """
    M = np.asarray(M, dtype=bool)
    return np.repeat(M, int(heads_per_kv), axis=0)


def bsr_to_block_bits(block_indptr, block_indices, n_kv_blocks):
    """The exact-block bitmap of BSR routing (same selection, bitmask layout)."""
    indptr = np.asarray(block_indptr, dtype=np.int64)
    idx = np.asarray(block_indices, dtype=np.int64)
    B, H, n1 = indptr.shape
    words = -(-n_kv_blocks // 32)
    out = np.zeros((B, H, n1 - 1, words), dtype=np.uint32)
    for b in range(B):
        for h in range(H):
            for r in range(n1 - 1):
                for kb in idx[indptr[b, h, r]:indptr[b, h, r + 1]]:
                    out[b, h, r, kb // 32] |= np.uint32(1) << np.uint32(kb % 32)
    return out


def bsr_is_canonical(block_indptr, block_indices, n_kv_blocks):
    """Canonical BSR rows: offsets non-decreasing and inside the index array, and
    every row's ids strictly increasing inside [0, n_kv_blocks)
    (flashinfer block_sparse_attention: BSR inputs are inspected "to validate
    canonical rows")."""
    indptr = np.asarray(block_indptr, dtype=np.int64)
    idx = np.asarray(block_indices, dtype=np.int64)
    n = idx.shape[0]
    for row in indptr.reshape(-1, indptr.shape[-1]):
        if np.any(np.diff(row) < 0) or row[0] < 0 or row[-1] > n:
            return False
        for r in range(len(row) - 1):
            ids = idx[row[r]:row[r + 1]]
            if ids.size and (ids.min() < 0 or ids.max() >= n_kv_blocks or np.any(np.diff(ids) <= 0)):
                return False
    return True


# --------------------------------------------------------------------------
# position-term predicates: OR of ANDs of band and box constraints
# --------------------------------------------------------------------------

def term(diag_lo=None, diag_hi=None, q_lo=None, q_hi=None, k_lo=None, k_hi=None):
    """One conjunction: diag_lo <= i - j <= diag_hi, q_lo <= i < q_hi, k_lo <= j < k_hi
    (None = unbounded).  ``causal`` is term(diag_lo=0); a past window of W keys is
    term(diag_lo=0, diag_hi=W - 1); global query rows are term(q_hi=G)."""
    return dict(diag_lo=diag_lo, diag_hi=diag_hi, q_lo=q_lo, q_hi=q_hi, k_lo=k_lo, k_hi=k_hi)


def predicate_dense(terms, Sq, Sk):
    """attend(i, j) = OR over ``terms`` of their constraints, positions local to the
    sequence; an empty list attends nothing.  Returns (Sq, Sk) bool."""
    i = np.arange(Sq)[:, None]
    j = np.arange(Sk)[None, :]
    M = np.zeros((Sq, Sk), dtype=bool)
    for t in terms:
        m = np.ones((Sq, Sk), dtype=bool)
        if t.get("diag_lo") is not None:
            m &= (i - j) >= t["diag_lo"]
        if t.get("diag_hi") is not None:
            m &= (i - j) <= t["diag_hi"]
        if t.get("q_lo") is not None:
            m &= i >= t["q_lo"]
        if t.get("q_hi") is not None:
            m &= i < t["q_hi"]
        if t.get("k_lo") is not None:
            m &= j >= t["k_lo"]
        if t.get("k_hi") is not None:
            m &= j < t["k_hi"]
        M |= m
    return M


# --------------------------------------------------------------------------
# predicate algebra (tensorplay.nn.attention.omni_attention, "Block masks")
# --------------------------------------------------------------------------

def causal(b, h, q_idx, kv_idx):
    """``q_idx >= kv_idx``."""
    return q_idx >= kv_idx


def window(W):
    """Predicate ``q_idx - kv_idx < W`` (combine with ``causal`` for a past window)."""
    def _w(b, h, q_idx, kv_idx):
        return (q_idx - kv_idx) < W
    return _w


def noop_mask(b, h, q_idx, kv_idx):
    """Allow-everything predicate."""
    return np.ones(np.broadcast(q_idx, kv_idx).shape, dtype=bool)


def and_masks(*mods):
    """Intersection of predicates."""
    def _and(b, h, q_idx, kv_idx):
        out = np.ones(np.broadcast(q_idx, kv_idx).shape, dtype=bool)
        for m in mods:
            out = out & m(b, h, q_idx, kv_idx)
        return out
    return _and


def or_masks(*mods):
    """Union of predicates."""
    def _or(b, h, q_idx, kv_idx):
        out = np.zeros(np.broadcast(q_idx, kv_idx).shape, dtype=bool)
        for m in mods:
            out = out | m(b, h, q_idx, kv_idx)
        return out
    return _or


def create_mask(mod, B, H, Q_LEN, KV_LEN):
    """Materialise a predicate into a dense (B, H, Q_LEN, KV_LEN) bool mask."""
    out = np.zeros((B, H, Q_LEN, KV_LEN), dtype=bool)
    qi = np.arange(Q_LEN)[:, None]
    ki = np.arange(KV_LEN)[None, :]
    for b in range(B):
        for h in range(H):
            out[b, h] = np.broadcast_to(mod(b, h, qi, ki), (Q_LEN, KV_LEN))
    return out
