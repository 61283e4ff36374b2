"""Mask-aware fused attention forward for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libbfa.so`` (``include/bfa.h``).  The
binding only marshals torch tensors into device pointers, sizes, strides and the
current CUDA stream; every step of the computation runs in the library's CUDA
kernels.  There is no CPU path: CPU tensors are rejected by the library.

    plan = plan_dense(mask)                      # (Sq, Sk) bool, True = attend
    out, lse = fwd(plan, q, k, v)                # q (B, Sq, H, D), k/v (B, Sk, Hkv, D)

Other mask sources: ``plan_blockids`` (opentau block ids, positions, varlen,
sliding window) and ``plan_bsr`` (BSR routing); ``make_att_block_ids`` builds
block ids from padding and block-opening flags.
"""

from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib
from ._lib import BfaError, PlanInfo

__all__ = ["Plan", "BfaError", "plan_dense", "plan_blockids", "plan_predicate", "plan_bsr", "plan_bsr_packed",
           "plan_block_bits",
           "fwd", "bwd", "fwd_paged",
           "make_att_block_ids",
           "is_available", "load_error", "set_wait_timeout_ns", "set_bwd_deterministic", "selftest_wait_timeout", "library_path"]

TILE = 128
KIND_NAMES = {1: "dense", 2: "blockids", 3: "positional", 4: "bsr", 5: "predicate"}
_I32_MIN, _I32_MAX = -(2 ** 31), 2 ** 31 - 1

library_path = _lib.LIB_PATH
_L = _lib.load()


def _stream(stream=None):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _u8(t):
    if t is None:
        return None
    if t.dtype == torch.bool:
        return t
    return (t != 0)


def is_available():
    """True if a B200-class device is present and the kernels load."""
    return bool(_L.bfa_is_available())


def load_error():
    """Message of the last failed library call on this thread, or None."""
    m = _L.bfa_last_error().decode(errors="replace")
    return m or None


def set_wait_timeout_ns(ns):
    _L.bfa_set_wait_timeout_ns(int(ns))


def set_bwd_deterministic(on=True):
    """Two-pass backward for every head dim (bitwise reproducible) when ``on``."""
    _L.bfa_set_bwd_deterministic(1 if on else 0)


def selftest_wait_timeout(stream=None):
    """Run the library's bounded-wait self test; returns the status name."""
    return _lib.STATUS.get(_L.bfa_selftest_wait_timeout(_stream(stream)))


class Plan:
    """A library-owned tile plan; freed when garbage collected or by ``destroy()``."""

    def __init__(self, handle, stream):
        self._h = handle
        self._stream = stream
        info = PlanInfo()
        _lib.check(_L.bfa_plan_get_info(self._h, ctypes.byref(info)))
        self.info = {f: getattr(info, f) for f, _ in PlanInfo._fields_}
        self.kind = KIND_NAMES[self.info["kind"]]

    @property
    def handle(self):
        if self._h is None:
            raise RuntimeError("plan was destroyed")
        return self._h

    def destroy(self):
        if self._h is not None:
            _L.bfa_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass

    def stats(self, stream=None):
        f, p, e = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _lib.check(_L.bfa_plan_stats(self.handle, ctypes.byref(f), ctypes.byref(p), ctypes.byref(e),
                                     _stream(stream)))
        return f.value, p.value, e.value

    def device_status(self, stream=None):
        """Raise BfaError(BFA_ERR_TIMEOUT) if a kernel using this plan hit its wait bound."""
        _lib.check(_L.bfa_plan_device_status(self.handle, _stream(stream)))

    def export_cols(self, stream=None):
        """Host copy of the transposed lists of the backward's key-tile pass:
        col_ptr, q_tile, tpart (-1 full, else the fine-word index), col_order."""
        n_full, n_part, _ = self.stats(stream)
        C = self.info["n_cols"]
        nnz = n_full + n_part
        col_ptr = np.zeros(C + 1, np.int32)
        q_tile = np.zeros(max(nnz, 1), np.int32)
        tpart = np.zeros(max(nnz, 1), np.int32)
        col_order = np.zeros(max(C, 1), np.int32)
        P = lambda a: a.ctypes.data_as(ctypes.c_void_p)
        _lib.check(_L.bfa_plan_export_cols(self.handle, P(col_ptr), P(q_tile), P(tpart), P(col_order),
                                           _stream(stream)))
        return dict(col_ptr=col_ptr, q_tile=q_tile[:nnz], tpart=tpart[:nnz], col_order=col_order[:C])

    def export(self, stream=None):
        """Host copy: row_ptr, kv_tile, partial, fine (packed-mask plans), order, classes, pairs."""
        n_full, n_part, _ = self.stats(stream)
        R = self.info["n_rows"]
        nnz = n_full + n_part
        row_ptr = np.zeros(R + 1, np.int32)
        kv_tile = np.zeros(max(nnz, 1), np.int32)
        partial = np.zeros(max(nnz, 1), np.uint8)
        fine = np.zeros((max(n_part, 1), TILE, 4), np.uint32) if self.info["packed_fine"] else None
        order = np.zeros(max(R, 1), np.int32)
        classes = np.zeros(max(self.info["grid_tiles"], 1), np.uint8)
        P = lambda a: a.ctypes.data_as(ctypes.c_void_p) if a is not None else None
        _lib.check(_L.bfa_plan_export(self.handle, P(row_ptr), P(kv_tile), P(partial), P(fine), P(order),
                                      P(classes), _stream(stream)))
        out = dict(row_ptr=row_ptr, kv_tile=kv_tile[:nnz], partial=partial[:nnz], order=order[:R],
                   classes=classes[:self.info["grid_tiles"]])
        n_pairs = self.info["n_pairs"]
        pair_row = np.zeros(max(n_pairs, 1), np.int32)
        pair_order = np.zeros(max(n_pairs, 1), np.int32)
        _lib.check(_L.bfa_plan_export_pairs(self.handle, P(pair_row), P(pair_order), _stream(stream)))
        out["pair_row"] = pair_row[:n_pairs]
        out["pair_order"] = pair_order[:n_pairs]
        if fine is not None:
            out["fine"] = fine[:n_part]
        return out


def make_att_block_ids(pad_masks, att_masks, n_cross_att_tokens=None, cross_att_pad_masks=None, stream=None):
    """(q_blk, k_blk, q_valid, k_valid) from padding and block-opening flags (opentau).

    pad_masks / att_masks: (B, N) bool or integer CUDA tensors; cross columns with
    block id INT32_MIN are prepended when ``n_cross_att_tokens`` is given.
    """
    pad = _u8(pad_masks).contiguous()
    att = _u8(att_masks).contiguous()
    B, N = pad.shape
    nc = int(n_cross_att_tokens or 0)
    cpad = _u8(cross_att_pad_masks).contiguous() if nc else None
    dev = pad.device
    q_blk = torch.empty((B, N), dtype=torch.int32, device=dev)
    k_blk = torch.empty((B, nc + N), dtype=torch.int32, device=dev)
    q_valid = torch.empty((B, N), dtype=torch.bool, device=dev)
    k_valid = torch.empty((B, nc + N), dtype=torch.bool, device=dev)
    _lib.check(_L.bfa_make_block_ids(_ptr(pad), _ptr(att), B, N, nc, _ptr(cpad), _ptr(q_blk), _ptr(k_blk),
                                     _ptr(q_valid), _ptr(k_valid), _stream(stream)))
    return q_blk, k_blk, q_valid, k_valid


def plan_dense(mask, stream=None):
    """Plan from a dense (Sq, Sk) bool CUDA mask (True = attend), shared by all batches/heads."""
    if mask.dim() != 2:
        raise ValueError("mask must be 2-D (Sq, Sk)")
    m = mask if mask.dtype in (torch.bool, torch.uint8) else (mask != 0)
    if m.stride(1) != 1:
        m = m.contiguous()
    h = ctypes.c_void_p()
    st = _stream(stream)
    _lib.check(_L.bfa_plan_dense(_ptr(m), m.stride(0), m.shape[0], m.shape[1], ctypes.byref(h), st))
    return Plan(h, st)


def plan_blockids(q_blk=None, k_blk=None, q_valid=None, k_valid=None, *, B=None, Sq=None, Sk=None,
                  cu_seqlens_q=None, cu_seqlens_k=None, seqused_k=None, max_q=0, max_k=0, window_left=-1,
                  stream=None):
    """Plan from block ids / validity (opentau) or, with ids None, from causal positions.

    Batched: ids (B, Sq) / (B, Sk).  Varlen: ids over packed tokens, ``cu_seqlens_*``
    int32 (B + 1,) starting at 0, ``max_q`` / ``max_k`` >= every sequence length.
    ``seqused_k`` int32 (B,) bounds the usable keys of each batch entry / sequence.
    ``window_left`` > 0 keeps keys with 0 <= q_pos - k_pos < window_left.
    """
    varlen = cu_seqlens_q is not None
    if varlen:
        B = cu_seqlens_q.numel() - 1
        Sq = Sk = 0
    elif q_blk is not None:
        B, Sq = q_blk.shape
        Sk = k_blk.shape[1]
    elif q_valid is not None:
        B, Sq = q_valid.shape
        Sk = k_valid.shape[1] if k_valid is not None else Sk
    for t in (q_blk, k_blk):
        if t is not None and t.dtype != torch.int32:
            raise TypeError("block ids must be int32")
    qv = _u8(q_valid).contiguous() if q_valid is not None else None
    kv = _u8(k_valid).contiguous() if k_valid is not None else None
    qb = q_blk.contiguous() if q_blk is not None else None
    kb = k_blk.contiguous() if k_blk is not None else None
    cq = cu_seqlens_q.to(torch.int32).contiguous() if varlen else None
    ck = (cu_seqlens_k if cu_seqlens_k is not None else cu_seqlens_q).to(torch.int32).contiguous() if varlen else None
    h = ctypes.c_void_p()
    st = _stream(stream)
    su = seqused_k.to(torch.int32).contiguous() if seqused_k is not None else None
    _lib.check(_L.bfa_plan_blockids(_ptr(qb), _ptr(kb), _ptr(qv), _ptr(kv), int(B), int(Sq or 0), int(Sk or 0),
                                    _ptr(cq), _ptr(ck), _ptr(su), int(max_q), int(max_k), int(window_left),
                                    ctypes.byref(h), st))
    return Plan(h, st)


def plan_predicate(terms, *, B=None, Sq=None, Sk=None, cu_seqlens_q=None, cu_seqlens_k=None, seqused_k=None,
                   max_q=0, max_k=0, stream=None):
    """Plan from position terms: attend(i, j) = OR over terms of
    diag_lo <= i - j <= diag_hi AND q_lo <= i < q_hi AND k_lo <= j < k_hi.

    ``terms``: list of dicts with those keys (missing / None = unbounded).  Layout
    as for ``plan_blockids`` (batched B, Sq, Sk or varlen cu_seqlens).
    """
    arr = (_lib.MaskTerm * max(len(terms), 1))()
    for n, t in enumerate(terms):
        get = lambda key, dflt: dflt if t.get(key) is None else int(t[key])
        arr[n] = _lib.MaskTerm(get("diag_lo", _I32_MIN), get("diag_hi", _I32_MAX), get("q_lo", _I32_MIN),
                               get("q_hi", _I32_MAX), get("k_lo", _I32_MIN), get("k_hi", _I32_MAX))
    varlen = cu_seqlens_q is not None
    if varlen:
        B = cu_seqlens_q.numel() - 1
        Sq = Sk = 0
    cq = cu_seqlens_q.to(torch.int32).contiguous() if varlen else None
    ck = (cu_seqlens_k if cu_seqlens_k is not None else cu_seqlens_q).to(torch.int32).contiguous() if varlen else None
    su = seqused_k.to(torch.int32).contiguous() if seqused_k is not None else None
    h = ctypes.c_void_p()
    st = _stream(stream)
    _lib.check(_L.bfa_plan_predicate(ctypes.cast(arr, ctypes.c_void_p), len(terms), int(B), int(Sq or 0),
                                     int(Sk or 0), _ptr(cq), _ptr(ck), _ptr(su), int(max_q), int(max_k),
                                     ctypes.byref(h), st))
    return Plan(h, st)


def plan_bsr(block_indptr, block_indices, Sq, Skv, q_block_size=TILE, kv_block_size=TILE, causal=False,
             kv_valid_bits=None, stream=None):
    """Plan from BSR routing: indptr (B, Hkv, ceil(Sq/q_block)+1) int32, indices int32.

    ``kv_valid_bits`` (B, ceil(Skv/32)) int32/uint32 marks valid key tokens, LSB first.
    """
    ip = block_indptr.to(torch.int32).contiguous()
    ix = block_indices.to(torch.int32).contiguous()
    kv = kv_valid_bits.contiguous() if kv_valid_bits is not None else None
    B, Hkv, _ = ip.shape
    h = ctypes.c_void_p()
    st = _stream(stream)
    _lib.check(_L.bfa_plan_bsr(_ptr(ip), _ptr(ix) if ix.numel() else None, ix.numel(), B, Hkv, int(Sq), int(Skv),
                               int(q_block_size), int(kv_block_size), 1 if causal else 0, _ptr(kv),
                               ctypes.byref(h), st))
    return Plan(h, st)


def plan_bsr_packed(block_indptr, block_indices, Sq, Skv, heads_per_kv, q_block_size=TILE, kv_block_size=TILE,
                    causal=False, kv_valid_bits=None, stream=None):
    """BSR plan with GQA-packed query tiles: each tile holds 128 / heads_per_kv query
    positions of all ``heads_per_kv`` query heads of a kv head (H = Hkv * heads_per_kv
    in the calls that use it, forward and backward)."""
    ip = block_indptr.to(torch.int32).contiguous()
    ix = block_indices.to(torch.int32).contiguous()
    kv = kv_valid_bits.contiguous() if kv_valid_bits is not None else None
    B, Hkv, _ = ip.shape
    h = ctypes.c_void_p()
    st = _stream(stream)
    _lib.check(_L.bfa_plan_bsr_packed(_ptr(ip), _ptr(ix) if ix.numel() else None, ix.numel(), B, Hkv,
                                      int(heads_per_kv), int(Sq), int(Skv), int(q_block_size), int(kv_block_size),
                                      1 if causal else 0, _ptr(kv), ctypes.byref(h), st))
    return Plan(h, st)


def plan_block_bits(exact_block_bits, Sq, Skv, q_block_size=TILE, kv_block_size=TILE, causal=False,
                    kv_valid_bits=None, stream=None):
    """Plan from an exact-block bitmap (B, Hkv, ceil(Sq/q_block), ceil(nkb/32)), LSB first."""
    bits = exact_block_bits.contiguous()
    kv = kv_valid_bits.contiguous() if kv_valid_bits is not None else None
    B, Hkv = bits.shape[:2]
    h = ctypes.c_void_p()
    st = _stream(stream)
    _lib.check(_L.bfa_plan_block_bits(_ptr(bits), B, Hkv, int(Sq), int(Skv), int(q_block_size), int(kv_block_size),
                                      1 if causal else 0, _ptr(kv), ctypes.byref(h), st))
    return Plan(h, st)


def _strides3(t):
    if t.dim() == 4:
        return (ctypes.c_int64 * 3)(t.stride(0), t.stride(1), t.stride(2))
    if t.dim() == 3:
        return (ctypes.c_int64 * 3)(0, t.stride(0), t.stride(1))
    raise ValueError("expected a 4-D (B, S, H, D) or 3-D (T, H, D) tensor")


def fwd(plan, q, k, v, scale=None, out=None, return_lse=True, lse=None, stream=None, softmax_threshold=None):
    """Masked attention forward; returns (out, lse or None).

    Batched q (B, Sq, H, D), k/v (B, Sk, Hkv, D); packed (varlen plans) q (Tq, H, D),
    k/v (Tk, Hkv, D).  bf16, last dim contiguous, D in {64, 128}.  A positive
    ``softmax_threshold`` turns on content-based block skipping (approximate).
    """
    for t in (q, k, v):
        if t.dtype != torch.bfloat16:
            raise TypeError("q, k, v must be bfloat16")
        if t.stride(-1) != 1:
            raise ValueError("the head dim of q, k, v must be contiguous")
    packed = q.dim() == 3
    if packed:
        B = plan.info["batch"]
        _, H, D = q.shape
        Hkv = k.shape[1]
        lse_shape = (H, q.shape[0])
    else:
        B, Sq, H, D = q.shape
        Hkv = k.shape[2]
        lse_shape = (B, H, Sq)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    if not return_lse:
        lse = None
    sc = float(scale) if scale is not None else 0.0
    if softmax_threshold is None:
        _lib.check(_L.bfa_fwd(plan.handle, _ptr(q), _ptr(k), _ptr(v), _strides3(q), _strides3(k), _strides3(v),
                              int(B), int(H), int(Hkv), int(D), ctypes.c_float(sc), _ptr(out), _strides3(out),
                              _ptr(lse), _stream(stream)))
    else:  # content-based block skipping (an approximation)
        _lib.check(_L.bfa_fwd_approx(plan.handle, _ptr(q), _ptr(k), _ptr(v), _strides3(q), _strides3(k),
                                     _strides3(v), int(B), int(H), int(Hkv), int(D), ctypes.c_float(sc),
                                     ctypes.c_float(float(softmax_threshold)), _ptr(out), _strides3(out), _ptr(lse),
                                     _stream(stream)))
    return out, lse


def bwd(plan, q, k, v, out, dout, lse, scale=None, dq=None, dk=None, dv=None, stream=None):
    """Gradients (dq, dk, dv) of ``fwd`` for an upstream gradient ``dout`` of ``out``.

    q, k, v, the plan and scale exactly as given to ``fwd``; out and lse as it
    returned them; dout shaped like q.  bf16 outputs shaped like q, k, v (dk and
    dv sum over the query heads of each kv head under GQA).
    """
    for t in (q, k, v, out, dout):
        if t.dtype != torch.bfloat16:
            raise TypeError("q, k, v, out, dout must be bfloat16")
        if t.stride(-1) != 1:
            raise ValueError("the head dim of q, k, v, out, dout must be contiguous")
    if lse is None or lse.dtype != torch.float32:
        raise TypeError("lse (float32, from fwd) is required")
    if dout.shape != q.shape or out.shape != q.shape:
        raise ValueError("out and dout must have the shape of q")
    packed = q.dim() == 3
    if packed:
        B = plan.info["batch"]
        _, H, D = q.shape
        Hkv = k.shape[1]
    else:
        B, _, H, D = q.shape
        Hkv = k.shape[2]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    sc = float(scale) if scale is not None else 0.0
    _lib.check(_L.bfa_bwd(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse.contiguous()),
                          _strides3(q), _strides3(k), _strides3(v), _strides3(out), _strides3(dout), int(B), int(H),
                          int(Hkv), int(D), ctypes.c_float(sc), _ptr(dq), _ptr(dk), _ptr(dv), _strides3(dq),
                          _strides3(dk), _strides3(dv), _stream(stream)))
    return dq, dk, dv


def fwd_paged(plan, q, k_cache, v_cache, block_table, scale=None, out=None, return_lse=True, lse=None, stream=None):
    """Masked attention forward with keys / values in a paged cache.

    k_cache / v_cache: (num_pages, page_size, Hkv, D) bf16; block_table: (n_seq,
    pages_per_seq) int32 page ids (tensorplay varlen ``block_table``).  q and the
    plan as for ``fwd``.
    """
    if q.dtype != torch.bfloat16 or k_cache.dtype != torch.bfloat16 or v_cache.dtype != torch.bfloat16:
        raise TypeError("q and the caches must be bfloat16")
    if k_cache.stride() != v_cache.stride() or k_cache.shape != v_cache.shape:
        raise ValueError("k_cache and v_cache must have the same shape and strides")
    packed = q.dim() == 3
    if packed:
        B = plan.info["batch"]
        _, H, D = q.shape
        lse_shape = (H, q.shape[0])
    else:
        B, Sq, H, D = q.shape
        lse_shape = (B, H, Sq)
    num_pages, page_size, Hkv, _ = k_cache.shape
    bt = block_table.to(torch.int32).contiguous()
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    if not return_lse:
        lse = None
    cs = (ctypes.c_int64 * 3)(k_cache.stride(0), k_cache.stride(1), k_cache.stride(2))
    sc = float(scale) if scale is not None else 0.0
    _lib.check(_L.bfa_fwd_paged(plan.handle, _ptr(q), _strides3(q), _ptr(k_cache), _ptr(v_cache), cs, num_pages,
                                page_size, _ptr(bt), bt.shape[1], int(B), int(H), int(Hkv), int(D),
                                ctypes.c_float(sc), _ptr(out), _strides3(out), _ptr(lse), _stream(stream)))
    return out, lse
