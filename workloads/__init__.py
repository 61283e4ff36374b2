"""Seeded synthetic inputs for the masked-attention workloads.

Inputs only.  This module draws q/k/v and the raw mask descriptions (token
padding and block-opening flags, sequence lengths, BSR routing, and the dense
boolean masks that *are* a workload's input); it holds no attention, block-id,
plan or predicate-evaluation arithmetic, and both the CUDA path and the CPU
oracle consume what it returns.

Seeds: tensor ``t`` of workload ``c`` uses ``1000 * c + t``.  q/k/v are drawn as
float32 N(0, 1) on the CPU with a seeded ``torch.Generator`` and cast to bf16, so
the same values come out on every machine.

Workloads (names used throughout the tests and the bench):

``tiny_blockcausal``   B=1, H=Hkv=2, N=256, D=64; 4 blocks opened at seeded
                       boundaries (token 0 plus 3 distinct positions), the last
                       16 tokens padded.
``causal_8192``        B=4, H=Hkv=32, N=8192, D=128; dense lower-triangular
                       (N, N) bool mask.  Same shape as BinFlash's usage example.
``blockcausal_gqa``    B=8, H=16, Hkv=4, N=1024, D=128; a 768-token bidirectional
                       prefix then 8 blocks of 32 tokens; per-row right padding of
                       U{0..128} tokens; 256 cross key columns ahead of the N keys,
                       26 of them (10 %) padded per batch row.
``varlen_16``          16 sequences with lengths U[512, 4096], packed THD,
                       H=32, Hkv=8, D=128; causal, and a 1024-key window run.
``bsr_16384``          B=2, H=32, Hkv=8, S=16384, D=128; BSR with 128-blocks, each
                       query block selecting its diagonal block plus floor(i/4)
                       distinct earlier blocks, independently per (b, hkv).
``union_16384``        same q/k/v shape; dense (S, S) mask = union of a 2048-key
                       causal window, 64 global tokens (rows 0..63 attend every key,
                       columns 0..63 are attended by every query) and random
                       128x128 tiles (each tile on with probability 0.1, each bit
                       of an on-tile Bernoulli(0.5)).
"""

from __future__ import annotations

import numpy as np
import torch

WORKLOADS = ("tiny_blockcausal", "causal_8192", "blockcausal_gqa", "varlen_16",
             "bsr_16384", "union_16384")

_CFG_ID = {"tiny_blockcausal": 1, "causal_8192": 2, "blockcausal_gqa": 3,
           "varlen_16": 4, "bsr_16384": 5, "union_16384": 5}


def _gen(seed):
    g = torch.Generator()
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, seed):
    """Seeded N(0, 1) float32 on the CPU, cast to bf16."""
    return torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32).to(torch.bfloat16)


def qkv(cfg, q_shape, kv_shape):
    return (randn_bf16(q_shape, 1000 * cfg + 0),
            randn_bf16(kv_shape, 1000 * cfg + 1),
            randn_bf16(kv_shape, 1000 * cfg + 2))


def tiny_blockcausal(B=1, H=2, N=256, D=64, n_pad=16, n_blocks=4):
    rng = np.random.default_rng(1000 * 1 + 3)
    att = np.zeros((B, N), dtype=np.uint8)
    att[:, 0] = 1
    for b in range(B):
        att[b, rng.choice(np.arange(1, N), size=n_blocks - 1, replace=False)] = 1
    pad = np.ones((B, N), dtype=bool)
    pad[:, N - n_pad:] = False
    q, k, v = qkv(1, (B, N, H, D), (B, N, H, D))
    return dict(name="tiny_blockcausal", B=B, H=H, Hkv=H, N=N, D=D, q=q, k=k, v=v,
                att_masks=att, pad_masks=pad, scale=D ** -0.5)


def causal_8192(B=4, H=32, N=8192, D=128, with_qkv=True):
    mask = torch.ones((N, N), dtype=torch.bool).tril_()
    out = dict(name="causal_8192", B=B, H=H, Hkv=H, N=N, D=D, mask=mask, scale=D ** -0.5)
    if with_qkv:
        out["q"], out["k"], out["v"] = qkv(2, (B, N, H, D), (B, N, H, D))
    return out


def blockcausal_gqa(B=8, H=16, Hkv=4, N=1024, D=128, n_cross=256, prefix=768, blk=32,
                    max_pad=128, n_cross_pad=26):
    rng = np.random.default_rng(1000 * 3 + 3)
    att = np.zeros((B, N), dtype=np.uint8)
    att[:, 0] = 1
    att[:, prefix::blk] = 1
    pad = np.ones((B, N), dtype=bool)
    p = rng.integers(0, max_pad + 1, size=B)
    for b in range(B):
        if p[b]:
            pad[b, N - p[b]:] = False
    cpad = np.ones((B, n_cross), dtype=bool)
    for b in range(B):
        cpad[b, rng.choice(n_cross, size=n_cross_pad, replace=False)] = False
    q, k, v = qkv(3, (B, N, H, D), (B, n_cross + N, Hkv, D))
    return dict(name="blockcausal_gqa", B=B, H=H, Hkv=Hkv, N=N, D=D, n_cross=n_cross,
                q=q, k=k, v=v, att_masks=att, pad_masks=pad, cross_pad_masks=cpad,
                pad_len=p, scale=D ** -0.5)


def varlen_16(n_seq=16, lo=512, hi=4096, H=32, Hkv=8, D=128, window=1024):
    rng = np.random.default_rng(1000 * 4 + 3)
    lens = rng.integers(lo, hi + 1, size=n_seq)
    cu = np.zeros(n_seq + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    T = int(cu[-1])
    q, k, v = qkv(4, (T, H, D), (T, Hkv, D))
    return dict(name="varlen_16", n_seq=n_seq, H=H, Hkv=Hkv, D=D, total=T, lens=lens,
                cu_seqlens=cu, max_len=int(lens.max()), window=window, q=q, k=k, v=v,
                scale=D ** -0.5)


def bsr_routing(B, Hkv, n_blocks, seed):
    """Diagonal block plus floor(i/4) distinct earlier blocks per query block."""
    rng = np.random.default_rng(seed)
    indptr = np.zeros((B, Hkv, n_blocks + 1), dtype=np.int32)
    idx = []
    pos = 0
    for b in range(B):
        for h in range(Hkv):
            indptr[b, h, 0] = pos
            for i in range(n_blocks):
                n_prev = i // 4
                prev = rng.choice(i, size=n_prev, replace=False) if n_prev else np.zeros(0, np.int64)
                row = np.sort(np.concatenate([prev, [i]])).astype(np.int32)
                idx.append(row)
                pos += row.size
                indptr[b, h, i + 1] = pos
    return indptr, np.concatenate(idx).astype(np.int32)


def bsr_rows_routing(B, Hkv, Sq, q_block, kv_block, seed):
    """BSR rows of q_block query tokens: the key block holding the row's first
    token plus floor(d / 4) distinct earlier key blocks (d = that block's index),
    drawn independently for every row."""
    rng = np.random.default_rng(seed)
    nqb = -(-Sq // q_block)
    indptr = np.zeros((B, Hkv, nqb + 1), dtype=np.int32)
    idx = []
    pos = 0
    for b in range(B):
        for h in range(Hkv):
            indptr[b, h, 0] = pos
            for r in range(nqb):
                d = (r * q_block) // kv_block
                n_prev = d // 4
                prev = rng.choice(d, size=n_prev, replace=False) if n_prev else np.zeros(0, np.int64)
                row = np.sort(np.concatenate([prev, [d]])).astype(np.int32)
                idx.append(row)
                pos += row.size
                indptr[b, h, r + 1] = pos
    return indptr, np.concatenate(idx).astype(np.int32)


def bsr_16384_q16_gqa8(B=2, H=32, Hkv=4, S=16384, D=128, q_block=16, kv_block=128, with_qkv=True):
    """BSR routing with 16-token query rows and 8 query heads per kv head (GQA)."""
    indptr, indices = bsr_rows_routing(B, Hkv, S, q_block, kv_block, 1000 * 5 + 7)
    out = dict(name="bsr_16384_q16_gqa8", B=B, H=H, Hkv=Hkv, S=S, D=D, q_block=q_block, kv_block=kv_block,
               block_indptr=indptr, block_indices=indices, causal=True, scale=D ** -0.5)
    if with_qkv:
        out["q"], out["k"], out["v"] = qkv(6, (B, S, H, D), (B, S, Hkv, D))
    return out


def bsr_16384(B=2, H=32, Hkv=8, S=16384, D=128, block=128, with_qkv=True):
    indptr, indices = bsr_routing(B, Hkv, -(-S // block), 1000 * 5 + 3)
    out = dict(name="bsr_16384", B=B, H=H, Hkv=Hkv, S=S, D=D, block=block,
               block_indptr=indptr, block_indices=indices, causal=True, scale=D ** -0.5)
    if with_qkv:
        out["q"], out["k"], out["v"] = qkv(5, (B, S, H, D), (B, S, Hkv, D))
    return out


def union_mask(S, window=2048, n_global=64, tile=128, p_tile=0.1, p_bit=0.5, seed=1000 * 5 + 4):
    """The dense union mask (S, S) bool of the second BSR-workload pass."""
    rng = np.random.default_rng(seed)
    M = np.zeros((S, S), dtype=bool)
    for r0 in range(0, S, 1024):                      # window band, built in row chunks
        r1 = min(S, r0 + 1024)
        i = np.arange(r0, r1)[:, None]
        j = np.arange(S)[None, :]
        M[r0:r1] = (j <= i) & (i - j < window)
    M[:n_global, :] = True
    M[:, :n_global] = True
    nt = -(-S // tile)
    on = rng.random((nt, nt)) < p_tile
    for qt, kt in zip(*np.nonzero(on)):
        q0, k0 = qt * tile, kt * tile
        q1, k1 = min(S, q0 + tile), min(S, k0 + tile)
        M[q0:q1, k0:k1] |= rng.random((q1 - q0, k1 - k0)) < p_bit
    return M


def union_16384(B=2, H=32, Hkv=8, S=16384, D=128, with_qkv=True):
    out = dict(name="union_16384", B=B, H=H, Hkv=Hkv, S=S, D=D,
               mask=torch.from_numpy(union_mask(S)), scale=D ** -0.5)
    if with_qkv:
        out["q"], out["k"], out["v"] = qkv(5, (B, S, H, D), (B, S, Hkv, D))
    return out


def get(name, **kw):
    return globals()[name](**kw)
