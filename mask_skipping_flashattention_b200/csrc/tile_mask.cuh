// Attend-bits of one row of a tile, for the mask forms of a plan (shared by the
// forward, the backward's query-tile pass and, transposed, its key-tile pass).
// `Ctx` carries the group fields the forms need: k_len, q_len, qid_off, kid_off,
// kbit_off.  The forms: packed fine words (dense and generic block-sparse plans),
// the block-id predicate q_valid & k_valid & (k_blk <= q_blk) (opentau
// flash_attn_blockmask), position terms (pred.cuh) and causal / window positions;
// full tiles need no mask except past the end of the keys (or queries).
#pragma once

#include <cstdint>

#include "plan_types.cuh"
#include "pred.cuh"

namespace bfa {

// attend-bits of one query row (position qpos in its group) against the 128
// columns of key tile `kt`
template <typename Ctx>
__device__ __forceinline__ void row_mask_words(const PlanDev& plan, const Ctx& wk, int qpos, int row, int kt, int part,
                                               uint32_t (&am)[4]) {
  const int ncols = wk.k_len - kt * kTile;  // in-range columns (may exceed 128)
  if (plan.mask_mode == MASK_BITS) {
    if (part >= 0) {
      const int64_t fp = BFA_IDX(static_cast<int64_t>(part), plan.cap_fine, plan.err);
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(plan.fine + fp * kFineWordsPerTile +
                                                           row * kWordsPerTileRow));
      am[0] = v.x; am[1] = v.y; am[2] = v.z; am[3] = v.w;
    } else {
      am[0] = am[1] = am[2] = am[3] = 0xffffffffu;
    }
  } else if (plan.mask_mode == MASK_BLOCKID) {
    if (part >= 0) {
      // called by whole warps (the tile is the same for the warp's 32 rows)
      const int64_t qi = BFA_IDX(static_cast<int64_t>(wk.qid_off) + qpos, plan.cap_qid, plan.err);
      const int32_t qb = plan.qid[qi];
      const bool qv = plan.qvalid[qi] != 0;
#ifdef BFA_CHECKED
      const bool kin = kt >= 0 && wk.kid_off + (kt + 1) * kTile <= plan.cap_kid &&
                       wk.kbit_off + (kt + 1) * kWordsPerTileRow <= plan.cap_kbits;
      if (!kin) atomicOr(plan.err, DEVERR_BOUNDS);
      const int64_t k0 = kin ? wk.kid_off + kt * kTile : 0;
      const int64_t b0 = kin ? wk.kbit_off + kt * kWordsPerTileRow : 0;
#else
      const int64_t k0 = wk.kid_off + kt * kTile;
      const int64_t b0 = wk.kbit_off + kt * kWordsPerTileRow;
#endif
      const int32_t* kids = plan.kid + k0;
      const int4* kb4 = reinterpret_cast<const int4*>(kids);
      const uint4 kv = __ldg(reinterpret_cast<const uint4*>(plan.kbits + b0));
      const uint32_t kvw[4] = {kv.x, kv.y, kv.z, kv.w};
      // Key ids non-decreasing across the tile (the usual form: cross columns at
      // INT32_MIN, then running block counts) make {j : k_blk[j] <= q_blk} a prefix
      // of the tile, whose length one binary search finds; otherwise every key is
      // compared.  The warp checks the order with one 16-byte load per lane.
      const int lane = row & 31;
      const int4 mine = __ldg(kb4 + lane);
      const int prev = __shfl_up_sync(0xffffffffu, mine.w, 1);
      const bool in_order = mine.x <= mine.y && mine.y <= mine.z && mine.z <= mine.w && (lane == 0 || prev <= mine.x);
      if (__all_sync(0xffffffffu, in_order)) {
        int lo = 0, hi = kTile;  // the first key with k_blk > q_blk lies in [lo, hi]
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          if (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(kids + mid) <= qb) lo = mid + 1;
            else hi = mid;
          }
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int z = lo - 32 * w;  // attended keys of this word: [0, z)
          const uint32_t bits = (z >= 32) ? 0xffffffffu : (z <= 0 ? 0u : ((1u << z) - 1u));
          am[w] = qv ? (bits & kvw[w]) : 0u;
        }
      } else {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t bits = 0;
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const int4 k = __ldg(kb4 + w * 8 + c4);
            bits |= (k.x <= qb ? 1u : 0u) << (c4 * 4 + 0);
            bits |= (k.y <= qb ? 1u : 0u) << (c4 * 4 + 1);
            bits |= (k.z <= qb ? 1u : 0u) << (c4 * 4 + 2);
            bits |= (k.w <= qb ? 1u : 0u) << (c4 * 4 + 3);
          }
          am[w] = qv ? (bits & kvw[w]) : 0u;
        }
      }
    } else {
      am[0] = am[1] = am[2] = am[3] = 0xffffffffu;
    }
  } else if (plan.mask_mode == MASK_PRED) {
    if (part >= 0) {
      pred_words(plan.terms, plan.n_terms, qpos, kt, wk.k_len, am);
    } else {
      am[0] = am[1] = am[2] = am[3] = 0xffffffffu;
    }
  } else {  // MASK_POS: causal kv_pos <= q_pos, optional window q_pos - kv_pos < W
    int hi = plan.causal ? (qpos - kt * kTile) : 127;                           // last attended column
    int lo = (plan.window >= 0) ? (qpos - kt * kTile - plan.window + 1) : 0;  // first attended column
    if (part < 0) { hi = 127; lo = 0; }
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int a = lo - 32 * w, z = hi - 32 * w;  // attended range inside this word
      uint32_t m_hi = (z >= 31) ? 0xffffffffu : (z < 0 ? 0u : ((2u << z) - 1u));
      uint32_t m_lo = (a <= 0) ? 0xffffffffu : (a > 31 ? 0u : ~((1u << a) - 1u));
      am[w] = m_hi & m_lo;
    }
  }
  // key tokens past the group's end (edge tile) are never attended
  if (ncols < kTile) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int z = ncols - 32 * w;
      const uint32_t m = (z >= 32) ? 0xffffffffu : (z <= 0 ? 0u : ((1u << z) - 1u));
      am[w] &= m;
    }
  }
}


// Attend-bits of one key (position kpos in its group, row `col` of key tile kt)
// against the 128 queries of query tile qt: bit i of word w is query 32 w + i of
// the tile.  `part` is the tile's entry in the transposed lists (-1 full).
// Queries past the group's end (edge tile) never attend.
template <typename Ctx>
__device__ __forceinline__ void col_mask_words(const PlanDev& plan, const Ctx& wk, int kpos, int col, int qt, int part,
                                               uint32_t (&am)[4]) {
  if (part < 0) {
    am[0] = am[1] = am[2] = am[3] = 0xffffffffu;
  } else if (plan.mask_mode == MASK_BITS) {
    // column `col` of the tile's row-major fine words.  A warp holds the keys
    // 32 (col / 32) .. + 31; for each block of 32 query rows its lane l loads row
    // l's word of those keys, and a 32 x 32 bit transpose across the warp (five
    // butterfly rounds of shuffles) hands lane l the column of its own key.  All
    // 32 lanes must call this together.
    const uint32_t* f = plan.fine + static_cast<int64_t>(part) * kFineWordsPerTile + (col >> 5);
    const int lane = col & 31;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t x = __ldg(f + (32 * w + lane) * kWordsPerTileRow);
#pragma unroll
      for (int j = 16; j > 0; j >>= 1) {
        const uint32_t m = j == 16 ? 0x0000ffffu : j == 8 ? 0x00ff00ffu : j == 4 ? 0x0f0f0f0fu
                         : j == 2 ? 0x33333333u : 0x55555555u;
        const uint32_t y = __shfl_xor_sync(0xffffffffu, x, j);
        x = (lane & j) ? ((x & ~m) | ((y >> j) & m)) : ((x & m) | ((y << j) & ~m));
      }
      am[w] = x;
    }
  } else if (plan.mask_mode == MASK_BLOCKID) {
    const int32_t kb = plan.kid[wk.kid_off + kpos];
    const bool kv = (plan.kbits[wk.kbit_off + (kpos >> 5)] >> (kpos & 31)) & 1u;
    // the tile's 128 query ids and validity bytes, read 16 bytes at a time (the
    // per-group copies are padded to whole tiles, so each tile starts 16-byte aligned)
    const int32_t* qids = plan.qid + wk.qid_off + qt * kTile;
    const int4* qb4 = reinterpret_cast<const int4*>(qids);
    const uint4* qv16 = reinterpret_cast<const uint4*>(plan.qvalid + wk.qid_off + qt * kTile);
    // Whole warps call this (one tile per warp).  Query ids non-decreasing over the
    // tile with every query valid (the usual form) make the attended rows a suffix
    // {i : q_blk[i] >= k_blk}, found by one binary search; otherwise every query is
    // compared.  The warp checks with one 16-byte id load and one 4-byte validity
    // load per lane.
    const int lane = col & 31;
    const int4 mine = __ldg(qb4 + lane);
    const uint32_t vmine = __ldg(reinterpret_cast<const uint32_t*>(qv16) + lane);
    const int prev = __shfl_up_sync(0xffffffffu, mine.w, 1);
    const bool fast = mine.x <= mine.y && mine.y <= mine.z && mine.z <= mine.w && (lane == 0 || prev <= mine.x) &&
                      (vmine & 0xffu) != 0 && (vmine & 0xff00u) != 0 && (vmine & 0xff0000u) != 0 &&
                      (vmine & 0xff000000u) != 0;
    if (__all_sync(0xffffffffu, fast)) {
      int lo = 0, hi = kTile;  // the first query with q_blk >= k_blk lies in [lo, hi]
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        if (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (__ldg(qids + mid) < kb) lo = mid + 1;
          else hi = mid;
        }
      }
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int a = lo - 32 * w;  // attended rows of this word: [a, 32)
        const uint32_t bits = (a <= 0) ? 0xffffffffu : (a >= 32 ? 0u : ~((1u << a) - 1u));
        am[w] = kv ? bits : 0u;
      }
    } else {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint4 v16a = __ldg(qv16 + 2 * w), v16b = __ldg(qv16 + 2 * w + 1);
        const uint32_t vw[8] = {v16a.x, v16a.y, v16a.z, v16a.w, v16b.x, v16b.y, v16b.z, v16b.w};
        uint32_t bits = 0;
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const int4 q = __ldg(qb4 + w * 8 + c4);
          const uint32_t vb = vw[c4];
          bits |= ((vb & 0xffu) != 0 && kb <= q.x ? 1u : 0u) << (c4 * 4 + 0);
          bits |= ((vb & 0xff00u) != 0 && kb <= q.y ? 1u : 0u) << (c4 * 4 + 1);
          bits |= ((vb & 0xff0000u) != 0 && kb <= q.z ? 1u : 0u) << (c4 * 4 + 2);
          bits |= ((vb & 0xff000000u) != 0 && kb <= q.w ? 1u : 0u) << (c4 * 4 + 3);
        }
        am[w] = kv ? bits : 0u;
      }
    }
  } else if (plan.mask_mode == MASK_PRED) {
    pred_words_col(plan.terms, plan.n_terms, kpos, qt, wk.q_len, am);
  } else {  // MASK_POS: causal q_pos >= kv_pos, optional window q_pos - kv_pos < W
    const int lo = plan.causal ? (kpos - qt * kTile) : 0;                                  // first attended row
    const int hi = (plan.window >= 0) ? (kpos - qt * kTile + plan.window - 1) : 127;      // last attended row
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int a = lo - 32 * w, z = hi - 32 * w;
      uint32_t m_hi = (z >= 31) ? 0xffffffffu : (z < 0 ? 0u : ((2u << z) - 1u));
      uint32_t m_lo = (a <= 0) ? 0xffffffffu : (a > 31 ? 0u : ~((1u << a) - 1u));
      am[w] = m_hi & m_lo;
    }
  }
  const int nrows = wk.q_len - qt * kTile;  // in-range query rows (may exceed 128)
  if (nrows < kTile) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int z = nrows - 32 * w;
      const uint32_t m = (z >= 32) ? 0xffffffffu : (z <= 0 ? 0u : ((1u << z) - 1u));
      am[w] &= m;
    }
  }
}

}  // namespace bfa
