// Plan layout shared by the host code, the planner kernels and the forward kernel.
#pragma once

#include <cstdint>

namespace bfa {

constexpr int kTile = 128;             // query and key tile edge
constexpr int kWordsPerTileRow = 4;    // 128 columns / 32 bits
constexpr int kFineWordsPerTile = kTile * kWordsPerTileRow;  // 512 uint32 = 2 KB

enum MaskMode : int32_t {
  MASK_BITS = 0,     // partial tiles carry packed fine masks (dense plans)
  MASK_BLOCKID = 1,  // partial tiles evaluate q_valid & k_valid & (k_blk <= q_blk)
  MASK_POS = 2,      // partial tiles evaluate causal (+ window) on positions
  MASK_PRED = 3      // partial tiles evaluate an OR of position terms (pred.cuh)
};

enum DevErr : uint32_t {
  DEVERR_TIMEOUT = 1u,       // a bounded wait gave up
  DEVERR_BSR_RANGE = 2u,     // BSR offsets out of range / decreasing
  DEVERR_BSR_ORDER = 4u,     // BSR ids unsorted, duplicated or out of range
  DEVERR_BOUNDS = 8u,        // checked build: an index left its array (the access was skipped)
  DEVERR_GUARD = 16u,        // checked build: guard bytes after a plan array were overwritten
};

// Index checks of the checked build (compiled with -DBFA_CHECKED): an index
// outside [0, n) sets DEVERR_BOUNDS in the plan's error word and is replaced by
// 0, so that the access stays inside the array; no trap, no assert.  The normal
// build compiles the index unchanged.
#ifdef BFA_CHECKED
__device__ __forceinline__ int64_t checked_index(int64_t i, int64_t n, uint32_t* err) {
  if (i < 0 || i >= n) {
    atomicOr(err, DEVERR_BOUNDS);
    return 0;
  }
  return i;
}
#define BFA_IDX(i, n, err) (::bfa::checked_index((i), (n), (err)))
#define BFA_CHECK(cond, err) \
  do {                       \
    if (!(cond)) atomicOr((err), ::bfa::DEVERR_BOUNDS); \
  } while (0)
#else
#define BFA_IDX(i, n, err) (i)
#define BFA_CHECK(cond, err) \
  do {                       \
  } while (0)
#endif

// One row group: a batch (batched plans), a sequence (varlen plans), a
// (batch, kv head) pair (BSR plans) or the single shared group of a dense plan.
struct GroupInfo {
  int32_t q_off;      // first query token of the group along the token axis
  int32_t q_len;      // query tokens
  int32_t k_off;      // first key token
  int32_t k_len;      // key tokens
  int32_t b;          // batch index used for strides (-1: any batch, dense plans)
  int32_t hkv;        // BSR: kv head of the routing; -1: every head
  int32_t row0;       // first plan row of the group
  int32_t nqt;        // query tiles
  int32_t nkt;        // key tiles
  int32_t qid_off;    // block-id plans: offset of the group's padded q ids / validity
  int32_t kid_off;    // block-id plans: offset of the group's padded k ids
  int32_t kbit_off;   // block-id plans: word offset of the group's k validity bits
  int64_t cls_off;    // offset of the group's (nqt x nkt) class grid
};
static_assert(sizeof(GroupInfo) == 56, "GroupInfo layout");

// Device view of a plan (pointers into the plan's slab).
struct PlanDev {
  const GroupInfo* groups;
  const int32_t* row_group;  // [n_rows]
  const int32_t* row_ptr;    // [n_rows + 1]
  const int32_t* kv_tile;    // [listed tiles]
  const int32_t* part;       // [listed tiles]: -1 full, else the tile's class-grid index
  const uint32_t* fine;      // [grid_tiles * 512] (dense plans) indexed by grid index
  const int32_t* order;      // [n_rows] longest first
  const int32_t* pair_row;   // [n_pairs] first row of each work pair (~row: single row)
  const int32_t* pair_order; // [n_pairs] longest first
  const int2* row_work;      // [n_rows] longest first: {row, group of the row}
  const int2* pair_work;     // [n_pairs] longest first: {pair_row, group of its first row}
  const int32_t* qid;        // padded q block ids  (block-id plans)
  const uint8_t* qvalid;     // padded q validity   (block-id plans)
  const int32_t* kid;        // padded k block ids  (block-id plans)
  const uint32_t* kbits;     // padded k validity bits (block-id plans)
  const int32_t* terms;      // position terms (predicate plans), 6 ints each
  uint32_t* err;             // device error word
  int64_t cap_tiles;         // entries of kv_tile / part (and of the class grid)
  int64_t cap_fine;          // tiles of packed fine words behind `fine`
  int64_t cap_qid, cap_kid, cap_kbits;  // entries of qid / qvalid, kid, kbits
  int32_t n_rows;
  int32_t n_pairs;
  int32_t n_groups;
  int32_t mask_mode;
  int32_t causal;
  int32_t window;            // -1 off
  int32_t kind;
  int32_t n_terms;
};

}  // namespace bfa
