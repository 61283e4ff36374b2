/*
 * bfa.h -- C ABI of the mask-aware fused attention forward for NVIDIA B200 (sm_100a).
 *
 * The library computes O = softmax(scale * Q K^T + mask) V and the natural-log
 * LSE of every query row, where the boolean mask (True = attend) is never
 * materialised inside the score loop.  A mask is first turned into a *plan*:
 * for every 128-row query tile, the ascending list of 128-column key tiles that
 * hold at least one attended pair, each marked full (every in-range pair
 * attended) or partial, plus 32-bit packed fine masks for the partial tiles of a
 * dense mask.  The forward kernel then visits only the listed tiles, runs full
 * tiles with no mask work, and masks partial tiles from the packed bits, from the
 * block-id predicate, or from positions.
 *
 * Sources (page title, section):
 *   - BinFlash, "Efficiently Dispatching FlashAttention For Partially Filled
 *     Attention Masks": a coarse per-block mask with the partial blocks' bits packed 32 to a word, sorted
 *     non-empty key-block list per query row, all-True blocks with no mask loads,
 *     all-False blocks skipped; mask (N, N) bool, True = attend; scale 1/sqrt(D).
 *   - opentau.policies.flash_attn_cuda, make_att_block_ids / flash_attn_blockmask:
 *     attend(i, j) = q_valid[i] & k_valid[j] & (k_blk[j] <= q_blk[i]); cross
 *     columns carry k_blk = INT32_MIN; q (B, Sq, H, D), k/v (B, Sk, Hkv, D),
 *     H % Hkv == 0; output has the dtype of q; is_available / load_error.
 *   - tensorplay.nn.attention.varlen, "Packed layout": (total_tokens, H, D)
 *     packing with int32 cumulative lengths starting at 0; under-stated max
 *     lengths are an error; window_size, out= form, CUDA-only.
 *   - flashinfer.attention.prims_ts.block_sparse_attention, Parameters: BSR
 *     block_indptr [B, Hkv, ceil(Sq/q_block_size)+1] / block_indices, canonical
 *     rows validated synchronously, mask_type dense|causal, plan once outside
 *     graph capture and capture only the run, caller-owned out.
 *   - tensorplay.nn.attention.omni_attention, "Outputs": return_lse.
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is a DEVICE pointer unless stated otherwise; a host
 *     pointer is rejected with BFA_ERR_NOT_DEVICE before anything is launched.
 *   - The caller owns every input and output buffer.  The library owns plans.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     stream-ordered on it.  bfa_fwd never synchronises and may be captured in a
 *     CUDA graph; the planners may synchronise once (see each).
 *   - Errors: a negative bfa_status; bfa_last_error() gives a message (per thread).
 *     Argument errors are detected on the host before any launch.
 *   - Tiles are 128 x 128 (BFA_TILE).  bf16 q/k/v/out, head dim D in {64, 128}.
 */
#ifndef BFA_H_
#define BFA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct bfa_plan bfa_plan; /* opaque, library-owned, freed by bfa_plan_destroy */

typedef enum bfa_status {
  BFA_OK = 0,
  BFA_ERR_INVALID_ARG = -1,      /* shape, stride, alignment or value out of range      */
  BFA_ERR_UNSUPPORTED = -2,      /* valid request this build does not implement         */
  BFA_ERR_NOT_DEVICE = -3,       /* a pointer that must be device memory is not         */
  BFA_ERR_NONCANONICAL_BSR = -4, /* BSR rows not sorted / unique / in range             */
  BFA_ERR_CAPACITY = -5,         /* sizes beyond what the library can index or allocate */
  BFA_ERR_CUDA = -6,             /* a CUDA runtime call failed                          */
  BFA_ERR_TIMEOUT = -7,          /* a device-side wait ran past its bound               */
  BFA_ERR_BOUNDS = -8            /* checked build: an index left its array, or the guard
                                    bytes after a plan array were overwritten; any build:
                                    a block of the fused backward was given shared memory
                                    that is not 1024-byte aligned and did no work         */
} bfa_status;

enum { BFA_TILE = 128 };

typedef enum bfa_plan_kind {
  BFA_PLAN_DENSE = 1,      /* from a dense (Sq, Sk) bool mask, shared by every batch and head   */
  BFA_PLAN_BLOCKIDS = 2,   /* from per-token block ids and validity, per batch / sequence       */
  BFA_PLAN_POSITIONAL = 3, /* causal (+ window) on token positions, per batch / sequence        */
  BFA_PLAN_BSR = 4,        /* from BSR routing or block bitmaps, per (batch, kv head)           */
  BFA_PLAN_PREDICATE = 5   /* from position terms (OR of band / box constraints), per sequence  */
} bfa_plan_kind;

/* One conjunction of position constraints on (i, j) = (query, key) positions
 * local to the sequence:  diag_lo <= i - j <= diag_hi  AND  q_lo <= i < q_hi
 * AND  k_lo <= j < k_hi.  INT32_MIN / INT32_MAX leave a bound open.  Examples:
 * causal {0, MAX, MIN, MAX, MIN, MAX}; past window of W keys {0, W-1, ...};
 * G global query rows {MIN, MAX, MIN, G, MIN, MAX}; P prefix keys
 * {MIN, MAX, MIN, MAX, MIN, P}. */
typedef struct bfa_mask_term {
  int32_t diag_lo, diag_hi;
  int32_t q_lo, q_hi;
  int32_t k_lo, k_hi;
} bfa_mask_term;

enum { BFA_MAX_MASK_TERMS = 16 };

/* Host-side description of a plan (no synchronisation needed to read it). */
typedef struct bfa_plan_info {
  int32_t kind;           /* bfa_plan_kind                                                        */
  int32_t varlen;         /* 1: packed THD layout through cu_seqlens                              */
  int32_t n_groups;       /* row groups: 1 (dense), B (blockids/positional), n_seq (varlen),
                             B*Hkv (BSR)                                                          */
  int32_t n_rows;         /* query-tile rows over all groups                                      */
  int64_t grid_tiles;     /* (row, key tile) positions over all groups = size of the class grid   */
  int32_t batch;          /* B of the plan (0 for dense plans: any B)                             */
  int32_t hkv;            /* BSR only: kv heads of the routing; else 0                            */
  int32_t sq, sk;         /* batched: per-batch lengths; varlen: total packed tokens              */
  int32_t max_kv_tiles;   /* longest key-tile count of a group                                    */
  int32_t window_left;    /* -1: no window                                                        */
  int32_t causal;         /* positional / BSR plans: 1 if kv_idx <= q_idx is applied             */
  int32_t n_pairs;        /* work pairs: consecutive query tiles (2i, 2i+1) of one group          */
  int32_t packed_fine;    /* 1: partial tiles carry packed fine masks (bfa_plan_export fills fine) */
  int32_t n_cols;         /* key-tile columns (sum over groups of their key tiles): the backward's
                             dK/dV work units, see bfa_plan_export_cols                         */
  int32_t heads_per_kv;   /* bfa_plan_bsr_packed: query heads packed into each row's tiles; else 1;
                             with packing, sq counts query positions and the groups' rows count
                             positions x heads_per_kv                                           */
} bfa_plan_info;

/* Library version string. */
const char* bfa_version(void);

/* Message of the last failed call on this thread ("" if none).  The analogue of
 * opentau's load_error(): a diagnostic string, valid until the next call. */
const char* bfa_last_error(void);

/* 1 if a device of compute capability 10.0 is present and the kernels can load,
 * else 0 (message in bfa_last_error).  Mirrors opentau's is_available(). */
int bfa_is_available(void);

/*
 * Block ids from padding and block-opening flags (opentau make_att_block_ids).
 *   pad_masks [B, N] u8 (nonzero = real token), att_masks [B, N] u8 (nonzero =
 *   the token opens a new block, zero = it continues the current one).
 *   q_blk[b, i] = number of block openings in att_masks[b, 0..i] (inclusive), so
 *   tokens before the first opening get id 0.  With n_cross > 0, n_cross key
 *   columns with id INT32_MIN and validity cross_pad[B, n_cross] are prepended.
 * Outputs (caller-owned, device): q_blk [B, N] i32, k_blk [B, n_cross + N] i32,
 *   q_valid [B, N] u8, k_valid [B, n_cross + N] u8.  Row-major, contiguous.
 * Stream-ordered, no synchronisation.
 */
bfa_status bfa_make_block_ids(const uint8_t* pad_masks, const uint8_t* att_masks, int B, int N,
                              int n_cross, const uint8_t* cross_pad, int32_t* q_blk, int32_t* k_blk,
                              uint8_t* q_valid, uint8_t* k_valid, void* stream);

/*
 * Plan from a dense bool mask (BinFlash preprocessing).
 *   mask: device, Sq rows of Sk bytes (nonzero = attend), row r at
 *   mask + r * mask_row_stride (bytes, >= Sk).  Shared by every batch and head.
 * Tile classes are decided over the in-range pairs of each tile; partial tiles
 * get 128 rows x 4 uint32 words, bit b of word w = column 32w + b (LSB first).
 * Stream-ordered, no synchronisation; the mask may be freed once the stream has
 * passed this call.
 */
bfa_status bfa_plan_dense(const uint8_t* mask, int64_t mask_row_stride, int Sq, int Sk, bfa_plan** out,
                          void* stream);

/*
 * Plan from the compact block-id form (opentau) or from positions.
 *   q_blk [B, Sq] / k_blk [B, Sk] i32 (batched) or [total_q] / [total_k] (varlen).
 *     Both NULL: identity positions local to each sequence, i.e. causal
 *     kv_idx <= q_idx (top-left aligned).
 *   q_valid / k_valid u8, same indexing; NULL = all valid.
 *   cu_seqlens_q / cu_seqlens_k: device i32 [B + 1] starting at 0 for the packed
 *     THD layout (tensorplay varlen), or NULL for the batched layout.  In varlen
 *     mode B is the number of sequences, Sq / Sk are ignored, and max_q / max_k
 *     must be >= every sequence length (under-stating is BFA_ERR_INVALID_ARG).
 *   seqused_k: device i32 [B] or NULL: only the first seqused_k[b] keys of batch
 *     entry / sequence b are usable (tensorplay varlen seqused_k); read back once.
 *   window_left: -1 = off; else keys with 0 <= q_pos - k_pos < window_left are
 *     kept (window of past keys including the query's own position).  Requires
 *     positional ids and no validity masks.
 * The kernel evaluates attend(i, j) = q_valid[i] & k_valid[j] & (k_blk[j] <= q_blk[i])
 * (or the position rule) on partial tiles; the plan keeps its own copy of the ids.
 * Varlen mode reads cu_seqlens back to the host once (one synchronisation).
 */
bfa_status bfa_plan_blockids(const int32_t* q_blk, const int32_t* k_blk, const uint8_t* q_valid,
                             const uint8_t* k_valid, int B, int Sq, int Sk, const int32_t* cu_seqlens_q,
                             const int32_t* cu_seqlens_k, const int32_t* seqused_k, int max_q, int max_k,
                             int window_left, bfa_plan** out, void* stream);

/*
 * Plan from a position predicate: attend(i, j) = OR over the n_terms terms of
 * their constraints (tensorplay omni_attention mask_mod algebra: causal,
 * window, and_masks inside a term, or_masks across terms; n_terms = 0 attends
 * nothing, one open term is noop_mask).  terms: HOST array, copied.  Layout as
 * for bfa_plan_blockids: batched (B, Sq, Sk) or varlen through cu_seqlens with
 * max_q / max_k, and optional seqused_k.  Tiles are classified exactly from the
 * terms; the kernel evaluates the terms on partial tiles only, so no mask is
 * materialised.  Varlen and seqused_k read back once.
 */
bfa_status bfa_plan_predicate(const bfa_mask_term* terms, int n_terms, int B, int Sq, int Sk,
                              const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, const int32_t* seqused_k,
                              int max_q, int max_k, bfa_plan** out, void* stream);

/*
 * Plan from BSR routing (flashinfer block_sparse_attention, sparse_format "bsr").
 *   indptr [B, Hkv, ceil(Sq/q_block)+1] i32: absolute offsets into indices, each
 *   (b, hkv) slice non-decreasing; indices [n_indices] i32: KV block ids, each
 *   row strictly increasing in [0, ceil(Skv/kv_block)).
 *   q_block >= 1 query tokens per BSR row; kv_block key tokens per block id,
 *   one of 8, 16, 32 or 64 m for an integer m >= 1 (the sizes the page allows).
 *   causal != 0 applies kv_idx <= q_idx on absolute positions inside the selected
 *   blocks (mask_type "causal"); otherwise every pair of a selected block attends.
 *   kv_valid_bits [B, ceil(Skv/32)] u32 or NULL: bit j % 32 of word j / 32 of row b
 *   marks key token j of batch b valid (kv_valid_bits); invalid keys never attend.
 * Query head h uses the routing of kv head h / (H / Hkv).
 * 128 x 128 blocks without validity bits map BSR rows onto tile rows directly
 * (blocks below the diagonal full, on it partial, above it dropped, masked by
 * position in the kernel); any other shape is reduced to tile classes plus packed
 * fine masks for the partial tiles.  Validation runs on the device and is read
 * back synchronously, like the page's plan step (one or two syncs); non-canonical
 * rows give BFA_ERR_NONCANONICAL_BSR.
 */
bfa_status bfa_plan_bsr(const int32_t* indptr, const int32_t* indices, int64_t n_indices, int B, int Hkv,
                        int Sq, int Skv, int q_block, int kv_block, int causal, const uint32_t* kv_valid_bits,
                        bfa_plan** out, void* stream);

/*
 * bfa_plan_bsr with GQA-packed query tiles (flashinfer block_sparse_attention,
 * q_block_size: one physical query tile holds the query tokens of BSR rows for
 * every query head of a kv head, so it never straddles two rows' lists when
 * q_block * heads_per_kv is a multiple of 128).  Plan row t of the (b, hkv)
 * routing slice is query position t / heads_per_kv of query head
 * hkv * heads_per_kv + t % heads_per_kv; a 128-row tile is 128 / heads_per_kv
 * positions of all heads_per_kv heads.  heads_per_kv = H / Hkv of the calls that
 * use the plan: a power of two up to 128, with q_block * heads_per_kv a multiple
 * of 8 (the page's rule); other arguments as for bfa_plan_bsr.  Every call takes
 * these plans (bfa_fwd, bfa_fwd_approx, bfa_fwd_paged, bfa_bwd) with H = Hkv *
 * heads_per_kv and a batched (B, Sq, H, D) query layout whose heads of one kv head
 * are adjacent, as BSHD has them; q, out, dout and dq move as 5-D boxes of all
 * the kv head's heads.
 */
bfa_status bfa_plan_bsr_packed(const int32_t* indptr, const int32_t* indices, int64_t n_indices, int B, int Hkv,
                               int heads_per_kv, int Sq, int Skv, int q_block, int kv_block, int causal,
                               const uint32_t* kv_valid_bits, bfa_plan** out, void* stream);

/*
 * Plan from an exact-block bitmap (flashinfer block_sparse_attention,
 * sparse_format "bitmask", exact_block_bits).
 *   block_bits [B, Hkv, ceil(Sq/q_block), ceil(nkb/32)] u32 with
 *   nkb = ceil(Skv/kv_block): bit j % 32 of word j / 32 of row (b, hkv, i) selects
 *   KV block j for query block i (LSB first).  q_block, kv_block, causal and
 *   kv_valid_bits as for bfa_plan_bsr.  The structural KV-block count is the
 *   capacity bound.  Reads the plan size back once (one sync).
 */
bfa_status bfa_plan_block_bits(const uint32_t* block_bits, int B, int Hkv, int Sq, int Skv, int q_block,
                               int kv_block, int causal, const uint32_t* kv_valid_bits, bfa_plan** out,
                               void* stream);

/*
 * Fused masked attention forward with a prebuilt plan.
 *   q: batched [B, Sq, H, D] or packed [total_q, H, D]; k, v: [B, Sk, Hkv, D] or
 *   [total_k, Hkv, D]; bf16; the D axis contiguous.  *_strides = {batch, token,
 *   head} in elements (batch stride ignored for packed plans); strides and base
 *   addresses must be multiples of 16 bytes.
 *   H % Hkv == 0 (query head h reads kv head h / (H / Hkv)); D in {64, 128}.
 *   scale <= 0 selects 1/sqrt(D).
 *   out: caller-owned bf16, same logical shape as q, strides o_strides.
 *   lse: caller-owned f32 or NULL; batched [B, H, Sq], packed [H, total_q],
 *   natural log.  Rows with no attended key get out = 0 and lse = -inf.
 *   For dense plans B is free; otherwise B must equal the plan's batch /
 *   sequence count, and for BSR plans Hkv must equal the routing's.
 * Asynchronous: a device-side timeout is reported by bfa_plan_device_status().
 */
bfa_status bfa_fwd(const bfa_plan* plan, const void* q, const void* k, const void* v,
                   const int64_t q_strides[3], const int64_t k_strides[3], const int64_t v_strides[3],
                   int B, int H, int Hkv, int D, float scale, void* out, const int64_t o_strides[3],
                   float* lse, void* stream);

/*
 * Backward of bfa_fwd (BinFlash: two passes, dK/dV over key blocks and dQ over
 * query blocks; tensorplay varlen: the forward's log-sum-exp serves the backward
 * again): for an upstream gradient dout of `out`,
 *   dV = P^T dO,  dS = P * (dO V^T - D),  D_i = dO_i . O_i,
 *   dQ = scale dS K,  dK = scale dS^T Q,  P = exp(scale Q K^T - LSE) on attended pairs.
 *   q, k, v, out, lse, scale, B, H, Hkv, D and the plan: exactly as given to (and
 *   produced by) bfa_fwd.  dout: bf16, the layout of q (do_strides); dq, dk, dv:
 *   caller-owned bf16 outputs shaped like q, k, v (their own strides), fully
 *   written (rows that attend nothing, or keys nothing attends, get 0).  Under
 *   GQA dk and dv sum over the query heads of each kv head.  All strides
 *   {batch, token, head} in elements, multiples of 8; bases 16-byte aligned.
 * The first call on a plan builds its transposed lists (bfa_plan_export_cols) on
 * `stream`; a per-call workspace comes from the plan's stream-ordered pool: 8
 * bytes per (replica, query row of the plan's tiles), plus 4 * D bytes for the
 * fused pass.  Asynchronous; a device-side timeout is reported by
 * bfa_plan_device_status().  Paged caches are not accepted here.
 * Forms: D = 128 runs one fused pass over the key-tile columns (S and dP made
 * once per pair; dQ summed across key tiles by fp32 reductions into the
 * workspace, then scaled into dq), whose dq is not bitwise reproducible from run
 * to run (the order of the fp32 sums varies); dk and dv are.  D = 64, and every D
 * after bfa_set_bwd_deterministic(1), run the two passes (dK/dV over key-tile
 * columns, dQ over query-tile rows), bitwise reproducible.
 */
bfa_status bfa_bwd(const bfa_plan* plan, const void* q, const void* k, const void* v, const void* out,
                   const void* dout, const float* lse, const int64_t q_strides[3], const int64_t k_strides[3],
                   const int64_t v_strides[3], const int64_t o_strides[3], const int64_t do_strides[3], int B, int H,
                   int Hkv, int D, float scale, void* dq, void* dk, void* dv, const int64_t dq_strides[3],
                   const int64_t dk_strides[3], const int64_t dv_strides[3], void* stream);

/*
 * bfa_fwd with content-based block skipping (BinFlash approximate_softmax +
 * softmax_threshold, "BLASST-style"): once a query tile's scores are computed,
 * a key tile is dropped -- no exponentials, no P V product -- when every query
 * row of the tile has all its scores in that key tile more than
 * softmax_threshold (natural-log units, > 0) below the row's running maximum.
 * Each dropped weight is then below exp(-softmax_threshold) relative to the
 * row's final maximum weight, so per row the output moves by at most
 * 2 * n_dropped * exp(-softmax_threshold) * max|v| and the LSE by at most
 * n_dropped * exp(-softmax_threshold).  The first tile of a row is never dropped.
 * Everything else as for bfa_fwd.  An approximation: the result differs from
 * bfa_fwd whenever a tile is dropped.
 */
bfa_status bfa_fwd_approx(const bfa_plan* plan, const void* q, const void* k, const void* v,
                          const int64_t q_strides[3], const int64_t k_strides[3], const int64_t v_strides[3],
                          int B, int H, int Hkv, int D, float scale, float softmax_threshold, void* out,
                          const int64_t o_strides[3], float* lse, void* stream);

/*
 * bfa_fwd with keys and values in a paged cache (tensorplay varlen block_table):
 * the cache need not be contiguous per sequence.
 *   k_cache, v_cache: bf16 [num_pages, page_size, Hkv, D] with the same strides
 *   cache_strides = {page, token, head} in elements (pages contiguous: page
 *   stride = page_size * token stride; D contiguous).
 *   block_table: device i32 [n_seq, pages_per_seq]; key token t of sequence s
 *   (batch entry s of a batched or dense plan, sequence s of a varlen plan) is
 *   row t % page_size of page block_table[s, t / page_size].  Entries past a
 *   sequence's keys are not read.  page_size in {8, 16, 32, 64} or a multiple of
 *   128; pages_per_seq * page_size must cover the plan's longest key range.
 *   Everything else as for bfa_fwd (the plan's key lengths bound the keys).
 */
bfa_status bfa_fwd_paged(const bfa_plan* plan, const void* q, const int64_t q_strides[3], const void* k_cache,
                         const void* v_cache, const int64_t cache_strides[3], int64_t num_pages, int page_size,
                         const int32_t* block_table, int pages_per_seq, int B, int H, int Hkv, int D,
                         float scale, void* out, const int64_t o_strides[3], float* lse, void* stream);

/* Host-side plan description (no sync). */
bfa_status bfa_plan_get_info(const bfa_plan* plan, bfa_plan_info* info);

/* Tile statistics over the whole class grid (BinFlash's dispatch statistics);
 * synchronises `stream`.  n_full + n_partial = number of listed tiles. */
bfa_status bfa_plan_stats(const bfa_plan* plan, int64_t* n_full, int64_t* n_partial, int64_t* n_empty,
                          void* stream);

/*
 * Copy a plan to HOST buffers (for parity checks); synchronises `stream`.
 * Sizes: row_ptr [n_rows + 1], kv_tile / partial [n_full + n_partial],
 * fine [n_partial * 512] uint32 (plans with packed_fine; partial tiles in list
 * order, 128 rows x 4 words each) or NULL, order [n_rows] (longest row first, ties by row
 * index), classes [grid_tiles] (0 empty, 1 partial, 2 full; groups in order,
 * each group row-major over (query tile, key tile)).  Any pointer may be NULL.
 */
bfa_status bfa_plan_export(const bfa_plan* plan, int32_t* row_ptr, int32_t* kv_tile, uint8_t* partial,
                           uint32_t* fine, int32_t* order, uint8_t* classes, void* stream);

/* Copy the plan's work pairs to HOST buffers (synchronises `stream`).  A work
 * pair is two consecutive query tiles (2i, 2i+1) of one group that one CTA of the
 * forward can run together; pair_row [n_pairs] holds the first row, bit-inverted
 * (~row) when the group has no second tile; pair_order [n_pairs] lists the pairs
 * longest first (by their total listed tiles), ties by pair index.  Either pointer
 * may be NULL. */
bfa_status bfa_plan_export_pairs(const bfa_plan* plan, int32_t* pair_row, int32_t* pair_order, void* stream);

/* Copy the plan's transposed lists to HOST buffers (built on first use, on
 * `stream`; synchronises it).  For the backward's key-tile pass (BinFlash's
 * dK/dV pass over key blocks): column c (group g, key tile kt; groups in order, key
 * tiles ascending) lists the query tiles whose tile (qt, kt) is not empty,
 * ascending, in q_tile[col_ptr[c] .. col_ptr[c+1]); tpart holds -1 for full tiles
 * and, for partial ones, the index of their packed fine words (the same index the
 * row lists' partial entries use); col_order [n_cols] lists the columns longest
 * first, ties by column index.  Sizes: col_ptr n_cols + 1, q_tile and tpart
 * col_ptr[n_cols], col_order n_cols (bfa_plan_info.n_cols).  Any pointer may be
 * NULL. */
bfa_status bfa_plan_export_cols(const bfa_plan* plan, int32_t* col_ptr, int32_t* q_tile, int32_t* tpart,
                                int32_t* col_order, void* stream);

/* Synchronise `stream` and report BFA_ERR_TIMEOUT if a kernel that used the plan
 * hit its wait bound since the last call (the flag is then cleared).
 * The checked build of the library (libbfa_checked.so, compiled with
 * -DBFA_CHECKED: a stand-in for a memory checker) also bounds-checks every
 * plan-indexed access of its kernels, skipping the access and flagging it, and
 * surrounds every plan array with guard bytes; this call then first verifies the
 * guard bytes and reports BFA_ERR_BOUNDS if an index left its array or a guard
 * was overwritten (the flags are then cleared). */
bfa_status bfa_plan_device_status(const bfa_plan* plan, void* stream);

/* Free a plan in stream order on the stream it was built on.  Work on other
 * streams that reads the plan must be ordered before this call.  NULL is a no-op. */
void bfa_plan_destroy(bfa_plan* plan);

/* Bound, in nanoseconds, on the device-side waits inside the kernels' loops
 * (a TMA copy, a product or another role of the block that does not arrive),
 * for kernels launched after this call: default 1e9, i.e. one second; 0 restores
 * the default; other values are clamped to [BFA_WAIT_NS_MIN, BFA_WAIT_NS_MAX].
 * Past the bound the block stops its work, and the plan's device status reports
 * BFA_ERR_TIMEOUT (bfa_plan_device_status).  The waits that keep a block alive
 * until the copies and products it has already issued are complete (before it
 * releases tensor memory and exits) do not follow this bound: they have a fixed
 * bound of 4 s, and those phases complete by themselves within microseconds. */
#define BFA_WAIT_NS_MIN 1000ull
#define BFA_WAIT_NS_MAX 60000000000ull
void bfa_set_wait_timeout_ns(uint64_t ns);

/* Backward form for calls made after this one (process-wide): on != 0 makes
 * bfa_bwd use the two-pass form for every head dim, so that its results are
 * bitwise reproducible; 0 (the default) lets D = 128 use the fused pass. */
void bfa_set_bwd_deterministic(int on);

/* Launch a one-thread-block kernel that waits, with the current bound, on a
 * barrier phase that nothing completes, and synchronise.  Returns
 * BFA_ERR_TIMEOUT when the bounded wait gives up as designed (and the context
 * stays usable), BFA_OK never.  Exercises the failure path without a fault. */
bfa_status bfa_selftest_wait_timeout(void* stream);

/*
 * Dense-mask planner that allocates nothing.  The source pages have no
 * counterpart: this entry point exists for callers that cannot let a library
 * allocate device memory -- for example a serving process whose memory manager
 * reserves the whole GPU up front, or code that must keep a fixed device-memory
 * footprint.  It computes the same plan as bfa_plan_dense, but as plain arrays
 * in buffers the caller owns, and calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *   Inputs: mask / mask_row_stride / Sq / Sk as for bfa_plan_dense.
 *   Outputs (device, caller-owned; nqt = ceil(Sq/128), nkt = ceil(Sk/128)):
 *     classes [nqt * nkt] u8 (0 empty, 1 partial, 2 full), row_ptr [nqt + 1],
 *     kv_tile [nqt * nkt] i32 and part [nqt * nkt] i32 (-1 full, else the tile's
 *     index in classes), used up to row_ptr[nqt]; fine [nqt * nkt * 512] u32,
 *     written at the class-grid index of every partial tile; order [nqt].
 *   Limits: nqt <= BFA_NOALLOC_MAX_ROWS and nkt <= BFA_NOALLOC_MAX_KV_TILES, else
 *     BFA_ERR_CAPACITY before anything is launched.
 * Its scratch (group table, row map, per-row counts: 256 + 8 * BFA_NOALLOC_MAX_ROWS
 * bytes) is a device array inside the library that every GPU loading the library
 * holds until exit.  The first call on a device looks up that array's address,
 * so make that first call before any stream capture.  All calls share the one
 * array: calls that overlap on the GPU (on different streams) race and must be
 * ordered by the caller.  Each call writes every scratch word it reads, so the
 * previous call's contents do not matter.  After a device reset
 * (cudaDeviceReset) the array may move: call bfa_is_available() once on that
 * device before this entry point's next call there, which then looks the
 * address up again (so it, too, must come before any stream capture).
 * Stream-ordered, no synchronisation.
 */
enum { BFA_NOALLOC_MAX_ROWS = 4096, BFA_NOALLOC_MAX_KV_TILES = 16384 };
bfa_status bfa_plan_dense_noalloc(const uint8_t* mask, int64_t mask_row_stride, int Sq, int Sk,
                                  uint8_t* classes, int32_t* row_ptr, int32_t* kv_tile, int32_t* part,
                                  uint32_t* fine, int32_t* order, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BFA_H_ */
