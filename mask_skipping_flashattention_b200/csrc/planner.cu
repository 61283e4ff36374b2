// Mask planner kernels: turn a dense mask, block ids / positions, or BSR routing
// into the tile plan (class grid -> per-row ascending key-tile lists -> longest
// first row order), plus packed fine masks for the partial tiles of dense masks.
//
// The method is BinFlash's preprocessing ("Efficiently Dispatching FlashAttention
// For Partially Filled Attention Masks": a coarse per-block mask, the partial
// blocks' bits packed 32 to a word, and sorted lists of the non-empty key blocks), with the block-id rule of
// opentau flash_attn_cuda and the BSR routing of flashinfer block_sparse_attention
// as the other two mask sources.  Everything is deterministic: counts are integer
// reductions, lists come from ballot prefix sums, and the order is a stable
// counting sort.
#include <cstdint>
#include <cuda_runtime.h>

#include "plan_types.cuh"
#include "pred.cuh"

namespace bfa {

// ----------------------------------------------------------------------------
// dense mask -> classes + fine words
// ----------------------------------------------------------------------------
// Grid (ceil(nkt / 4), nqt); 256 threads.  A CTA reads a 128-row band of 4 key
// tiles (512 columns): lane L of a warp covers 16 columns (tile L / 8, chunk L % 8)
// with one 16-byte load per row, so each warp instruction reads 512 contiguous
// mask bytes.  Each warp owns 16 rows.
constexpr int kDenseTilesPerCta = 4;
constexpr size_t kRowsStageBytes = 160 * 1024;  // k_rows: largest staged group table + row map + class grid

__device__ __forceinline__ uint32_t nz_bytes4(uint32_t x) {
  // bit k (k < 4) set iff byte k of x is nonzero
  uint32_t t = x | (x >> 4);
  t |= t >> 2;
  t |= t >> 1;
  t &= 0x01010101u;
  return ((t * 0x01020408u) >> 24) & 0xFu;
}

// Optional set-up of a dense plan done by the classify launch itself (one
// launch fewer): its single group, the row -> group map and the status words.
struct DenseInit {
  GroupInfo* groups;  // nullptr: nothing to do
  GroupInfo group;
  int32_t* row_group;
  uint32_t* err;
  int32_t* max_width;
};

__global__ void __launch_bounds__(256) k_dense_classify(const uint8_t* __restrict__ mask, int64_t ld, int Sq,
                                                        int Sk, int nkt, uint8_t* __restrict__ cls,
                                                        uint32_t* __restrict__ fine, int vec_ok,
                                                        const DenseInit init) {
  __shared__ uint32_t words[kDenseTilesPerCta][kTile][kWordsPerTileRow];  // 8 KB
  __shared__ int tile_cnt[kDenseTilesPerCta];
  const int qt = blockIdx.y;
  const int kt0 = blockIdx.x * kDenseTilesPerCta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < kDenseTilesPerCta) tile_cnt[threadIdx.x] = 0;
  if (init.groups != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
    init.row_group[qt] = 0;
    if (qt == 0) {
      *init.groups = init.group;
      *init.err = 0u;
      *init.max_width = 0;
    }
  }
  const int t = lane >> 3, chunk = lane & 7;
  const int64_t col0 = static_cast<int64_t>(kt0 + t) * kTile + chunk * 16;
  const int rows_here = min(kTile, Sq - qt * kTile);

  uint32_t m16[16];
  // A CTA whose 128 rows x 512 bytes all lie inside the mask (every CTA but those
  // on the ragged edges) issues its 16 row loads per thread before using any of
  // them, so that they are all in flight at once; the edge path below checks
  // each row and column.
  const bool inside = vec_ok && rows_here == kTile && (kt0 + kDenseTilesPerCta) * kTile <= Sk;
  if (inside) {
    uint4 v[16];
    const uint8_t* base = mask + static_cast<int64_t>(qt * kTile + warp * 16) * ld + col0;
#pragma unroll
    for (int rr = 0; rr < 16; ++rr) v[rr] = __ldg(reinterpret_cast<const uint4*>(base + rr * ld));
#pragma unroll
    for (int rr = 0; rr < 16; ++rr) {
      const uint4 x = v[rr];
      if (((x.x | x.y | x.z | x.w) & 0xFEFEFEFEu) == 0u) {
        m16[rr] = ((x.x * 0x01020408u) >> 24) | (((x.y * 0x01020408u) >> 24) << 4) |
                  (((x.z * 0x01020408u) >> 24) << 8) | (((x.w * 0x01020408u) >> 24) << 12);
      } else {
        m16[rr] = nz_bytes4(x.x) | (nz_bytes4(x.y) << 4) | (nz_bytes4(x.z) << 8) | (nz_bytes4(x.w) << 12);
      }
    }
  } else {
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) {
    const int r = warp * 16 + rr;
    uint32_t m = 0;
    if (r < rows_here && col0 < Sk) {
      const uint8_t* p = mask + static_cast<int64_t>(qt * kTile + r) * ld + col0;
      if (vec_ok && col0 + 16 <= Sk) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        if (((v.x | v.y | v.z | v.w) & 0xFEFEFEFEu) == 0u) {
          // bytes 0 / 1 (a bool tensor): one multiply gathers bit 0 of the four bytes
          // of a word into bits 24..27, in byte order (no carries between the terms)
          m = ((v.x * 0x01020408u) >> 24) | (((v.y * 0x01020408u) >> 24) << 4) |
              (((v.z * 0x01020408u) >> 24) << 8) | (((v.w * 0x01020408u) >> 24) << 12);
        } else {
          m = nz_bytes4(v.x) | (nz_bytes4(v.y) << 4) | (nz_bytes4(v.z) << 8) | (nz_bytes4(v.w) << 12);
        }
      } else {
        for (int c = 0; c < 16; ++c)
          if (col0 + c < Sk && p[c] != 0) m |= 1u << c;
      }
    }
    m16[rr] = m;
  }
  }
  int cnt = 0;
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) {
    const uint32_t hi = __shfl_down_sync(0xffffffffu, m16[rr], 1);
    cnt += __popc(m16[rr]);
    if ((chunk & 1) == 0) words[t][warp * 16 + rr][chunk >> 1] = m16[rr] | (hi << 16);
  }
  // reduce the counts of the 8 lanes of each tile
  cnt += __shfl_xor_sync(0xffffffffu, cnt, 1);
  cnt += __shfl_xor_sync(0xffffffffu, cnt, 2);
  cnt += __shfl_xor_sync(0xffffffffu, cnt, 4);
  __syncthreads();  // tile_cnt zeroed
  if (chunk == 0) atomicAdd(&tile_cnt[t], cnt);
  __syncthreads();
  for (int tt = 0; tt < kDenseTilesPerCta; ++tt) {
    const int kt = kt0 + tt;
    if (kt >= nkt) break;
    const int cols = min(kTile, Sk - kt * kTile);
    const int n_in = rows_here * cols;
    const int c = tile_cnt[tt];
    const int klass = (c == 0) ? 0 : (c == n_in ? 2 : 1);
    const int64_t gidx = static_cast<int64_t>(qt) * nkt + kt;
    if (threadIdx.x == 0) cls[gidx] = static_cast<uint8_t>(klass);
    if (klass == 1) {
      uint32_t* dst = fine + gidx * kFineWordsPerTile;
      const uint32_t* src = &words[tt][0][0];
      for (int i = threadIdx.x; i < kFineWordsPerTile; i += blockDim.x) dst[i] = src[i];
    }
  }
}

// ----------------------------------------------------------------------------
// block ids / positions -> padded id copies + classes (one CTA per group)
// ----------------------------------------------------------------------------
struct TileStat {
  int32_t lo, hi;   // min / max id over valid in-range tokens of the tile
  int32_t any, all; // any valid, all in-range tokens valid
};

__device__ __forceinline__ void warp_minmax(int32_t& lo, int32_t& hi, int32_t& any, int32_t& all) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  any = __any_sync(0xffffffffu, any);
  all = __all_sync(0xffffffffu, all);
}

// Stats of one tile of `len` tokens starting at local index `t0`; copies the ids
// and validity into the padded arrays when requested.  One warp.
__device__ TileStat tile_stats(const int32_t* ids, const uint8_t* valid, int tok0, int len, int t0,
                               int32_t* out_id, uint8_t* out_valid, uint32_t* out_bits, int lane) {
  int32_t lo = INT32_MAX, hi = INT32_MIN, any = 0, all = 1;
  for (int c = 0; c < kTile / 32; ++c) {
    const int j = t0 + c * 32 + lane;   // local index
    const bool in = j < len;
    int32_t id = in ? (ids ? ids[tok0 + j] : j) : INT32_MAX;
    const bool v = in && (valid ? valid[tok0 + j] != 0 : true);
    if (v) {
      lo = min(lo, id);
      hi = max(hi, id);
      any = 1;
    }
    if (in && !v) all = 0;
    if (out_id) out_id[t0 + c * 32 + lane] = in ? id : INT32_MAX;
    if (out_valid) out_valid[t0 + c * 32 + lane] = v ? 1 : 0;
    const uint32_t bits = __ballot_sync(0xffffffffu, v);
    if (out_bits && lane == 0) out_bits[(t0 >> 5) + c] = bits;
  }
  warp_minmax(lo, hi, any, all);
  return TileStat{lo, hi, any, all};
}

__global__ void __launch_bounds__(256) k_blockid_classify(const GroupInfo* __restrict__ groups,
                                                          const int32_t* __restrict__ q_blk,
                                                          const int32_t* __restrict__ k_blk,
                                                          const uint8_t* __restrict__ q_valid,
                                                          const uint8_t* __restrict__ k_valid, int batched,
                                                          int Sq, int Sk, int window, int copy_ids,
                                                          int32_t* qid, uint8_t* qv, int32_t* kid,
                                                          uint32_t* kbits, uint8_t* cls) {
  extern __shared__ TileStat st[];  // nqt + nkt entries
  const GroupInfo g = groups[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  // token offsets of the group inside the caller's id / validity arrays
  const int qtok = batched ? g.b * Sq : g.q_off;
  const int ktok = batched ? g.b * Sk : g.k_off;
  TileStat* sq = st;
  TileStat* sk = st + g.nqt;
  for (int qt = warp; qt < g.nqt; qt += nw)
    sq[qt] = tile_stats(q_blk, q_valid, qtok, g.q_len, qt * kTile, copy_ids ? qid + g.qid_off : nullptr,
                        copy_ids ? qv + g.qid_off : nullptr, nullptr, lane);
  for (int kt = warp; kt < g.nkt; kt += nw)
    sk[kt] = tile_stats(k_blk, k_valid, ktok, g.k_len, kt * kTile, copy_ids ? kid + g.kid_off : nullptr,
                        nullptr, copy_ids ? kbits + g.kbit_off : nullptr, lane);
  __syncthreads();
  const int64_t n = static_cast<int64_t>(g.nqt) * g.nkt;
  for (int64_t e = threadIdx.x; e < n; e += blockDim.x) {
    const int qt = static_cast<int>(e / g.nkt), kt = static_cast<int>(e % g.nkt);
    const TileStat a = sq[qt], b = sk[kt];
    // attend(i, j) = valid_i & valid_j & id_j <= id_i   [& i - j < window on positions]
    bool exists = a.any && b.any && b.lo <= a.hi;
    bool full = a.all && b.all && b.hi <= a.lo;
    if (window >= 0) {
      // positions: i - j ranges over [lo_q - hi_k, hi_q - lo_k] without gaps
      exists = exists && (a.lo - b.hi) < window;
      full = full && (a.hi - b.lo) < window;
    }
    cls[g.cls_off + e] = static_cast<uint8_t>(exists ? (full ? 2 : 1) : 0);
  }
}

// ----------------------------------------------------------------------------
// BSR routing -> validation + classes (one thread per BSR row)
// ----------------------------------------------------------------------------
__global__ void k_bsr_classify(const int32_t* __restrict__ indptr, const int32_t* __restrict__ indices,
                               int64_t n_indices, const GroupInfo* __restrict__ groups, int n_groups,
                               int nqt, int causal, uint8_t* cls, uint32_t* err, int32_t* max_width) {
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= static_cast<int64_t>(n_groups) * nqt) return;
  const int grp = static_cast<int>(gid / nqt), qt = static_cast<int>(gid % nqt);
  const GroupInfo g = groups[grp];
  const int32_t* ip = indptr + static_cast<int64_t>(grp) * (nqt + 1);
  const int32_t a = ip[qt], b = ip[qt + 1];
  if (a < 0 || b < a || static_cast<int64_t>(b) > n_indices) {
    atomicOr(err, DEVERR_BSR_RANGE);
    return;
  }
  atomicMax(max_width, b - a);
  const int i0 = qt * kTile, i1 = min(g.q_len, i0 + kTile) - 1;
  int32_t prev = -1;
  for (int32_t e = a; e < b; ++e) {
    const int32_t kt = indices[e];
    if (kt <= prev || kt >= g.nkt) {
      atomicOr(err, DEVERR_BSR_ORDER);
      return;
    }
    prev = kt;
    int klass = 2;
    if (causal) {
      const int j0 = kt * kTile, j1 = min(g.k_len, j0 + kTile) - 1;
      klass = (j0 > i1) ? 0 : (j1 <= i0 ? 2 : 1);
    }
    cls[g.cls_off + static_cast<int64_t>(qt) * g.nkt + kt] = static_cast<uint8_t>(klass);
  }
}

// ----------------------------------------------------------------------------
// classes -> CSR lists + longest-first orders (one CTA of 1024 threads)
// ----------------------------------------------------------------------------
// Exclusive prefix sum over n values read through `get(i)`; out[i] = sum of the
// values before i; returns the total.  All threads of the CTA call it.
template <typename Get>
__device__ int block_exclusive_scan(int n, Get get, int32_t* out, int32_t* warp_sums, int32_t* carry) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) *carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + tid;
    const int v = i < n ? get(i) : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_sums[lane] = w;
    }
    __syncthreads();
    const int incl = x + (warp ? warp_sums[warp - 1] : 0) + *carry;
    if (i < n) out[i] = incl - v;
    __syncthreads();
    if (tid == blockDim.x - 1) *carry = incl;
    __syncthreads();
  }
  const int total = *carry;
  __syncthreads();
  return total;
}

// Stable sort of the indices 0..n-1 by descending key (keys in [0, max_key]):
// a counting sort whose placement runs chunk by chunk and warp by warp, so equal
// keys keep index order.  `bucket` is shared memory of max_key + 1 ints.
__device__ void block_stable_order_desc(int n, const int32_t* keys, int max_key, int32_t* bucket,
                                        int32_t* order) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int i = tid; i <= max_key; i += blockDim.x) bucket[i] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += blockDim.x) atomicAdd(&bucket[keys[i]], 1);
  __syncthreads();
  if (tid == 0) {  // bucket[k] <- first output slot of key k
    int acc = 0;
    for (int k = max_key; k >= 0; --k) {
      const int h = bucket[k];
      bucket[k] = acc;
      acc += h;
    }
  }
  __syncthreads();
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + tid;
    const int key = i < n ? keys[i] : -1;
    const uint32_t same = __match_any_sync(0xffffffffu, key);
    const int rank = __popc(same & lt_mask);
    for (int w = 0; w < nw; ++w) {
      if (warp == w && key >= 0) order[bucket[key] + rank] = i;
      __syncthreads();
      if (warp == w && key >= 0 && rank == 0) bucket[key] += __popc(same);
      __syncthreads();
    }
  }
}

// The same order for n <= kSmallOrder keys: every thread ranks its own element
// directly (larger keys first, ties by index) against the keys in shared memory;
// cheaper than the bucket passes for the few hundred rows most plans have.
constexpr int kSmallOrder = 256;
__device__ void block_stable_order_desc_small(int n, const int32_t* keys, int32_t* skeys, int32_t* order) {
  const int tid = threadIdx.x;
  if (tid < n) skeys[tid] = keys[tid];
  __syncthreads();
  if (tid < n) {
    const int k = skeys[tid];
    int rank = 0;
    for (int j = 0; j < n; ++j) {
      const int kj = skeys[j];
      rank += (kj > k || (kj == k && j < tid)) ? 1 : 0;
    }
    order[rank] = tid;
  }
  __syncthreads();
}

// Rows -> lists and row order; with pair outputs also the work pairs (two
// consecutive query tiles of one group) and their longest-first order.
// Dynamic shared memory: (2 * max_nkt + 1) ints.
__global__ void __launch_bounds__(1024) k_rows(const GroupInfo* __restrict__ groups,
                                               const int32_t* __restrict__ row_group,
                                               const uint8_t* __restrict__ cls, int n_rows, int max_nkt,
                                               int32_t* __restrict__ row_cnt, int32_t* __restrict__ row_ptr,
                                               int32_t* __restrict__ kv_tile, int32_t* __restrict__ part,
                                               int32_t* __restrict__ order, int32_t* __restrict__ pair_row,
                                               int32_t* __restrict__ pair_cost, int32_t* __restrict__ pair_order,
                                               int32_t* __restrict__ pair_idx, int part_is_pos,
                                               int2* __restrict__ row_work, int2* __restrict__ pair_work,
                                               int n_groups, int64_t grid_tiles, int stage) {
  extern __shared__ __align__(16) int32_t bucket[];
  __shared__ int32_t small_keys[kSmallOrder];
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;

  // 0. with `stage`, the group table, the row -> group map and the class grid are
  //    copied to shared memory first (coalesced), so that the per-row passes
  //    below read them there instead of in dependent global loads; the area is
  //    reused by the sort buckets from step 4 on
  const GroupInfo* sgroups = groups;
  const int32_t* srow_group = row_group;
  const uint8_t* scls = cls;
  if (stage) {
    GroupInfo* g_s = reinterpret_cast<GroupInfo*>(bucket);
    int32_t* rg_s = reinterpret_cast<int32_t*>(g_s + n_groups);
    uint8_t* c_s = reinterpret_cast<uint8_t*>(rg_s + n_rows);
    const int32_t* gw = reinterpret_cast<const int32_t*>(groups);
    int32_t* gws = reinterpret_cast<int32_t*>(g_s);
    for (int i = tid; i < n_groups * static_cast<int>(sizeof(GroupInfo) / 4); i += blockDim.x) gws[i] = gw[i];
    for (int i = tid; i < n_rows; i += blockDim.x) rg_s[i] = row_group[i];
    const int64_t n16 = grid_tiles >> 4;  // the class grid starts 256-byte aligned in the plan slab
    const uint4* c16 = reinterpret_cast<const uint4*>(cls);
    for (int64_t i = tid; i < n16; i += blockDim.x) {
      const uint4 v = c16[i];
      uint8_t* d = c_s + 16 * i;
      reinterpret_cast<uint32_t*>(d)[0] = v.x;  // c_s is 4-byte aligned
      reinterpret_cast<uint32_t*>(d)[1] = v.y;
      reinterpret_cast<uint32_t*>(d)[2] = v.z;
      reinterpret_cast<uint32_t*>(d)[3] = v.w;
    }
    for (int64_t i = 16 * n16 + tid; i < grid_tiles; i += blockDim.x) c_s[i] = cls[i];
    __syncthreads();
    sgroups = g_s;
    srow_group = rg_s;
    scls = c_s;
  }

  // 1. count the listed tiles of every row (warp per row, ballot + popc)
  for (int r = warp; r < n_rows; r += nw) {
    const GroupInfo g = sgroups[srow_group[r]];
    const uint8_t* c = scls + g.cls_off + static_cast<int64_t>(r - g.row0) * g.nkt;
    int n = 0;
    for (int k0 = 0; k0 < g.nkt; k0 += 32) {
      const int kt = k0 + lane;
      n += __popc(__ballot_sync(0xffffffffu, kt < g.nkt && c[kt] != 0));
    }
    if (lane == 0) row_cnt[r] = n;
  }
  __syncthreads();

  // 2. exclusive scan of the counts -> row_ptr
  const int total = block_exclusive_scan(n_rows, [&](int i) { return row_cnt[i]; }, row_ptr, warp_sums, &carry);
  if (tid == 0) row_ptr[n_rows] = total;
  __syncthreads();

  // 3. write each row's ascending list (warp per row)
  for (int r = warp; r < n_rows; r += nw) {
    const GroupInfo g = sgroups[srow_group[r]];
    const int64_t rowoff = g.cls_off + static_cast<int64_t>(r - g.row0) * g.nkt;
    const uint8_t* c = scls + rowoff;
    int out = row_ptr[r];
    for (int k0 = 0; k0 < g.nkt; k0 += 32) {
      const int kt = k0 + lane;
      const int klass = kt < g.nkt ? c[kt] : 0;
      const uint32_t bal = __ballot_sync(0xffffffffu, klass != 0);
      if (klass != 0) {
        const int pos = out + __popc(bal & lt_mask);
        kv_tile[pos] = kt;
        part[pos] = (klass == 1) ? (part_is_pos ? pos : static_cast<int32_t>(rowoff + kt)) : -1;
      }
      out += __popc(bal);
    }
  }

  // 4. longest-first stable row order
  __syncthreads();
  if (n_rows <= kSmallOrder) block_stable_order_desc_small(n_rows, row_cnt, small_keys, order);
  else block_stable_order_desc(n_rows, row_cnt, max_nkt, bucket, order);
  // work items in that order with the group of their row, so a kernel finds its
  // row and group with one load
  if (row_work != nullptr)
    for (int i = tid; i < n_rows; i += blockDim.x) row_work[i] = make_int2(order[i], row_group[order[i]]);
  if (pair_row == nullptr) return;

  // 5. pairs: a row opens a pair when its tile index inside its group is even;
  //    pair_row = first row (bit-inverted when the pair has a single row)
  auto opens = [&](int r) {
    const GroupInfo g = groups[row_group[r]];
    return ((r - g.row0) & 1) == 0 ? 1 : 0;
  };
  const int n_pairs = block_exclusive_scan(n_rows, opens, pair_idx, warp_sums, &carry);
  for (int r = tid; r < n_rows; r += blockDim.x) {
    const GroupInfo g = groups[row_group[r]];
    if (((r - g.row0) & 1) != 0) continue;
    const bool two = r + 1 < g.row0 + g.nqt;
    const int pi = pair_idx[r];
    pair_row[pi] = two ? r : ~r;
    pair_cost[pi] = row_cnt[r] + (two ? row_cnt[r + 1] : 0);
  }
  __syncthreads();
  if (n_pairs <= kSmallOrder) block_stable_order_desc_small(n_pairs, pair_cost, small_keys, pair_order);
  else block_stable_order_desc(n_pairs, pair_cost, 2 * max_nkt, bucket, pair_order);
  if (pair_work != nullptr)
    for (int i = tid; i < n_pairs; i += blockDim.x) {
      const int pr = pair_row[pair_order[i]];
      pair_work[i] = make_int2(pr, row_group[pr >= 0 ? pr : ~pr]);
    }
}

// Transposed lists for the backward's key-tile pass (BinFlash's dK/dV pass over
// key blocks): for every key-tile column (group g, key tile kt), the ascending
// query tiles whose class is not empty, each with its fine-word index when the
// tile is partial (-1 when full), and the columns in longest-first order.
// One CTA of 1024 threads; dynamic shared memory: max_nqt + 1 ints.
__global__ void __launch_bounds__(1024) k_cols(const GroupInfo* __restrict__ groups, int n_groups,
                                               const uint8_t* __restrict__ cls, const int32_t* __restrict__ row_ptr,
                                               const int32_t* __restrict__ kv_tile, int part_is_pos, int max_nqt,
                                               int n_cols, int32_t* __restrict__ col0, int32_t* __restrict__ col_group,
                                               int32_t* __restrict__ col_cnt, int32_t* __restrict__ col_ptr,
                                               int32_t* __restrict__ q_tile, int32_t* __restrict__ tpart,
                                               int32_t* __restrict__ col_order) {
  extern __shared__ int32_t bucket[];
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;

  // 1. first column of every group, and the group of every column
  const int total_cols = block_exclusive_scan(n_groups, [&](int g) { return groups[g].nkt; }, col0, warp_sums, &carry);
  if (tid == 0) col0[n_groups] = total_cols;
  __syncthreads();
  for (int c = tid; c < n_cols; c += blockDim.x) {
    int lo = 0, hi = n_groups - 1;  // last group whose first column is <= c
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (col0[mid] <= c) lo = mid;
      else hi = mid - 1;
    }
    col_group[c] = lo;
  }
  __syncthreads();

  // 2. listed query tiles per column (warp per column, ballot + popc)
  for (int c = warp; c < n_cols; c += nw) {
    const GroupInfo g = groups[col_group[c]];
    const int kt = c - col0[col_group[c]];
    const uint8_t* cc = cls + g.cls_off + kt;
    int n = 0;
    for (int q0 = 0; q0 < g.nqt; q0 += 32) {
      const int qt = q0 + lane;
      n += __popc(__ballot_sync(0xffffffffu, qt < g.nqt && cc[static_cast<int64_t>(qt) * g.nkt] != 0));
    }
    if (lane == 0) col_cnt[c] = n;
  }
  __syncthreads();

  // 3. exclusive scan -> col_ptr
  const int total = block_exclusive_scan(n_cols, [&](int i) { return col_cnt[i]; }, col_ptr, warp_sums, &carry);
  if (tid == 0) col_ptr[n_cols] = total;
  __syncthreads();

  // 4. ascending lists with the fine-word index of partial tiles
  for (int c = warp; c < n_cols; c += nw) {
    const int grp = col_group[c];
    const GroupInfo g = groups[grp];
    const int kt = c - col0[grp];
    int out = col_ptr[c];
    for (int q0 = 0; q0 < g.nqt; q0 += 32) {
      const int qt = q0 + lane;
      const int64_t cell = g.cls_off + static_cast<int64_t>(qt) * g.nkt + kt;
      const int klass = qt < g.nqt ? cls[cell] : 0;
      const uint32_t bal = __ballot_sync(0xffffffffu, klass != 0);
      if (klass != 0) {
        const int pos = out + __popc(bal & lt_mask);
        q_tile[pos] = qt;
        int32_t pi = -1;
        if (klass == 1) {
          if (part_is_pos) {  // fine words stored by list position: find kt in row (row0 + qt)
            const int r = g.row0 + qt;
            int lo = row_ptr[r], hi = row_ptr[r + 1] - 1;
            while (lo < hi) {
              const int mid = (lo + hi) >> 1;
              if (kv_tile[mid] < kt) lo = mid + 1;
              else hi = mid;
            }
            pi = lo;
          } else {
            pi = static_cast<int32_t>(cell);
          }
        }
        tpart[pos] = pi;
      }
      out += __popc(bal);
    }
  }

  // 5. longest-first stable column order
  __syncthreads();
  block_stable_order_desc(n_cols, col_cnt, max_nqt, bucket, col_order);
}

// ----------------------------------------------------------------------------
// generic block sparsity (any BSR block sizes, exact-block bitmaps, key validity)
// ----------------------------------------------------------------------------
// Block bitmap layout: [group][query block][wpr words], bit kb % 32 of word
// kb / 32 selects KV block kb.

// BSR rows -> block bitmap, validating canonical rows (one thread per row).
__global__ void k_bsr_to_bits(const int32_t* __restrict__ indptr, const int32_t* __restrict__ indices,
                              int64_t n_indices, int n_groups, int nqb, int nkb, int wpr, uint32_t* __restrict__ bits,
                              uint32_t* err) {
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= static_cast<int64_t>(n_groups) * nqb) return;
  const int grp = static_cast<int>(gid / nqb), qb = static_cast<int>(gid % nqb);
  const int32_t* ip = indptr + static_cast<int64_t>(grp) * (nqb + 1);
  const int32_t a = ip[qb], b = ip[qb + 1];
  if (a < 0 || b < a || static_cast<int64_t>(b) > n_indices) {
    atomicOr(err, DEVERR_BSR_RANGE);
    return;
  }
  uint32_t* row = bits + gid * wpr;
  int32_t prev = -1;
  for (int32_t e = a; e < b; ++e) {
    const int32_t kb = indices[e];
    if (kb <= prev || kb >= nkb) {
      atomicOr(err, DEVERR_BSR_ORDER);
      return;
    }
    prev = kb;
    row[kb >> 5] |= 1u << (kb & 31);
  }
}

struct BlockSparseArgs {
  const uint32_t* bits;      // block bitmap [group][nqb][wpr]
  const uint32_t* kv_valid;  // [batch][kv_wpb] token validity bits, or null
  int nqb, wpr, kv_wpb;
  int q_block, kv_block, causal;
  // GQA-packed query rows: plan row t of a group is query position t / g_pack of
  // head t % g_pack of its kv head (1: rows are positions)
  int g_pack;
};

// attend-bits of query position i (row of query block qb) over the 32 columns
// starting at c0 (a multiple of 32) of a group with k_len keys
__device__ __forceinline__ uint32_t block_word(const BlockSparseArgs& a, const uint32_t* rowbits,
                                               const uint32_t* kvrow, int i, int c0, int k_len) {
  if (c0 >= k_len) return 0u;
  uint32_t w;
  if (a.kv_block % 32 == 0) {  // the 32 columns lie in one KV block
    const int kb = c0 / a.kv_block;
    w = ((rowbits[kb >> 5] >> (kb & 31)) & 1u) ? 0xffffffffu : 0u;
  } else {                     // kv_block in {8, 16}: several blocks per word
    w = 0u;
    const uint32_t run = (1u << a.kv_block) - 1u;
    for (int c = 0; c < 32 && c0 + c < k_len; c += a.kv_block) {  // blocks past the end are never read
      const int kb = (c0 + c) / a.kv_block;
      if ((rowbits[kb >> 5] >> (kb & 31)) & 1u) w |= run << c;
    }
  }
  const int ncols = k_len - c0;
  if (ncols < 32) w &= (1u << ncols) - 1u;
  if (a.causal) {  // keep columns c0 + c <= i
    const int z = i - c0;
    w &= (z >= 31) ? 0xffffffffu : (z < 0 ? 0u : ((2u << z) - 1u));
  }
  if (kvrow) w &= kvrow[c0 >> 5];
  return w;
}

// Tile classes from the block bitmap: CTA per (group, query tile), thread per row.
__global__ void __launch_bounds__(128) k_bits_classify(BlockSparseArgs a, const GroupInfo* __restrict__ groups,
                                                       uint8_t* __restrict__ cls) {
  __shared__ int warp_cnt[4];
  const GroupInfo g = groups[blockIdx.x];
  const int qt = blockIdx.y;
  if (qt >= g.nqt) return;
  const int r = threadIdx.x, warp = r >> 5, lane = r & 31;
  const int t = qt * kTile + r;  // plan row
  const bool in = t < g.q_len;
  const int i = t / a.g_pack;    // query position
  const uint32_t* rowbits = a.bits + (static_cast<int64_t>(blockIdx.x) * a.nqb + (in ? i / a.q_block : 0)) * a.wpr;
  const uint32_t* kvrow = a.kv_valid ? a.kv_valid + static_cast<int64_t>(g.b) * a.kv_wpb : nullptr;
  const int rows_in = min(kTile, g.q_len - qt * kTile);
  for (int kt = 0; kt < g.nkt; ++kt) {
    int cnt = 0;
    if (in) {
#pragma unroll
      for (int w = 0; w < 4; ++w) cnt += __popc(block_word(a, rowbits, kvrow, i, kt * kTile + 32 * w, g.k_len));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) warp_cnt[warp] = cnt;
    __syncthreads();
    if (r == 0) {
      const int c = warp_cnt[0] + warp_cnt[1] + warp_cnt[2] + warp_cnt[3];
      const int n_in = rows_in * min(kTile, g.k_len - kt * kTile);
      cls[g.cls_off + static_cast<int64_t>(qt) * g.nkt + kt] = static_cast<uint8_t>(c == 0 ? 0 : (c == n_in ? 2 : 1));
    }
    __syncthreads();
  }
}

// Packed fine words of every partial listed tile, stored at its list position
// (CTA per plan row, thread per tile row).
__global__ void __launch_bounds__(128) k_bits_fine(BlockSparseArgs a, const GroupInfo* __restrict__ groups,
                                                   const int32_t* __restrict__ row_group,
                                                   const int32_t* __restrict__ row_ptr,
                                                   const int32_t* __restrict__ kv_tile,
                                                   const int32_t* __restrict__ part, uint32_t* __restrict__ fine) {
  const int row = blockIdx.x;
  const int grp = row_group[row];
  const GroupInfo g = groups[grp];
  const int qt = row - g.row0, r = threadIdx.x;
  const int t = qt * kTile + r;  // plan row
  const bool in = t < g.q_len;
  const int i = t / a.g_pack;    // query position
  const uint32_t* rowbits = a.bits + (static_cast<int64_t>(grp) * a.nqb + (in ? i / a.q_block : 0)) * a.wpr;
  const uint32_t* kvrow = a.kv_valid ? a.kv_valid + static_cast<int64_t>(g.b) * a.kv_wpb : nullptr;
  for (int e = row_ptr[row]; e < row_ptr[row + 1]; ++e) {
    const int slot = part[e];
    if (slot < 0) continue;
    const int kt = kv_tile[e];
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (in) {
      w.x = block_word(a, rowbits, kvrow, i, kt * kTile + 0, g.k_len);
      w.y = block_word(a, rowbits, kvrow, i, kt * kTile + 32, g.k_len);
      w.z = block_word(a, rowbits, kvrow, i, kt * kTile + 64, g.k_len);
      w.w = block_word(a, rowbits, kvrow, i, kt * kTile + 96, g.k_len);
    }
    reinterpret_cast<uint4*>(fine + static_cast<int64_t>(slot) * kFineWordsPerTile)[r] = w;
  }
}

// ----------------------------------------------------------------------------
// position-term predicates -> exact tile classes (CTA per (group, query tile))
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_pred_classify(const int32_t* __restrict__ terms, int n_terms,
                                                       const GroupInfo* __restrict__ groups, uint8_t* __restrict__ cls) {
  __shared__ int warp_cnt[4];
  const GroupInfo g = groups[blockIdx.x];
  const int qt = blockIdx.y;
  if (qt >= g.nqt) return;
  const int r = threadIdx.x, warp = r >> 5, lane = r & 31;
  const int i = qt * kTile + r;
  const bool in = i < g.q_len;
  const int rows_in = min(kTile, g.q_len - qt * kTile);
  for (int kt = 0; kt < g.nkt; ++kt) {
    int cnt = 0;
    if (in) {
      uint32_t am[4];
      pred_words(terms, n_terms, i, kt, g.k_len, am);
      cnt = __popc(am[0]) + __popc(am[1]) + __popc(am[2]) + __popc(am[3]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) warp_cnt[warp] = cnt;
    __syncthreads();
    if (r == 0) {
      const int c = warp_cnt[0] + warp_cnt[1] + warp_cnt[2] + warp_cnt[3];
      const int n_in = rows_in * min(kTile, g.k_len - kt * kTile);
      cls[g.cls_off + static_cast<int64_t>(qt) * g.nkt + kt] = static_cast<uint8_t>(c == 0 ? 0 : (c == n_in ? 2 : 1));
    }
    __syncthreads();
  }
}

// ----------------------------------------------------------------------------
// make_att_block_ids: inclusive running count of block openings (CTA per batch)
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_make_block_ids(const uint8_t* __restrict__ pad,
                                                         const uint8_t* __restrict__ att, int N, int n_cross,
                                                         const uint8_t* __restrict__ cross_pad,
                                                         int32_t* __restrict__ q_blk, int32_t* __restrict__ k_blk,
                                                         uint8_t* __restrict__ q_valid,
                                                         uint8_t* __restrict__ k_valid) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  const int b = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t Nk = static_cast<int64_t>(n_cross) + N;
  for (int j = tid; j < n_cross; j += blockDim.x) {
    k_blk[b * Nk + j] = INT32_MIN;
    k_valid[b * Nk + j] = cross_pad[static_cast<int64_t>(b) * n_cross + j] != 0;
  }
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < N; base += blockDim.x) {
    const int i = base + tid;
    const int v = (i < N && att[static_cast<int64_t>(b) * N + i] != 0) ? 1 : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_sums[lane] = w;
    }
    __syncthreads();
    const int incl = x + (warp ? warp_sums[warp - 1] : 0) + carry;
    if (i < N) {
      const int64_t qi = static_cast<int64_t>(b) * N + i;
      const uint8_t pv = pad[qi] != 0;
      q_blk[qi] = incl;
      q_valid[qi] = pv;
      k_blk[b * Nk + n_cross + i] = incl;
      k_valid[b * Nk + n_cross + i] = pv;
    }
    __syncthreads();
    if (tid == blockDim.x - 1) carry = incl;
    __syncthreads();
  }
}

// ----------------------------------------------------------------------------
// group table of a regular layout (every group the same shape): group g is
// batch g / n_hkv and, for BSR plans, kv head g % n_hkv
// ----------------------------------------------------------------------------
__global__ void k_init_regular_groups(GroupInfo tmpl, int n_groups, int n_hkv, int bsr, int copy_ids,
                                      GroupInfo* __restrict__ groups, int32_t* __restrict__ row_group,
                                      int n_rows, uint32_t* __restrict__ err, int32_t* __restrict__ max_width) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i == 0 && err != nullptr) {  // the plan's status words start cleared
    *err = 0u;
    *max_width = 0;
  }
  if (i < n_groups) {
    GroupInfo g = tmpl;
    g.b = (tmpl.b < 0) ? -1 : i / n_hkv;
    g.hkv = bsr ? i % n_hkv : -1;
    g.row0 = i * tmpl.nqt;
    g.cls_off = static_cast<int64_t>(i) * tmpl.nqt * tmpl.nkt;
    g.qid_off = copy_ids ? i * tmpl.nqt * kTile : 0;
    g.kid_off = copy_ids ? i * tmpl.nkt * kTile : 0;
    g.kbit_off = copy_ids ? i * tmpl.nkt * kWordsPerTileRow : 0;
    groups[i] = g;
  }
  if (i < n_rows) row_group[i] = tmpl.nqt > 0 ? i / tmpl.nqt : 0;
}

// ----------------------------------------------------------------------------
// launchers (host)
// ----------------------------------------------------------------------------
cudaError_t launch_init_regular_groups(const GroupInfo& tmpl, int n_groups, int n_hkv, int bsr, int copy_ids,
                                       GroupInfo* groups, int32_t* row_group, int n_rows, cudaStream_t s,
                                       uint32_t* err, int32_t* max_width) {
  int n = n_groups > n_rows ? n_groups : n_rows;
  if (n <= 0) {
    if (err == nullptr) return cudaSuccess;
    n = 1;  // the status words still need clearing
  }
  k_init_regular_groups<<<(n + 255) / 256, 256, 0, s>>>(tmpl, n_groups, n_hkv, bsr, copy_ids, groups, row_group,
                                                       n_rows, err, max_width);
  return cudaGetLastError();
}

// Checked build: every guard region of a plan slab (offsets in `offs`) must
// still hold the guard byte.
__global__ void k_check_guards(const uint8_t* __restrict__ slab, const uint64_t* __restrict__ offs, int n,
                               uint32_t guard_bytes, int guard_byte, uint32_t* err) {
  for (int g = blockIdx.x; g < n; g += gridDim.x) {
    const uint8_t* p = slab + offs[g];
    for (uint32_t i = threadIdx.x; i < guard_bytes; i += blockDim.x)
      if (p[i] != static_cast<uint8_t>(guard_byte)) atomicOr(err, DEVERR_GUARD);
  }
}

cudaError_t launch_check_guards(const void* slab, const uint64_t* offs, int n, uint32_t guard_bytes, int guard_byte,
                                uint32_t* err, cudaStream_t s) {
  if (n <= 0 || slab == nullptr) return cudaSuccess;
  k_check_guards<<<n < 64 ? n : 64, 64, 0, s>>>(static_cast<const uint8_t*>(slab), offs, n, guard_bytes, guard_byte,
                                                err);
  return cudaGetLastError();
}

cudaError_t launch_dense_classify(const uint8_t* mask, int64_t ld, int Sq, int Sk, uint8_t* cls, uint32_t* fine,
                                  cudaStream_t s, GroupInfo* groups, const GroupInfo* group, int32_t* row_group,
                                  uint32_t* err, int32_t* max_width) {
  const int nqt = (Sq + kTile - 1) / kTile, nkt = (Sk + kTile - 1) / kTile;
  const int vec_ok = ((reinterpret_cast<uintptr_t>(mask) & 15u) == 0 && (ld & 15) == 0) ? 1 : 0;
  DenseInit init;
  init.groups = groups;
  if (groups != nullptr) init.group = *group;
  init.row_group = row_group;
  init.err = err;
  init.max_width = max_width;
  dim3 grid((nkt + kDenseTilesPerCta - 1) / kDenseTilesPerCta, nqt);
  k_dense_classify<<<grid, 256, 0, s>>>(mask, ld, Sq, Sk, nkt, cls, fine, vec_ok, init);
  return cudaGetLastError();
}

cudaError_t launch_blockid_classify(const GroupInfo* groups, int n_groups, int max_tiles_q, int max_tiles_k,
                                    const int32_t* q_blk, const int32_t* k_blk, const uint8_t* q_valid,
                                    const uint8_t* k_valid, int batched, int Sq, int Sk, int window, int copy_ids,
                                    int32_t* qid, uint8_t* qv, int32_t* kid, uint32_t* kbits, uint8_t* cls,
                                    cudaStream_t s) {
  const size_t smem = sizeof(TileStat) * static_cast<size_t>(max_tiles_q + max_tiles_k);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_blockid_classify, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  k_blockid_classify<<<n_groups, 256, smem, s>>>(groups, q_blk, k_blk, q_valid, k_valid, batched, Sq, Sk,
                                                 window, copy_ids, qid, qv, kid, kbits, cls);
  return cudaGetLastError();
}

cudaError_t launch_bsr_classify(const int32_t* indptr, const int32_t* indices, int64_t n_indices,
                                const GroupInfo* groups, int n_groups, int nqt, int causal, uint8_t* cls,
                                uint32_t* err, int32_t* max_width, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(n_groups) * nqt;
  const int threads = 128;
  k_bsr_classify<<<static_cast<unsigned>((n + threads - 1) / threads), threads, 0, s>>>(
      indptr, indices, n_indices, groups, n_groups, nqt, causal, cls, err, max_width);
  return cudaGetLastError();
}

cudaError_t launch_rows(const GroupInfo* groups, const int32_t* row_group, const uint8_t* cls, int n_rows,
                        int max_nkt, int32_t* row_cnt, int32_t* row_ptr, int32_t* kv_tile, int32_t* part,
                        int32_t* order, cudaStream_t s, int32_t* pair_row, int32_t* pair_cost,
                        int32_t* pair_order, int32_t* pair_idx, int part_is_pos, int2* row_work,
                        int2* pair_work, int n_groups, int64_t grid_tiles) {
  // bucket of the counting sorts (keys up to 2 max_nkt), shared with the staged
  // copies of the group table, the row map and the class grid when they fit
  const size_t bucket_bytes = sizeof(int32_t) * static_cast<size_t>(2 * max_nkt + 1);
  const size_t stage_bytes = sizeof(GroupInfo) * static_cast<size_t>(n_groups) +
                             sizeof(int32_t) * static_cast<size_t>(n_rows) + static_cast<size_t>(grid_tiles);
  const int stage = (n_groups > 0 && grid_tiles >= 0 && stage_bytes <= kRowsStageBytes) ? 1 : 0;
  const size_t smem = stage ? (bucket_bytes > stage_bytes ? bucket_bytes : stage_bytes) : bucket_bytes;
  if (smem > 48 * 1024) {
    cudaError_t e =
        cudaFuncSetAttribute(k_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  k_rows<<<1, 1024, smem, s>>>(groups, row_group, cls, n_rows, max_nkt, row_cnt, row_ptr, kv_tile, part, order,
                               pair_row, pair_cost, pair_order, pair_idx, part_is_pos, row_work, pair_work, n_groups,
                               grid_tiles, stage);
  return cudaGetLastError();
}

cudaError_t launch_cols(const GroupInfo* groups, int n_groups, const uint8_t* cls, const int32_t* row_ptr,
                        const int32_t* kv_tile, int part_is_pos, int max_nqt, int n_cols, int32_t* col0,
                        int32_t* col_group, int32_t* col_cnt, int32_t* col_ptr, int32_t* q_tile, int32_t* tpart,
                        int32_t* col_order, cudaStream_t s) {
  const size_t smem = sizeof(int32_t) * static_cast<size_t>(max_nqt + 1);
  if (smem > 48 * 1024) {
    cudaError_t e =
        cudaFuncSetAttribute(k_cols, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  k_cols<<<1, 1024, smem, s>>>(groups, n_groups, cls, row_ptr, kv_tile, part_is_pos, max_nqt, n_cols, col0,
                               col_group, col_cnt, col_ptr, q_tile, tpart, col_order);
  return cudaGetLastError();
}

cudaError_t launch_bsr_to_bits(const int32_t* indptr, const int32_t* indices, int64_t n_indices, int n_groups,
                               int nqb, int nkb, int wpr, uint32_t* bits, uint32_t* err, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(n_groups) * nqb;
  if (n <= 0) return cudaSuccess;
  k_bsr_to_bits<<<static_cast<unsigned>((n + 127) / 128), 128, 0, s>>>(indptr, indices, n_indices, n_groups, nqb, nkb,
                                                                        wpr, bits, err);
  return cudaGetLastError();
}

cudaError_t launch_bits_classify(const uint32_t* bits, const uint32_t* kv_valid, int nqb, int wpr, int kv_wpb,
                                 int q_block, int kv_block, int causal, int g_pack, const GroupInfo* groups,
                                 int n_groups, int nqt, uint8_t* cls, cudaStream_t s) {
  if (n_groups <= 0 || nqt <= 0) return cudaSuccess;
  BlockSparseArgs a{bits, kv_valid, nqb, wpr, kv_wpb, q_block, kv_block, causal, g_pack};
  k_bits_classify<<<dim3(n_groups, nqt), 128, 0, s>>>(a, groups, cls);
  return cudaGetLastError();
}

cudaError_t launch_bits_fine(const uint32_t* bits, const uint32_t* kv_valid, int nqb, int wpr, int kv_wpb,
                             int q_block, int kv_block, int causal, int g_pack, const GroupInfo* groups,
                             const int32_t* row_group, int n_rows, const int32_t* row_ptr, const int32_t* kv_tile,
                             const int32_t* part, uint32_t* fine, cudaStream_t s) {
  if (n_rows <= 0) return cudaSuccess;
  BlockSparseArgs a{bits, kv_valid, nqb, wpr, kv_wpb, q_block, kv_block, causal, g_pack};
  k_bits_fine<<<n_rows, 128, 0, s>>>(a, groups, row_group, row_ptr, kv_tile, part, fine);
  return cudaGetLastError();
}

cudaError_t launch_pred_classify(const int32_t* terms, int n_terms, const GroupInfo* groups, int n_groups, int nqt,
                                 uint8_t* cls, cudaStream_t s) {
  if (n_groups <= 0 || nqt <= 0) return cudaSuccess;
  k_pred_classify<<<dim3(n_groups, nqt), 128, 0, s>>>(terms, n_terms, groups, cls);
  return cudaGetLastError();
}

cudaError_t launch_make_block_ids(const uint8_t* pad, const uint8_t* att, int B, int N, int n_cross,
                                  const uint8_t* cross_pad, int32_t* q_blk, int32_t* k_blk, uint8_t* q_valid,
                                  uint8_t* k_valid, cudaStream_t s) {
  k_make_block_ids<<<B, 1024, 0, s>>>(pad, att, N, n_cross, cross_pad, q_blk, k_blk, q_valid, k_valid);
  return cudaGetLastError();
}

}  // namespace bfa
