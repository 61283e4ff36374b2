// Fused mask-aware attention forward for sm_100a.
//
// Each CTA runs two 128-row query tiles ("slots") that share their keys and
// values: either two heads of one kv head on the same query tile (GQA with an
// even group), or two consecutive query tiles of one head, or (GQA-packed plans,
// kPacked) two consecutive tiles of 128 / G positions x all G heads of a kv head.  The CTA walks the
// union of the two tiles' plan lists (BinFlash: walk each query block's sorted list of
// non-empty key blocks, run all-True blocks with no mask loads, apply the mask on
// partial blocks only, skip all-False blocks).  Work items are taken in the
// plan's longest-first order, so the hardware's in-order CTA dispatch balances
// SMs by the number of non-empty tiles.
//
// Warp roles (384 threads, one CTA per SM):
//   warp 0        TMA producer: Q of both slots, then K_u / V_u of every union
//                 tile u into a two-stage ring
//   warp 1        TMEM owner and single-thread tcgen05.mma issuer, ping-pong:
//                   O0 += P0(u) V(u); S0 = Q0 K(u+1)^T; O1 += P1(u) V(u); S1 = Q1 K(u+1)^T
//                 (S: SS, both operands K-major in shared memory; P V: TS, P is
//                 the A operand in TMEM, V an MN-major shared-memory operand)
//   warps 2..3    idle (they give their registers to the softmax warpgroups)
//   warps 4..7    softmax of slot 0, warps 8..11 softmax of slot 1: one query
//                 row per thread, the whole S row in registers; mask on partial
//                 and edge tiles only, online base-2 softmax in fp32, P written
//                 back to TMEM over S as packed bf16, lazy rescale of O in TMEM;
//                 epilogue O / l -> bf16 and LSE.
// While one slot's softmax runs, the tensor core works on the other slot.
//
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D).
// Shared memory: Q0, Q1 and two K and two V stages (128 x D bf16 each) in
// 64-column panels with the 128-byte swizzle that TMA and the tensor core share.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fwd_params.cuh"
#include "plan_types.cuh"
#include "pred.cuh"
#include "ptx.cuh"
#include "tile_mask.cuh"

namespace bfa {

using namespace ptx;

// 128 * kRegsWG0 + 256 * kRegsSoftmax must equal kThreads * kRegsLaunch: the
// increase draws only on the registers the block was launched with.  The
// compiled kernel's launch count is checked before every first launch.
constexpr int kThreads = 384;
constexpr int kRegsLaunch = 168;
constexpr uint32_t kRegsWG0 = 72;
constexpr uint32_t kRegsSoftmax = 216;
static_assert(128 * kRegsWG0 + 256 * kRegsSoftmax == kThreads * kRegsLaunch, "register split");
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled only when the max grows by > 2^8
constexpr int kStages = 2;

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kSmemBytes = (2 + 2 * kStages) * kTileBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128;
  static constexpr uint32_t kColO0 = 256, kColO1 = 256 + D;
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 1);
};

struct Work {
  int32_t row[2];       // plan row of each slot (-1: slot unused)
  int32_t e0[2], n[2];  // first listed tile and count of each slot's row
  int32_t qt[2];        // query tile inside the group
  int32_t h[2];         // query head of each slot
  int32_t b, hk;
  int32_t seq;          // row of the page table (paged keys / values)
  int32_t same_row;     // both slots run the same row (so the same list)
  int32_t q_off, q_len, k_off, k_len;
  int32_t qid_off, kid_off, kbit_off;
};

// replica index -> (batch, head) of a plan row
__device__ __forceinline__ void replica_bh(const FwdParams& p, const GroupInfo& g, int j, int& b, int& h) {
  if (p.plan.kind == 1 /*BFA_PLAN_DENSE*/) {
    b = j / p.H;
    h = j % p.H;
  } else if (p.plan.kind == 4 /*BFA_PLAN_BSR*/) {
    b = g.b;
    h = g.hkv * (p.H / p.Hkv) + j;
  } else {
    b = p.varlen ? 0 : g.b;
    h = j;
  }
}

__device__ __forceinline__ void decode_work(const FwdParams& p, int w, Work& wk) {
  const int64_t units = p.pair_heads ? p.plan.n_rows : p.plan.n_pairs;
  const int64_t items = p.pair_heads ? p.rep / 2 : p.rep;  // replica units per row / pair
  const int64_t chunk = p.head_chunk;
  const int64_t hg = w / (units * chunk);
  const int64_t rem = w - hg * units * chunk;
  const int64_t gs = min(chunk, items - hg * chunk);
  const int i = static_cast<int>(rem / gs);
  const int j = static_cast<int>(hg * chunk + rem % gs);
  // the plan lists the work items in longest-first order with their group
  int r0, r1, grp;
  uint32_t* const err = p.plan.err;
  (void)err;
  if (p.pair_heads) {
    const int2 rw = p.plan.row_work[BFA_IDX(i, p.plan.n_rows, err)];
    r0 = r1 = rw.x;
    grp = rw.y;
  } else {
    const int2 pw = p.plan.pair_work[BFA_IDX(i, p.plan.n_pairs, err)];
    r0 = pw.x >= 0 ? pw.x : ~pw.x;
    r1 = pw.x >= 0 ? r0 + 1 : -1;
    grp = pw.y;
  }
  const GroupInfo g = p.plan.groups[BFA_IDX(grp, p.plan.n_groups, err)];
  wk.same_row = p.pair_heads;
  wk.row[0] = r0;
  wk.row[1] = r1;
  for (int s = 0; s < 2; ++s) {
    const int r = wk.row[s];
    BFA_CHECK(r < 0 || (r >= g.row0 && r < g.row0 + g.nqt), err);
    wk.e0[s] = r >= 0 ? p.plan.row_ptr[BFA_IDX(r, p.plan.n_rows, err)] : 0;
    wk.n[s] = r >= 0 ? p.plan.row_ptr[BFA_IDX(r + 1, p.plan.n_rows + 1, err)] - wk.e0[s] : 0;
#ifdef BFA_CHECKED
    // a list outside the plan's arrays is reported and not walked
    if (!(wk.n[s] >= 0 && wk.n[s] <= g.nkt && wk.e0[s] >= 0 && wk.e0[s] + wk.n[s] <= p.plan.cap_tiles)) {
      atomicOr(err, DEVERR_BOUNDS);
      wk.e0[s] = 0;
      wk.n[s] = 0;
    }
#endif
    wk.qt[s] = r >= 0 ? r - g.row0 : 0;
  }
  int b, h0, h1;
  if (p.pair_heads) {
    replica_bh(p, g, 2 * j, b, h0);
    replica_bh(p, g, 2 * j + 1, b, h1);
  } else {
    replica_bh(p, g, j, b, h0);
    h1 = h0;
  }
  wk.b = b;
  wk.seq = p.varlen ? grp : b;
  wk.h[0] = h0;
  wk.h[1] = h1;
  wk.hk = h0 / (p.H / p.Hkv);
  wk.q_off = g.q_off;
  wk.q_len = g.q_len;
  wk.k_off = g.k_off;
  wk.k_len = g.k_len;
  wk.qid_off = g.qid_off;
  wk.kid_off = g.kid_off;
  wk.kbit_off = g.kbit_off;
}

// Walk the union of the two slots' ascending key-tile lists.  The entry after
// each list's head is loaded one step early, so a step only moves registers and
// issues the load for a later step: no global-memory latency on the caller.
struct UnionWalk {
  static constexpr int kEnd = 0x7fffffff;
  const int32_t* kv;
  int ea, na, eb, nb, ia, ib;
  int ka, kb, ka2, kb2;  // heads of both lists and the entries after them
  bool same;
  __device__ __forceinline__ void init(const FwdParams& p, const Work& wk) {
    kv = p.plan.kv_tile;  // the list bounds were checked when the work item was decoded
    ea = wk.e0[0];
    na = wk.n[0];
    eb = wk.e0[1];
    nb = wk.n[1];
    ia = ib = 0;
    same = wk.same_row != 0;
    ka = na > 0 ? kv[ea] : kEnd;
    ka2 = na > 1 ? kv[ea + 1] : kEnd;
    kb = (!same && nb > 0) ? kv[eb] : kEnd;
    kb2 = (!same && nb > 1) ? kv[eb + 1] : kEnd;
  }
  // next tile: kt, and whether slot 0 / slot 1 have it; false at the end
  __device__ __forceinline__ bool next(int& kt, bool& a, bool& b) {
    kt = min(ka, kb);
    if (kt == kEnd) return false;
    a = same || ka == kt;
    b = same || kb == kt;
    if (ka == kt) {
      ++ia;
      ka = ka2;
      ka2 = ia + 1 < na ? kv[ea + ia + 1] : kEnd;
    }
    if (!same && kb == kt) {
      ++ib;
      kb = kb2;
      kb2 = ib + 1 < nb ? kv[eb + ib + 1] : kEnd;
    }
    return true;
  }
};

// TMA of one 128-token K or V tile (all D/64 panels) into `dst`, completing on
// `bar`.  Contiguous layouts take one box per panel at token row `ks`; paged
// layouts look the pages up in the page table: pages of >= 128 tokens give one
// box, smaller pages one box per page, each landing at its row offset of the
// swizzled tile (a multiple of 8 rows, so the 128-byte swizzle pattern lines up).
// Pages past the sequence's end re-read its last valid page: finite values that
// the edge mask never lets into the result.
template <int kPanels>
__device__ __forceinline__ void load_kv_tile(const FwdParams& p, const Work& wk, const CUtensorMap* map, uint8_t* dst,
                                             uint32_t bar, int kt, int ks) {
  if (p.page_size == 0) {
#pragma unroll
    for (int pn = 0; pn < kPanels; ++pn) tma_load_4d(smem_u32(dst + pn * 16384), map, bar, pn * 64, wk.hk, ks, wk.b);
    return;
  }
  const int32_t* bt = p.block_table + static_cast<int64_t>(wk.seq) * p.pages_per_seq;
  const int t0 = kt * kTile;
  if (p.page_size >= kTile) {
    const int row = bt[t0 / p.page_size] * p.page_size + t0 % p.page_size;
#pragma unroll
    for (int pn = 0; pn < kPanels; ++pn) tma_load_4d(smem_u32(dst + pn * 16384), map, bar, pn * 64, wk.hk, row, 0);
    return;
  }
  const int last = max(wk.k_len - 1, 0) / p.page_size;
  for (int sub = 0; sub < kTile / p.page_size; ++sub) {
    const int t = t0 + sub * p.page_size;
    const int page = bt[min(t / p.page_size, last)];
    const int row = page * p.page_size;
#pragma unroll
    for (int pn = 0; pn < kPanels; ++pn)
      tma_load_4d(smem_u32(dst + pn * 16384 + sub * p.page_size * 128), map, bar, pn * 64, wk.hk, row, 0);
  }
}

// approximate mode: whether the softmax warps of a slot dropped its tile t
// (their votes were written before they arrived on the P barrier)
template <bool kSkip>
__device__ __forceinline__ bool tile_skipped(const int (&votes)[2][4], int t) {
  if (!kSkip || t == 0) return false;
  const volatile int* v = votes[t & 1];
  return (v[0] & v[1] & v[2] & v[3]) != 0;
}

// The base descriptors pass through an empty asm so that the compiler builds
// them at the point of use (one add per step) instead of hoisting every step's
// descriptor out of the tile loop, where they would stay live in the MMA
// thread's registers.  A step's descriptor is the base plus its byte offset / 16
// (the start-address field; shared-memory offsets stay inside the field).
__device__ __forceinline__ uint64_t opaque_u64(uint64_t x) {
  asm volatile("" : "+l"(x));
  return x;
}

template <int D>
__device__ __forceinline__ void issue_s(uint32_t tS, uint8_t* sQ, uint8_t* sK) {
  const uint64_t dq = opaque_u64(smem_desc(smem_u32(sQ), 16, 1024));
  const uint64_t dk = opaque_u64(smem_desc(smem_u32(sK), 16, 1024));
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off16 = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
    umma_ss(tS, dq + off16, dk + off16, Cfg<D>::kIdescQK, kk > 0);
  }
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t tO, uint32_t tP, uint8_t* sV, bool acc) {
  const uint64_t dv = opaque_u64(smem_desc(smem_u32(sV), 16384, 1024));
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    umma_ts(tO, tP + kk * 8, dv + kk * (2048 >> 4), Cfg<D>::kIdescPV, (acc || kk > 0) ? 1u : 0u);
}

// kSkip: approximate mode (content-based block skipping); the exact kernel is
// compiled without any of its code.  kPacked: GQA-packed query tiles (5-D Q / O
// boxes, rows mapped to (position, head)); the other kernels hold none of it.
template <int D, bool kSkip, bool kPacked>
__global__ void __launch_bounds__(kThreads, 1)
    bfa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const FwdParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* const sQ0 = smem;
  uint8_t* const sQ1 = smem + C::kTileBytes;
  uint8_t* const sK0 = smem + 2 * C::kTileBytes;
  uint8_t* const sV0 = smem + (2 + kStages) * C::kTileBytes;

  // BQ: Q0, Q1 and the first K.  BF[2]: V(j) and K(j + 1).  BE[2]: stages free.
  // BS[2] / BP[2]: S ready / P ready per slot.  BO: all products done.
  enum { BQ = 0, BF = 1, BE = 3, BS = 5, BP = 7, BO = 9, BDONE = 10, NBAR = 11 };
  __shared__ __align__(8) uint64_t bars[NBAR];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ Work wk_s;
  __shared__ int skip_votes[2][2][4];  // approximate mode: [slot][tile parity][warp] "tile negligible"

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  auto sK = [&](int st) { return sK0 + st * C::kTileBytes; };
  auto sV = [&](int st) { return sV0 + st * C::kTileBytes; };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), (i == BP || i == BP + 1) ? 4 : 1);
    fence_barrier_init();
    decode_work(p, blockIdx.x, wk_s);
    // Thread 0 is the TMA producer: the Q tiles go out as soon as the work item is
    // known, before the block-wide barrier and the key list's first entry (K(0)
    // follows on the same barrier, whose byte count covers it).
    if (wk_s.n[0] + wk_s.n[1] > 0) {
      prefetch_tmap(&tmQ);
      mbar_expect_tx(bar(BQ), ((wk_s.n[0] > 0 ? 1 : 0) + (wk_s.n[1] > 0 ? 1 : 0) + 1) * C::kTileBytes);
      for (int s = 0; s < 2; ++s) {
        if (wk_s.n[s] == 0) continue;
        const int qs = wk_s.q_off + wk_s.qt[s] * kTile;
        uint8_t* dq = s ? sQ1 : sQ0;
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn) {
          if constexpr (kPacked)  // 128 >> pack_shift positions of every head of the kv head
            tma_load_5d(smem_u32(dq + pn * 16384), &tmQ, bar(BQ), pn * 64, 0, wk_s.hk, qs >> p.pack_shift, wk_s.b);
          else
            tma_load_4d(smem_u32(dq + pn * 16384), &tmQ, bar(BQ), pn * 64, wk_s.h[s], qs, wk_s.b);
        }
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const Work& wk = wk_s;  // read from shared memory where used: keeps warpgroup 0 within its registers
  const uint64_t cap = p.wait_ns;
  const bool any_tiles = wk.n[0] + wk.n[1] > 0;

  if (warp < 4) {
    // ============================================================ warpgroup 0
    regs_dec<kRegsWG0>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      // Q of both slots (issued during the set-up) and K of the first union tile on
      // BQ; then at step j, V of union tile j and K of tile j + 1 together on
      // F[j & 1], once the MMAs of commit j - 1 (which read the previous occupants
      // of both stages) are done.
      if (lane == 0 && any_tiles) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        UnionWalk walk;
        walk.init(p, wk);
        int kt, kt_n;
        bool ha, hb;
        walk.next(kt, ha, hb);  // any_tiles: the union has a first tile
        BFA_CHECK(kt >= 0 && kt * kTile < wk.k_len, p.plan.err);
        load_kv_tile<C::kPanels>(p, wk, &tmK, sK(0), bar(BQ), kt, wk.k_off + kt * kTile);
        int last_f[2] = {-1, -1};  // last step that filled F[0] / F[1]
        for (int j = 0;; ++j) {
          const bool have_next = walk.next(kt_n, ha, hb);
          BFA_CHECK(!have_next || (kt_n >= 0 && kt_n * kTile < wk.k_len), p.plan.err);
          if (j >= 1 && !mbar_wait_fast(bar(BE + ((j - 1) & 1)), ((j - 1) >> 1) & 1, cap, &abort_flag)) break;
          const uint32_t f = bar(BF + (j & 1));
          mbar_expect_tx(f, (have_next ? 2 : 1) * C::kTileBytes);
          load_kv_tile<C::kPanels>(p, wk, &tmV, sV(j & 1), f, kt, wk.k_off + kt * kTile);
          if (have_next) load_kv_tile<C::kPanels>(p, wk, &tmK, sK((j + 1) & 1), f, kt_n, wk.k_off + kt_n * kTile);
          last_f[j & 1] = j;
          if (!have_next) break;
          kt = kt_n;
        }
        // every copy this CTA issued must land before it can exit (on the normal
        // path these phases completed long ago; the drain bound is fixed)
        mbar_drain(bar(BQ), 0, &abort_flag);
        for (int b = 0; b < 2; ++b)
          if (last_f[b] >= 0) mbar_drain(bar(BF + b), (last_f[b] >> 1) & 1, &abort_flag);
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      // Commit c = 0 follows the first S products, commit c = u + 1 the products of
      // iteration u; E[c & 1] tells the producer that K(c) and V(c - 1) are free.
      if (lane == 0 && any_tiles) {
        const uint32_t tS0 = tmem + C::kColS0, tS1 = tmem + C::kColS1;
        const uint32_t tO0 = tmem + C::kColO0, tO1 = tmem + C::kColO1;
        UnionWalk walk;
        walk.init(p, wk);
        bool ok = mbar_wait_fast(bar(BQ), 0, cap, &abort_flag);
        int cnt0 = 0, cnt1 = 0;  // P phases consumed per slot
        bool started0 = false, started1 = false;
        int kt;
        bool a, b, na_, nb_;
        bool have = ok && walk.next(kt, a, b);
        if (have) {
          tc_fence_after();
          if (a) { issue_s<D>(tS0, sQ0, sK(0)); umma_commit(bar(BS + 0)); }
          if (b) { issue_s<D>(tS1, sQ1, sK(0)); umma_commit(bar(BS + 1)); }
          umma_commit(bar(BE + 0));
        }
        for (int u = 0; ok && have; ++u) {
          const int st = u & 1, st1 = (u + 1) & 1;
          const bool have_next = walk.next(kt, na_, nb_);
          // V(u) and K(u + 1)
          if (!mbar_wait_fast(bar(BF + st), (u >> 1) & 1, cap, &abort_flag)) { ok = false; break; }
          // slot 0: O0 += P0(u) V(u), then S0 = Q0 K(u+1)^T over the consumed P0
          if (a) {
            if (!mbar_wait_fast(bar(BP + 0), cnt0 & 1, cap, &abort_flag)) { ok = false; break; }
            const bool skip0 = tile_skipped<kSkip>(skip_votes[0], cnt0);
            ++cnt0;
            if (!skip0) {
              tc_fence_after();
              issue_pv<D>(tO0, tS0, sV(st), started0);
              started0 = true;
            }
          }
          if (have_next && na_) {
            tc_fence_after();
            issue_s<D>(tS0, sQ0, sK(st1));
            umma_commit(bar(BS + 0));
          }
          // slot 1: O1 += P1(u) V(u), then S1 = Q1 K(u+1)^T
          if (b) {
            if (!mbar_wait_fast(bar(BP + 1), cnt1 & 1, cap, &abort_flag)) { ok = false; break; }
            const bool skip1 = tile_skipped<kSkip>(skip_votes[1], cnt1);
            ++cnt1;
            if (!skip1) {
              tc_fence_after();
              issue_pv<D>(tO1, tS1, sV(st), started1);
              started1 = true;
            }
          }
          if (have_next && nb_) {
            tc_fence_after();
            issue_s<D>(tS1, sQ1, sK(st1));
            umma_commit(bar(BS + 1));
          }
          umma_commit(bar(BE + st1));
          a = na_;
          b = nb_;
          have = have_next;
        }
        if (ok) umma_commit(bar(BO));
        // every MMA issued must be finished before TMEM is released (bounded)
        umma_commit(bar(BDONE));
        mbar_drain(bar(BDONE), 0, &abort_flag);
      }
    }
  } else {
    // ============================================================ softmax warpgroups
    regs_inc<kRegsSoftmax>();
    const int slot = (warp >> 2) - 1;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int my_row = slot ? wk.row[1] : wk.row[0];
    if (my_row >= 0) {
      const uint32_t tS = tmem_addr(tmem + (slot ? C::kColS1 : C::kColS0), quarter * 32, 0);
      const uint32_t tO = tmem_addr(tmem + (slot ? C::kColO1 : C::kColO0), quarter * 32, 0);
      const uint32_t barS = bar(BS + slot), barP = bar(BP + slot);
      const int n = slot ? wk.n[1] : wk.n[0];
      const int e0 = slot ? wk.e0[1] : wk.e0[0];
      const int qpos = (slot ? wk.qt[1] : wk.qt[0]) * kTile + row;  // position of this row inside its group
      const float c = p.scale_log2;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      int kt_next = n > 0 ? p.plan.kv_tile[e0] : 0;
      int part_next = n > 0 ? p.plan.part[e0] : -1;
      for (int t = 0; t < n; ++t) {
        const int kt = kt_next, part = part_next;
        if (t + 1 < n) {  // next list entry, off the critical path
          kt_next = p.plan.kv_tile[e0 + t + 1];
          part_next = p.plan.part[e0 + t + 1];
        }
        const bool masked = part >= 0 || (kt + 1) * kTile > wk.k_len;
        uint32_t am[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
        if (masked) row_mask_words(p.plan, wk, qpos, row, kt, part, am);

        const bool got = mbar_wait(barS, t & 1, cap, &abort_flag);
        if constexpr (kSkip) {
          // the vote below is a barrier of the slot's four warps, so they leave
          // the loop together (slot-uniform exit)
          if (named_bar_red_or(1 + slot, 128, !got)) { ok = false; break; }
        } else {
          if (__any_sync(0xffffffffu, !got)) { ok = false; break; }  // warp-uniform exit
        }
        tc_fence_after();
        // the whole S row in registers: four loads in flight, one wait
        uint32_t sr[128];
        tmem_ld_32x32b_x32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld_32x32b_x32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld_32x32b_x32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld_32x32b_x32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tmem_wait_ld();
        reg_fence(sr);
        float* s = reinterpret_cast<float*>(sr);
        if (masked) {
#pragma unroll
          for (int j = 0; j < 128; ++j)
            if (!((am[j >> 5] >> (j & 31)) & 1u)) s[j] = -INFINITY;
        }
        // row max, 8 independent chains of three-input max
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
        for (int j = 8; j < 128; j += 2) mx8[(j >> 1) & 7] = fmax3(mx8[(j >> 1) & 7], s[j], s[j + 1]);
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        // Approximate mode (content-based block skipping): the tile is dropped when
        // every row of the slot has its tile max more than the threshold below its
        // running reference max (rows past the sequence count as negligible).  The
        // four warps of the slot vote through shared memory; the MMA thread reads
        // the same votes after the P barrier and then issues no P V for the tile.
        bool skip = false;
        if constexpr (kSkip) {
          if (t > 0) {
            const bool neg = qpos >= wk.q_len || mx * c < m - p.skip_log2;
            const bool wall = __all_sync(0xffffffffu, neg);
            if (lane == 0) skip_votes[slot][t & 1][quarter] = wall ? 1 : 0;
            named_bar_sync(1 + slot, 128);
            const volatile int* v = skip_votes[slot][t & 1];
            skip = (v[0] & v[1] & v[2] & v[3]) != 0;
          }
        }
        const float mnew = skip ? m : fmaxf(m, mx * c);
        // The reference max m only moves when some row of the warp grew by more
        // than 2^8; then every row of the warp moves to its true running max
        // (alpha is 1 for rows that did not grow).  The decision is warp-uniform
        // because the O rescale uses whole-warp TMEM loads and stores.
        if (__any_sync(0xffffffffu, mnew > m + kRescaleThreshold)) {
          const float alpha = (mnew == m) ? 1.f : ex2_approx(m - mnew);  // 0 when m = -inf
          l *= alpha;
          if (t > 0) {
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[32];
              tmem_ld_32x32b_x32(tO + cc * 32, o);
              tmem_wait_ld();
              reg_fence(o);
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
              tmem_st_32x32b_x32(tO + cc * 32, o);
            }
          }
          m = mnew;
        }
        if (!skip) {
          const float mref = (m == -INFINITY) ? 0.f : m;
          // p = 2^(s*c - m), 4 independent row-sum chains; packed bf16 pairs go to
          // the first 64 columns of S (the A operand of the P V product)
          // (pairs of columns go through the packed fp32x2 fma and add: half the
          // FMA-pipe instructions of the scalar form)
          uint64_t rs2[4] = {0, 0, 0, 0};
          const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-mref, -mref);
          uint32_t pk[64];
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const uint64_t x2 = f2_fma(f2_pack(s[2 * j], s[2 * j + 1]), c2, nm2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            rs2[j & 3] = f2_add(rs2[j & 3], f2_pack(p0, p1));
            pk[j] = pack_bf16x2(p0, p1);
          }
          float r[8];
          f2_unpack(f2_add(rs2[0], rs2[1]), r[0], r[1]);
          f2_unpack(f2_add(rs2[2], rs2[3]), r[2], r[3]);
          l += (r[0] + r[2]) + (r[1] + r[3]);
          tmem_st_32x32b_x32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
          tmem_st_32x32b_x32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(barP);
      }
      // ---------------------------------------------------------- epilogue
      if (ok && n > 0) {
        const bool got = mbar_wait(bar(BO), 0, cap, &abort_flag);
        ok = !__any_sync(0xffffffffu, !got);
      }
      tc_fence_after();
      const bool store = qpos < wk.q_len;  // TMEM loads below stay whole-warp; only stores are per row
      const int h = slot ? wk.h[1] : wk.h[0];
      // the row's query head and position (GQA-packed tiles: rows position-major over the kv head's heads)
      const int hrow = kPacked ? (wk.hk << p.pack_shift) + (qpos & (p.pack_g - 1)) : h;
      const int prow = kPacked ? qpos >> p.pack_shift : qpos;
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      const int qt0 = (slot ? wk.qt[1] : wk.qt[0]) * kTile;  // first row of the tile in its group
      if (qt0 + kTile <= wk.q_len) {
        // A tile wholly inside its sequence leaves as one TMA store: each row goes,
        // as bf16, into this slot's Q buffer (free: every product is done) in the
        // 128-byte swizzled layout of the box, then one thread stores the tile.
        // All four warps of the slot reach the barrier whatever happened before,
        // and the store is skipped if any wait of the block gave up.
        const uint32_t stg = smem_u32(slot ? sQ1 : sQ0);
        if (ok) {
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            if (n > 0) {
              tmem_ld_32x32b_x32(tO + cc * 32, o);
              tmem_wait_ld();
              reg_fence(o);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = 0u;
            }
            uint32_t pkd[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pkd[j] = pack_bf16x2(__uint_as_float(o[2 * j]) * inv, __uint_as_float(o[2 * j + 1]) * inv);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int c16 = cc * 4 + j;  // 16-byte chunk of the row
              const uint32_t addr = stg + (c16 >> 3) * 16384 + row * 128 + (((c16 & 7) ^ (row & 7)) << 4);
              st_shared_v4(addr, pkd[4 * j], pkd[4 * j + 1], pkd[4 * j + 2], pkd[4 * j + 3]);
            }
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1 + slot, 128);
        if (quarter == 0 && lane == 0 && ok && !*static_cast<volatile int*>(&abort_flag)) {
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn)
            if constexpr (kPacked)
              tma_store_5d(&tmO, stg + pn * 16384, pn * 64, 0, wk.hk, (wk.q_off + qt0) >> p.pack_shift, wk.b);
            else
              tma_store_4d(&tmO, stg + pn * 16384, pn * 64, h, wk.q_off + qt0, wk.b);
          bulk_commit_group();
          bulk_wait_group_read0();
        }
      } else if (ok) {
        const int64_t tok = static_cast<int64_t>(wk.q_off) + prow;
        __nv_bfloat16* op =
            p.out + static_cast<int64_t>(wk.b) * p.o_sb + tok * p.o_ss + static_cast<int64_t>(hrow) * p.o_sh;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          if (n > 0) {
            tmem_ld_32x32b_x32(tO + cc * 32, o);
            tmem_wait_ld();
            reg_fence(o);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
          uint32_t pkd[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            pkd[j] = pack_bf16x2(__uint_as_float(o[2 * j]) * inv, __uint_as_float(o[2 * j + 1]) * inv);
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(op + cc * 32);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pkd[4 * j], pkd[4 * j + 1], pkd[4 * j + 2], pkd[4 * j + 3]);
          }
        }
      }
      if (ok) {
        const int64_t tok = static_cast<int64_t>(wk.q_off) + prow;
        if (p.lse && store) {
          const float lse = (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
          const int64_t li = p.varlen ? static_cast<int64_t>(hrow) * p.Sq_lse + tok
                                      : (static_cast<int64_t>(wk.b) * p.H + hrow) * p.Sq_lse + prow;
          p.lse[li] = lse;
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (abort_flag && threadIdx.x == 0) atomicOr(p.plan.err, DEVERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ----------------------------------------------------------------------------
// bounded-wait self test: a barrier phase nothing completes
// ----------------------------------------------------------------------------
__global__ void k_wait_selftest(uint32_t* err, uint64_t cap) {
  __shared__ __align__(8) uint64_t b;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&b), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(smem_u32(&b), 0, cap, &abort_flag)) atomicOr(err, DEVERR_TIMEOUT);
}

// ----------------------------------------------------------------------------
// launchers (host)
// ----------------------------------------------------------------------------
int fwd_smem_bytes(int D) { return D == 64 ? Cfg<64>::kSmemBytes : Cfg<128>::kSmemBytes; }

// The setmaxnreg split is only safe if every thread is launched with exactly
// kRegsLaunch registers; refuse to launch otherwise.
template <typename K>
static cudaError_t prepare(K kernel, int smem) {
  cudaFuncAttributes a;
  cudaError_t e = cudaFuncGetAttributes(&a, kernel);
  if (e != cudaSuccess) return e;
  if (a.numRegs != kRegsLaunch) return cudaErrorInvalidKernelImage;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

template <int D, bool kSkip, bool kPacked>
static cudaError_t launch_one(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const CUtensorMap& to, const FwdParams& p, int64_t n_work, cudaStream_t s) {
  static cudaError_t ready = prepare(bfa_fwd_kernel<D, kSkip, kPacked>, Cfg<D>::kSmemBytes);
  if (ready != cudaSuccess) return ready;
  bfa_fwd_kernel<D, kSkip, kPacked><<<static_cast<unsigned>(n_work), kThreads, Cfg<D>::kSmemBytes, s>>>(tq, tk, tv,
                                                                                                       to, p);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& to, const FwdParams& p, int64_t n_work, cudaStream_t s) {
  const bool approx = p.skip_log2 > 0.f, packed = p.pack_g > 1;
  if (packed)
    return approx ? launch_one<D, true, true>(tq, tk, tv, to, p, n_work, s)
                  : launch_one<D, false, true>(tq, tk, tv, to, p, n_work, s);
  return approx ? launch_one<D, true, false>(tq, tk, tv, to, p, n_work, s)
                : launch_one<D, false, false>(tq, tk, tv, to, p, n_work, s);
}

cudaError_t launch_fwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdParams& p, int64_t n_work, cudaStream_t s) {
  if (n_work <= 0) return cudaSuccess;
  if (n_work > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  return D == 64 ? launch_d<64>(tq, tk, tv, to, p, n_work, s) : launch_d<128>(tq, tk, tv, to, p, n_work, s);
}

cudaError_t launch_wait_selftest(uint32_t* err, uint64_t cap, cudaStream_t s) {
  k_wait_selftest<<<1, 32, 0, s>>>(err, cap);
  return cudaGetLastError();
}

cudaError_t probe_fwd_kernels() {
  cudaFuncAttributes a;
  cudaError_t e = cudaFuncGetAttributes(&a, bfa_fwd_kernel<128, false, false>);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, bfa_fwd_kernel<64, false, false>);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, bfa_fwd_kernel<128, true, false>);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, bfa_fwd_kernel<64, true, false>);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, bfa_fwd_kernel<128, false, true>);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, bfa_fwd_kernel<64, false, true>);
  return e;
}

}  // namespace bfa
