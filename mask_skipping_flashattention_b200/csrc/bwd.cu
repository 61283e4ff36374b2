// Backward of the mask-aware attention for sm_100a: gradients of
//   O = softmax(scale Q K^T + mask) V
// with respect to Q, K and V for an upstream gradient dO, reusing the forward's
// plan and LSE (BinFlash, "How it works": the backward is two passes, one over
// key blocks for dK and dV and one over query blocks for dQ, both dispatched from
// the same gathered block lists; tensorplay varlen: the log-sum-exp is returned
// by the forward so that the backward can use it again).
//
// With P = exp(scale S - LSE) (S = Q K^T, masked pairs 0), dP = dO V^T and
// D_i = dO_i . O_i, the score gradient is dS = P * (dP - D), and
//   dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
//
// Kernels:
//   k_bwd_prep  per query row: D = dO . O and LSE * log2(e) into a workspace
//               padded to whole tiles (HBM-bound, one pass over O and dO); for
//               the fused pass it also zeroes the fp32 dQ sums;
//   k_bwd_fused (D = 128, the default) one pass over the key-tile columns: the
//               k_bwd_dkdv pass below plus dQ^T = K^T dS^T from the same dS,
//               summed across key tiles by fp32 reductions; k_bwd_dq_store then
//               scales the sums into dq (S and dP are made once per tile pair);
// and the two passes (D = 64, or bitwise-reproducible results on request):
//   k_bwd_dq    one CTA per (plan row, replica), walking the row's key-tile list:
//               S = Q K^T and dP = dO V^T (SS), dS into TMEM as bf16, dQ += dS K
//               (TS); the next tile's S and dP run while this tile's dS is made
//               (dS double-buffered in TMEM); the mask on partial and edge tiles
//               only;
//   k_bwd_dkdv  one CTA per (key-tile column, kv replica), walking the column's
//               query-tile list for every query head of the kv head (GQA sums in
//               TMEM, no atomics): S^T = K Q^T and dP^T = V dO^T (SS), P^T and dS^T
//               into TMEM as bf16 over them, dV += P^T dO and dK += dS^T Q (TS);
//               the products run in the order dV(s), S^T(s+1), dK(s), dP^T(s+1),
//               so the next step's P^T is made while dK(s) and dP^T(s+1) run.
// Warp roles of the two tile kernels: warp 0 TMA producer, warp 1 TMEM owner and
// single-thread tcgen05.mma issuer; k_bwd_dq (384 threads): warps 4..11, one
// query row per thread and half of the tile's keys per warp; k_bwd_dkdv (256
// threads): warps 4..7, one key row per thread.  Every wait is bounded.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bwd_params.cuh"
#include "plan_types.cuh"
#include "ptx.cuh"
#include "tile_mask.cuh"

namespace bfa {

using namespace ptx;

namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdStages = 2;
constexpr int kDqKStages = 3;  // K(u) stays until dQ(u) is done, a tile after V(u) is free

template <int D>
struct BCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kVecBytes = 2 * kTile * 4;  // LSE * log2(e) and D of one query tile
  // two resident tiles, then kBwdStages stages of two tiles (+ the vectors in k_bwd_dkdv)
  static constexpr int kSmemBytes = (2 + 2 * kBwdStages) * kTileBytes + kBwdStages * kVecBytes + 1024;
  // k_bwd_dq: Q, dO, kDqKStages K stages and kBwdStages V stages
  static constexpr int kDqSmemBytes = (2 + kDqKStages + kBwdStages) * kTileBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdescNN = idesc_bf16_f32(128, 128, 0);  // both operands K-major, N = 128
  static constexpr uint32_t kIdescD = idesc_bf16_f32(128, D, 1);     // B MN-major, N = D
};

// Context of one group's tile for the mask functions of tile_mask.cuh.
struct GroupCtx {
  int32_t q_len, k_len, qid_off, kid_off, kbit_off;
};

__device__ __forceinline__ GroupCtx group_ctx(const GroupInfo& g) {
  GroupCtx c;
  c.q_len = g.q_len;
  c.k_len = g.k_len;
  c.qid_off = g.qid_off;
  c.kid_off = g.kid_off;
  c.kbit_off = g.kbit_off;
  return c;
}

// replica index -> (batch, head) of a plan row (as in the forward)
__device__ __forceinline__ void replica_bh(const BwdParams& p, const GroupInfo& g, int j, int& b, int& h) {
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

// (batch, head) -> replica index of the workspace
__device__ __forceinline__ int replica_of(const BwdParams& p, const GroupInfo& g, int b, int h) {
  if (p.plan.kind == 1) return b * p.H + h;
  if (p.plan.kind == 4) return h - g.hkv * (p.H / p.Hkv);
  return h;
}

// plan row `qpos` of a query tile -> its query position and head, for the row's
// base head h (GQA-packed plans: rows position-major over the kv head's heads)
__device__ __forceinline__ void row_pos_head(const BwdParams& p, int qpos, int h, int& prow, int& hrow) {
  if (p.pack_g > 1) {
    prow = qpos >> p.pack_shift;
    hrow = h + (qpos & (p.pack_g - 1));
  } else {
    prow = qpos;
    hrow = h;
  }
}

// one 128-row tile of Q or dO: a 4-D box of one head, or a 5-D box of every head
// of the kv head (GQA-packed plans)
template <int kPanels>
__device__ __forceinline__ void load_q_tile(const BwdParams& p, const CUtensorMap* map, uint8_t* dst, uint32_t bar,
                                            int h, int hk, int qs, int b) {
#pragma unroll
  for (int pn = 0; pn < kPanels; ++pn) {
    if (p.pack_g > 1)
      tma_load_5d(smem_u32(dst + pn * 16384), map, bar, pn * 64, 0, hk, qs >> p.pack_shift, b);
    else
      tma_load_4d(smem_u32(dst + pn * 16384), map, bar, pn * 64, h, qs, b);
  }
}

// kv replica index -> (batch, kv head) of a key-tile column
__device__ __forceinline__ void kv_replica_bh(const BwdParams& p, const GroupInfo& g, int j, int& b, int& hk) {
  if (p.plan.kind == 1) {
    b = j / p.Hkv;
    hk = j % p.Hkv;
  } else if (p.plan.kind == 4) {
    b = g.b;
    hk = g.hkv;
  } else {
    b = p.varlen ? 0 : g.b;
    hk = j;
  }
}

// work item -> (unit in longest-first order, replica), chunked so a chunk's
// replicas of consecutive units run together (keys / values or queries in L2)
__device__ __forceinline__ void chunked_decode(int64_t w, int64_t units, int64_t items, int64_t chunk, int& i, int& j) {
  const int64_t hg = w / (units * chunk);
  const int64_t rem = w - hg * units * chunk;
  const int64_t gs = min(chunk, items - hg * chunk);
  i = static_cast<int>(rem / gs);
  j = static_cast<int>(hg * chunk + rem % gs);
}

// The base descriptors pass through an empty asm so that the compiler builds
// them at the point of use (one add per step) instead of hoisting every step's
// descriptor out of the tile loop into the MMA thread's registers.  A step's
// descriptor is the base plus its byte offset / 16 (the start-address field).
__device__ __forceinline__ uint64_t opaque_u64(uint64_t x) {
  asm volatile("" : "+l"(x));
  return x;
}

// MN-major operand of a TS product: 16-key steps 2048 bytes apart
__device__ __forceinline__ uint64_t mn_desc(const uint8_t* s) {
  return opaque_u64(smem_desc(smem_u32(s), 16384, 1024));
}

template <int D>
__device__ __forceinline__ void issue_nn(uint32_t tD, const uint8_t* sA, const uint8_t* sB) {
  const uint64_t da = opaque_u64(smem_desc(smem_u32(sA), 16, 1024));
  const uint64_t db = opaque_u64(smem_desc(smem_u32(sB), 16, 1024));
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off16 = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
    umma_ss(tD, da + off16, db + off16, BCfg<D>::kIdescNN, kk > 0);
  }
}

// fp32 accumulator row (TMEM, D columns) * scale -> bf16 row in global memory
template <int D>
__device__ __forceinline__ void store_row(uint32_t tAcc, bool have, float scale, __nv_bfloat16* dst, bool store) {
#pragma unroll 1
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t o[32];
    if (have) {
      tmem_ld_32x32b_x32(tAcc + cc * 32, o);
      tmem_wait_ld();
      reg_fence(o);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) o[j] = 0u;
    }
    uint32_t pkd[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      pkd[j] = pack_bf16x2(__uint_as_float(o[2 * j]) * scale, __uint_as_float(o[2 * j + 1]) * scale);
    if (store) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
      for (int j = 0; j < 4; ++j) d4[j] = make_uint4(pkd[4 * j], pkd[4 * j + 1], pkd[4 * j + 2], pkd[4 * j + 3]);
    }
  }
}

}  // namespace

// ----------------------------------------------------------------------------
// preprocess: D = dO . O and LSE * log2(e), per (replica, plan row, tile row)
// ----------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) k_bwd_prep(const BwdParams p) {
  const int64_t blk = blockIdx.x;
  const int r = static_cast<int>(blk % p.plan.n_rows);
  const int j = static_cast<int>(blk / p.plan.n_rows);
  const GroupInfo g = p.plan.groups[p.plan.row_group[r]];
  int b, h0;
  replica_bh(p, g, j, b, h0);
  const int qpos = (r - g.row0) * kTile + threadIdx.x;
  int prow, h;
  row_pos_head(p, qpos, h0, prow, h);
  float dval = 0.f, lse2 = 0.f;
  if (qpos < g.q_len) {
    const int64_t tok = static_cast<int64_t>(g.q_off) + prow;
    const uint4* o4 = reinterpret_cast<const uint4*>(p.out + static_cast<int64_t>(b) * p.o_sb + tok * p.o_ss +
                                                     static_cast<int64_t>(h) * p.o_sh);
    const uint4* d4 = reinterpret_cast<const uint4*>(p.dout + static_cast<int64_t>(b) * p.do_sb + tok * p.do_ss +
                                                     static_cast<int64_t>(h) * p.do_sh);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint4 a = __ldg(o4 + c), z = __ldg(d4 + c);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w}, zv[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[e]));
        const float2 fz = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&zv[e]));
        acc[e] = fmaf(fa.x, fz.x, acc[e]);
        acc[e] = fmaf(fa.y, fz.y, acc[e]);
      }
    }
    dval = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    const int64_t li = p.varlen ? static_cast<int64_t>(h) * p.Sq_lse + tok
                                : (static_cast<int64_t>(b) * p.H + h) * p.Sq_lse + prow;
    const float L = p.lse[li];
    lse2 = (L == -INFINITY) ? 0.f : L * 1.4426950408889634f;  // a row that attends nothing has no listed pair
  }
  const int64_t wi = (static_cast<int64_t>(j) * p.plan.n_rows + r) * kTile + threadIdx.x;
  p.ws_lse2[wi] = -lse2;  // stored negated: the tile kernels add them
  p.ws_d[wi] = -dval;
  if (p.dq_acc) {  // the fused pass sums into this tile's dQ rows (contiguous, D floats a row)
    float4* z = reinterpret_cast<float4*>(p.dq_acc + (wi - threadIdx.x) * D);
#pragma unroll 4
    for (int i = threadIdx.x; i < kTile * D / 4; i += 128) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// ----------------------------------------------------------------------------
// dQ pass: one CTA per (plan row, replica), over the row's key-tile list
// ----------------------------------------------------------------------------
struct DqWork {
  GroupInfo g;
  int32_t r, e0, n, qt, b, h, hk, j;
};

// Warp roles of k_bwd_dq (384 threads): warp 0 TMA producer, warp 1 TMEM owner
// and MMA issuer, warps 2..3 idle, warps 4..11 the dS rows: warps 4..7 take keys
// [0, 64) of a tile and warps 8..11 keys [64, 128), one query row per thread (a
// warp reaches the TMEM lanes of its rank in the warpgroup).  Each warp loads its
// half of S and dP at once and releases the S / dP columns, so the next tile's
// S and dP products run on the tensor core while this tile's dS is made; dS
// alternates between two TMEM buffers, so a tile's dS never overwrites the one
// the previous tile's dQ products may still read.
constexpr int kDqThreads = 384;

template <int D>
__global__ void __launch_bounds__(kDqThreads, 1)
    k_bwd_dq(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
             const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const BwdParams p) {
  using C = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* const sQ = smem;
  uint8_t* const sdO = smem + C::kTileBytes;
  uint8_t* const sK0 = smem + 2 * C::kTileBytes;
  uint8_t* const sV0 = smem + (2 + kDqKStages) * C::kTileBytes;
  // BQ: Q and dO.  BF [2]: K(u) and V(u) landed (by tile parity).  KE [3]: K
  // stage free (dQ(u) done).  VE [2]: V stage free (dP(u) done).  BS: S and dP of
  // a tile ready.  BC: every dS warp has loaded its S / dP columns (8 warps).
  // BP [2]: dS of the tile written (8 warps), per tile parity, so a warp a tile
  // ahead never arrives on a phase the MMA thread still waits for.  BO: every
  // product done.
  enum { BQ = 0, BF = 1, KE = 3, VE = 6, BS = 8, BC = 9, BP = 10, BO = 12, BDONE = 13, NBAR = 14 };
  __shared__ __align__(8) uint64_t bars[NBAR];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ DqWork wk_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  auto sK = [&](int st) { return sK0 + st * C::kTileBytes; };
  auto sV = [&](int st) { return sV0 + st * C::kTileBytes; };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), (i == BC || i == BP || i == BP + 1) ? 8 : 1);
    fence_barrier_init();
    int i, j;
    chunked_decode(blockIdx.x, p.plan.n_rows, p.rep, p.head_chunk, i, j);
    uint32_t* const err = p.plan.err;
    (void)err;
    const int2 rw = p.plan.row_work[BFA_IDX(i, p.plan.n_rows, err)];  // {row, its group}, longest first
    const int r = static_cast<int>(BFA_IDX(rw.x, p.plan.n_rows, err));
    DqWork w;
    w.g = p.plan.groups[BFA_IDX(rw.y, p.plan.n_groups, err)];
    w.r = r;
    w.e0 = p.plan.row_ptr[r];
    w.n = p.plan.row_ptr[r + 1] - w.e0;
#ifdef BFA_CHECKED
    // a list outside the plan's arrays, or a row outside its group, is reported and not walked
    if (!(w.n >= 0 && w.n <= w.g.nkt && w.e0 >= 0 && w.e0 + w.n <= p.plan.cap_tiles && r >= w.g.row0 &&
          r < w.g.row0 + w.g.nqt && j >= 0 && j < p.rep)) {
      atomicOr(err, DEVERR_BOUNDS);
      w.e0 = 0;
      w.n = 0;
    }
#endif
    w.qt = r - w.g.row0;
    w.j = j;
    replica_bh(p, w.g, j, w.b, w.h);
    w.hk = w.h / (p.H / p.Hkv);
    wk_s = w;
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const DqWork& wk = wk_s;
  const uint64_t cap = p.wait_ns;
  const int n = wk.n;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmdO);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const int qs = wk.g.q_off + wk.qt * kTile;
      mbar_expect_tx(bar(BQ), 2 * C::kTileBytes);
      load_q_tile<C::kPanels>(p, &tmQ, sQ, bar(BQ), wk.h, wk.hk, qs, wk.b);
      load_q_tile<C::kPanels>(p, &tmdO, sdO, bar(BQ), wk.h, wk.hk, qs, wk.b);
      const int32_t* kv = p.plan.kv_tile + wk.e0;
      int last[kBwdStages] = {-1, -1};
      int kt_next = kv[0];
      for (int u = 0; u < n; ++u) {
        const int kt = kt_next;
        if (u + 1 < n) kt_next = kv[u + 1];
        const int st = u & 1, sk = u % kDqKStages;
        // K(u) over K(u - 3) once dQ(u - 3) is done; V(u) over V(u - 2) once dP(u - 2) is
        if (u >= kDqKStages && !mbar_wait_fast(bar(KE + sk), (u / kDqKStages - 1) & 1, cap, &abort_flag)) break;
        if (u >= kBwdStages && !mbar_wait_fast(bar(VE + st), ((u >> 1) - 1) & 1, cap, &abort_flag)) break;
        const uint32_t f = bar(BF + st);
        mbar_expect_tx(f, 2 * C::kTileBytes);
        const int ks = wk.g.k_off + kt * kTile;
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn) {
          tma_load_4d(smem_u32(sK(sk) + pn * 16384), &tmK, f, pn * 64, wk.hk, ks, wk.b);
          tma_load_4d(smem_u32(sV(st) + pn * 16384), &tmV, f, pn * 64, wk.hk, ks, wk.b);
        }
        last[st] = u;
      }
      mbar_drain(bar(BQ), 0, &abort_flag);
      for (int st = 0; st < kBwdStages; ++st)
        if (last[st] >= 0) mbar_drain(bar(BF + st), (last[st] >> 1) & 1, &abort_flag);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per tile u: once every dS warp holds S(u) and dP(u), S(u+1) and dP(u+1)
    // go to the tensor core; then, once dS(u) is written, dQ += dS(u) K(u) in one
    // burst (it queues behind S(u+1), dP(u+1), so finer grains gain nothing and
    // cost a wait each).  The commit after S(t), dP(t) also frees V(t); the one
    // after dQ(u) frees K(u).
    if (lane == 0 && n > 0) {
      // TMEM: S [0,128), dP [128,256), dQ [256,256+D), dS (bf16 pairs) [384,448) / [448,512)
      const uint32_t tS = tmem, tdP = tmem + 128, tdQ = tmem + 256;
      bool ok = mbar_wait_fast(bar(BQ), 0, cap, &abort_flag);
      if (ok) ok = mbar_wait_fast(bar(BF), 0, cap, &abort_flag);
      if (ok) {
        tc_fence_after();
        issue_nn<D>(tS, sQ, sK(0));    // S = Q K^T
        issue_nn<D>(tdP, sdO, sV(0));  // dP = dO V^T
        umma_commit(bar(BS));
        umma_commit(bar(VE + 0));
      }
      for (int u = 0; ok && u < n; ++u) {
        const int sk = u % kDqKStages;
        const uint32_t tdS = tmem + 384 + 64 * (u & 1);
        if (!mbar_wait_fast(bar(BC), u & 1, cap, &abort_flag)) { ok = false; break; }
        if (u + 1 < n) {
          const int st1 = (u + 1) & 1;
          if (!mbar_wait_fast(bar(BF + st1), ((u + 1) >> 1) & 1, cap, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_nn<D>(tS, sQ, sK((u + 1) % kDqKStages));
          issue_nn<D>(tdP, sdO, sV(st1));
          umma_commit(bar(BS));
          umma_commit(bar(VE + st1));
        }
        if (!mbar_wait_fast(bar(BP + (u & 1)), (u >> 1) & 1, cap, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dk = mn_desc(sK(sk));
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ts(tdQ, tdS + kk * 8, dk + kk * (2048 >> 4), C::kIdescD, (u > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(KE + sk));
      }
      if (ok) umma_commit(bar(BO));
      umma_commit(bar(BDONE));
      mbar_drain(bar(BDONE), 0, &abort_flag);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ dS rows
    const int quarter = warp & 3;
    const int half = (warp >> 2) - 1;  // keys [64 half, 64 half + 64) of each tile
    const int row = quarter * 32 + lane;
    const int qpos = wk.qt * kTile + row;
    const uint32_t tLane = tmem_addr(tmem, quarter * 32, 0);
    const GroupCtx ctx = group_ctx(wk.g);
    const int64_t wi = (static_cast<int64_t>(wk.j) * p.plan.n_rows + wk.r) * kTile + row;
    const float nlse2 = p.ws_lse2[wi], nd = p.ws_d[wi];  // -LSE * log2(e), -D
    const float c = p.scale_log2;
    bool ok = true;
    int kt_next = n > 0 ? p.plan.kv_tile[wk.e0] : 0;
    int part_next = n > 0 ? p.plan.part[wk.e0] : -1;
    for (int u = 0; u < n; ++u) {
      const int kt = kt_next, part = part_next;
      if (u + 1 < n) {
        kt_next = p.plan.kv_tile[wk.e0 + u + 1];
        part_next = p.plan.part[wk.e0 + u + 1];
      }
      uint32_t am[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      const bool masked = part >= 0 || (kt + 1) * kTile > wk.g.k_len;
      if (masked) row_mask_words(p.plan, ctx, qpos, row, kt, part, am);
      const bool got = mbar_wait(bar(BS), u & 1, cap, &abort_flag);
      if (__any_sync(0xffffffffu, !got)) { ok = false; break; }
      tc_fence_after();
      // this warp's 64 columns of S and dP in one round of loads; then the
      // columns are released for the next tile's products
      uint32_t sv[2][32], dv[2][32];
      tmem_ld_32x32b_x32(tLane + 64 * half, sv[0]);
      tmem_ld_32x32b_x32(tLane + 64 * half + 32, sv[1]);
      tmem_ld_32x32b_x32(tLane + 128 + 64 * half, dv[0]);
      tmem_ld_32x32b_x32(tLane + 128 + 64 * half + 32, dv[1]);
      tmem_wait_ld();
      reg_fence(sv[0]);
      reg_fence(sv[1]);
      reg_fence(dv[0]);
      reg_fence(dv[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BC));
      const uint32_t tdS = tLane + 384 + 64 * (u & 1);
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int gc = 2 * half + cc;  // 32-key chunk of the tile
        if (masked) {  // masked scores become -inf, so 2^(...) is 0 (partial and edge tiles only)
          const uint32_t bits = half ? am[2 + cc] : am[cc];
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (!((bits >> j) & 1u)) sv[cc][j] = __float_as_uint(-INFINITY);
        }
        uint32_t pk[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int c0 = 2 * jj, c1 = 2 * jj + 1;
          const float s0 = __uint_as_float(sv[cc][c0]), s1 = __uint_as_float(sv[cc][c1]);
          const float p0 = ex2_approx(fmaf(s0, c, nlse2));
          const float p1 = ex2_approx(fmaf(s1, c, nlse2));
          pk[jj] = pack_bf16x2(p0 * (__uint_as_float(dv[cc][c0]) + nd), p1 * (__uint_as_float(dv[cc][c1]) + nd));
        }
        tmem_st_32x32b_x16(tdS + gc * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BP + (u & 1)));
    }
    bool done = ok;
    if (ok && n > 0) {
      const bool got = mbar_wait(bar(BO), 0, cap, &abort_flag);
      done = !__any_sync(0xffffffffu, !got);
    }
    tc_fence_after();
    if (done) {
      int prow, hrow;
      row_pos_head(p, qpos, wk.h, prow, hrow);
      const int64_t tok = static_cast<int64_t>(wk.g.q_off) + prow;
      __nv_bfloat16* dst =
          p.dq + static_cast<int64_t>(wk.b) * p.dq_sb + tok * p.dq_ss + static_cast<int64_t>(hrow) * p.dq_sh;
      // each half of the warps writes half of the row's D columns
      store_row<D / 2>(tLane + 256 + half * (D / 2), n > 0, p.scale, dst + half * (D / 2), qpos < wk.g.q_len);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (abort_flag && threadIdx.x == 0) atomicOr(p.plan.err, DEVERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ----------------------------------------------------------------------------
// dK / dV pass: one CTA per (key-tile column, kv replica), over the column's
// query tiles for every query head that reads the kv head
// ----------------------------------------------------------------------------
struct KvWork {
  GroupInfo g;
  int32_t kt, e0, nq, nh, b, hk, steps;
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    k_bwd_dkdv(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO, const BwdParams p) {
  using C = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* const sK = smem;
  uint8_t* const sV = smem + C::kTileBytes;
  uint8_t* const sQ0 = smem + 2 * C::kTileBytes;                      // + 2 st tiles
  float* const sVec0 = reinterpret_cast<float*>(smem + (2 + 2 * kBwdStages) * C::kTileBytes);  // + st * 256
  // BKV: K and V.  BF / BE [2]: Q, dO and the query vectors of a step full /
  // free.  BS1 / BS2: S^T / dP^T of a step ready.  BP1 [4]: P^T of one 32-query
  // chunk written, BP2: dS^T of the step written (4 warps each).  BO: every
  // product done.
  enum { BKV = 0, BF = 1, BE = 3, BS1 = 5, BS2 = 6, BP1 = 7, BP2 = 11, BO = 12, BDONE = 13, NBAR = 14 };
  __shared__ __align__(8) uint64_t bars[NBAR];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ KvWork wk_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  auto sQ = [&](int st) { return sQ0 + (2 * st) * C::kTileBytes; };
  auto sdO = [&](int st) { return sQ0 + (2 * st + 1) * C::kTileBytes; };
  auto sVec = [&](int st) { return sVec0 + st * 2 * kTile; };  // [lse2 x 128][D x 128]

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), (i >= BP1 && i <= BP2) ? 4 : 1);
    fence_barrier_init();
    int i, jk;
    chunked_decode(blockIdx.x, p.n_cols, p.rep_kv, p.kv_chunk, i, jk);
    uint32_t* const err = p.plan.err;
    (void)err;
    const int c = static_cast<int>(BFA_IDX(p.col_order[BFA_IDX(i, p.n_cols, err)], p.n_cols, err));
    const int grp = static_cast<int>(BFA_IDX(p.col_group[c], p.plan.n_groups, err));
    KvWork w;
    w.g = p.plan.groups[grp];
    w.kt = c - p.col0[grp];
    w.e0 = p.col_ptr[c];
    w.nq = p.col_ptr[c + 1] - w.e0;
#ifdef BFA_CHECKED
    // a column outside the transposed lists, or a key tile outside its group, is reported and not walked
    if (!(w.nq >= 0 && w.nq <= w.g.nqt && w.e0 >= 0 && w.e0 + w.nq <= p.plan.cap_tiles && w.kt >= 0 &&
          w.kt < w.g.nkt && jk >= 0 && jk < p.rep_kv)) {
      atomicOr(err, DEVERR_BOUNDS);
      w.e0 = 0;
      w.nq = 0;
    }
#endif
    w.nh = p.pack_g > 1 ? 1 : p.H / p.Hkv;  // packed tiles hold every head of the kv head
    kv_replica_bh(p, w.g, jk, w.b, w.hk);
    w.steps = w.nq * w.nh;
    wk_s = w;
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const KvWork& wk = wk_s;
  const uint64_t cap = p.wait_ns;
  const int steps = wk.steps;
  // step s -> query head (packed plans: the base head of the kv head) and list entry
  auto step_head = [&](int s) { return (wk.hk * wk.nh + s / wk.nq) << p.pack_shift; };
  auto step_entry = [&](int s) { return wk.e0 + s % wk.nq; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && steps > 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmdO);
      const int ks = wk.g.k_off + wk.kt * kTile;
      mbar_expect_tx(bar(BKV), 2 * C::kTileBytes);
#pragma unroll
      for (int pn = 0; pn < C::kPanels; ++pn) {
        tma_load_4d(smem_u32(sK + pn * 16384), &tmK, bar(BKV), pn * 64, wk.hk, ks, wk.b);
        tma_load_4d(smem_u32(sV + pn * 16384), &tmV, bar(BKV), pn * 64, wk.hk, ks, wk.b);
      }
      int last[kBwdStages] = {-1, -1};
      for (int s = 0; s < steps; ++s) {
        const int st = s & 1;
        if (s >= kBwdStages && !mbar_wait_fast(bar(BE + st), ((s >> 1) - 1) & 1, cap, &abort_flag)) break;
        const int h = step_head(s);
        const int qt = p.q_tile[step_entry(s)];
        BFA_CHECK(qt >= 0 && qt < wk.g.nqt, p.plan.err);
        const int r = wk.g.row0 + qt;
        const int64_t wi = (static_cast<int64_t>(replica_of(p, wk.g, wk.b, h)) * p.plan.n_rows + r) * kTile;
        BFA_CHECK(wi >= 0 && wi + kTile <= static_cast<int64_t>(p.rep) * p.plan.n_rows * kTile, p.plan.err);
        const uint32_t f = bar(BF + st);
        mbar_expect_tx(f, 2 * C::kTileBytes + C::kVecBytes);
        const int qs = wk.g.q_off + qt * kTile;
        load_q_tile<C::kPanels>(p, &tmQ, sQ(st), f, h, wk.hk, qs, wk.b);
        load_q_tile<C::kPanels>(p, &tmdO, sdO(st), f, h, wk.hk, qs, wk.b);
        bulk_load(smem_u32(sVec(st)), p.ws_lse2 + wi, kTile * 4, f);
        bulk_load(smem_u32(sVec(st) + kTile), p.ws_d + wi, kTile * 4, f);
        last[st] = s;
      }
      mbar_drain(bar(BKV), 0, &abort_flag);
      for (int st = 0; st < kBwdStages; ++st)
        if (last[st] >= 0) mbar_drain(bar(BF + st), (last[st] >> 1) & 1, &abort_flag);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && steps > 0) {
      // Pipe order: dV(s), S^T(s+1), dK(s), dP^T(s+1), dV(s+1), ...  S^T(s+1) goes
      // over P^T(s) once dV(s) is issued and dP^T(s+1) over dS^T(s) once dK(s) is,
      // so the rows turn S^T(s+1) into P^T(s+1) while dK(s) and dP^T(s+1) run.
      const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;
      bool ok = mbar_wait_fast(bar(BKV), 0, cap, &abort_flag);
      if (ok) ok = mbar_wait_fast(bar(BF), 0, cap, &abort_flag);
      if (ok) {
        tc_fence_after();
        issue_nn<D>(tS, sK, sQ(0));  // S^T = K Q^T
        umma_commit(bar(BS1));
        issue_nn<D>(tdP, sV, sdO(0));  // dP^T = V dO^T
        umma_commit(bar(BS2));
      }
      for (int s = 0; ok && s < steps; ++s) {
        const int st = s & 1, st1 = st ^ 1;
        // dV += P^T dO, chunk by chunk as the rows write P^T
        for (int cc = 0; cc < 4; ++cc) {
          if (!mbar_wait_fast(bar(BP1 + cc), s & 1, cap, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ddo = mn_desc(sdO(st));
#pragma unroll
          for (int kk = 2 * cc; kk < 2 * cc + 2; ++kk)
            umma_ts(tdV, tS + kk * 8, ddo + kk * (2048 >> 4), C::kIdescD, (s > 0 || kk > 0) ? 1u : 0u);
        }
        if (!ok) break;
        if (s + 1 < steps) {
          if (!mbar_wait_fast(bar(BF + st1), ((s + 1) >> 1) & 1, cap, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_nn<D>(tS, sK, sQ(st1));
          umma_commit(bar(BS1));
        }
        // dK += dS^T Q
        if (!mbar_wait_fast(bar(BP2), s & 1, cap, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dq = mn_desc(sQ(st));
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ts(tdK, tdP + kk * 8, dq + kk * (2048 >> 4), C::kIdescD, (s > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(BE + st));
        if (s + 1 < steps) {
          issue_nn<D>(tdP, sV, sdO(st1));
          umma_commit(bar(BS2));
        }
      }
      if (ok) umma_commit(bar(BO));
      umma_commit(bar(BDONE));
      mbar_drain(bar(BDONE), 0, &abort_flag);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ P^T, dS^T rows (one key per thread)
    const int quarter = warp & 3;
    const int krow = quarter * 32 + lane;
    const int kpos = wk.kt * kTile + krow;
    const uint32_t tLane = tmem_addr(tmem, quarter * 32, 0);
    const GroupCtx ctx = group_ctx(wk.g);
    const float c = p.scale_log2;
    const uint64_t c2 = f2_pack(c, c);
    bool ok = true;
    for (int s = 0; s < steps; ++s) {
      const int st = s & 1;
      const int e = step_entry(s);
      const int qt = p.q_tile[e], part = p.tpart[e];
      BFA_CHECK(qt >= 0 && qt < wk.g.nqt, p.plan.err);
      uint32_t am[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      const bool masked = part >= 0 || (qt + 1) * kTile > wk.g.q_len;
      if (masked) col_mask_words(p.plan, ctx, kpos, krow, qt, part, am);
      // the step's query vectors (bulk copy on BF) and its S^T (BS1)
      const bool gv = mbar_wait(bar(BF + st), (s >> 1) & 1, cap, &abort_flag);
      const bool gs = gv && mbar_wait(bar(BS1), s & 1, cap, &abort_flag);
      if (__any_sync(0xffffffffu, !gs)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sLse = smem_u32(sVec(st)), sDv = smem_u32(sVec(st) + kTile);
      // phase 1: P^T = 2^(scale log2(e) S^T - LSE log2(e)) for the 128 queries, kept
      // in fp32 for phase 2 and written as bf16 over S^T (chunks of 32 queries,
      // the next chunk's load in flight; a chunk's P^T columns lie in columns
      // already read)
      uint64_t pv[64];  // P pairs
      {
        uint32_t sA[32], sB[32];
        tmem_ld_32x32b_x32(tLane, sA);
        tmem_wait_ld();
        reg_fence(sA);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t(&sv)[32] = (cc & 1) ? sB : sA;
          if (cc + 1 < 4) tmem_ld_32x32b_x32(tLane + (cc + 1) * 32, (cc & 1) ? sA : sB);
          if (masked) {  // masked scores become -inf, so 2^(...) is 0 (partial and edge steps only)
            const uint32_t bits = am[cc];
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (!((bits >> j) & 1u)) sv[j] = __float_as_uint(-INFINITY);
          }
          uint32_t pkp[16];
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 L = ld_shared_f4(sLse + (cc * 32 + q4 * 4) * 4);
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int col = q4 * 4 + 2 * h2;
              const float s0 = __uint_as_float(sv[col]), s1 = __uint_as_float(sv[col + 1]);
              const uint64_t nl = h2 ? f2_pack(L.z, L.w) : f2_pack(L.x, L.y);  // -LSE * log2(e)
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(s0, s1), c2, nl), x0, x1);
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              pv[cc * 16 + 2 * q4 + h2] = f2_pack(p0, p1);
              pkp[2 * q4 + h2] = pack_bf16x2(p0, p1);
            }
          }
          tmem_st_32x32b_x16(tLane + cc * 16, pkp);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BP1 + cc));
          if (cc + 1 < 4) {
            tmem_wait_ld();
            reg_fence((cc & 1) ? sA : sB);
          }
        }
      }
      // phase 2: dS^T = P^T * (dP^T - D), written as bf16 over dP^T
      const bool gd = mbar_wait(bar(BS2), s & 1, cap, &abort_flag);
      if (__any_sync(0xffffffffu, !gd)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t dA[32], dB[32];
        tmem_ld_32x32b_x32(tLane + 128, dA);
        tmem_wait_ld();
        reg_fence(dA);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t(&dp)[32] = (cc & 1) ? dB : dA;
          if (cc + 1 < 4) tmem_ld_32x32b_x32(tLane + 128 + (cc + 1) * 32, (cc & 1) ? dA : dB);
          uint32_t pks[16];
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 Dv = ld_shared_f4(sDv + (cc * 32 + q4 * 4) * 4);
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int col = q4 * 4 + 2 * h2;
              const uint64_t nd = h2 ? f2_pack(Dv.z, Dv.w) : f2_pack(Dv.x, Dv.y);  // -D
              float d0, d1;
              f2_unpack(f2_mul(pv[cc * 16 + 2 * q4 + h2],
                               f2_add(f2_pack(__uint_as_float(dp[col]), __uint_as_float(dp[col + 1])), nd)),
                        d0, d1);
              pks[2 * q4 + h2] = pack_bf16x2(d0, d1);
            }
          }
          tmem_st_32x32b_x16(tLane + 128 + cc * 16, pks);
          if (cc + 1 < 4) {
            tmem_wait_ld();
            reg_fence((cc & 1) ? dA : dB);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BP2));
    }
    bool done = ok;
    if (ok && steps > 0) {
      const bool got = mbar_wait(bar(BO), 0, cap, &abort_flag);
      done = !__any_sync(0xffffffffu, !got);
    }
    tc_fence_after();
    if (done) {
      const bool store = kpos < wk.g.k_len;
      const int64_t tok = static_cast<int64_t>(wk.g.k_off) + kpos;
      __nv_bfloat16* dvp =
          p.dv + static_cast<int64_t>(wk.b) * p.dv_sb + tok * p.dv_ss + static_cast<int64_t>(wk.hk) * p.dv_sh;
      __nv_bfloat16* dkp =
          p.dk + static_cast<int64_t>(wk.b) * p.dk_sb + tok * p.dk_ss + static_cast<int64_t>(wk.hk) * p.dk_sh;
      store_row<D>(tLane + 256, steps > 0, 1.f, dvp, store);
      store_row<D>(tLane + 256 + D, steps > 0, p.scale, dkp, store);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (abort_flag && threadIdx.x == 0) atomicOr(p.plan.err, DEVERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ----------------------------------------------------------------------------
// fused pass (D = 128): one CTA per (key-tile column, kv replica), walking the
// column's query-tile list as k_bwd_dkdv does, and making dQ from the same dS:
// dQ^T = K^T dS^T runs into the dP^T columns once dK has read dS^T there, and
// two more warpgroups read it out and sum it into an fp32 workspace.  Each
// (query tile, key tile) pair then costs five 128 x 128 x 128 products instead
// of the two passes' seven (S and dP are made once).
// ----------------------------------------------------------------------------
// Warp roles (512 threads): warp 0 TMA producer, warp 1 TMEM owner and MMA
// issuer, warps 2..3 idle, warps 4..7 the P^T / dS^T rows (one key per thread;
// dS^T also goes to shared memory as the B operand of dQ^T), warps 8..15 the dQ
// rows (one head dimension per thread, the TMEM lanes of dQ^T; warps 8..11 take
// queries [0, 64) and warps 12..15 queries [64, 128): on its own, one SM needs
// eight warps of scalar reductions in flight to reach the rate L2 accepts them
// at; inside this pass four and eight warps measured the same).
// Shared memory (1024-aligned, nothing static): K, V, Q[2], dO[2], dS^T, the
// query vectors of two steps, then the barriers and the work item.
// TMEM (512 columns): S^T [0,128) (P^T over [0,64)), dP^T [128,256) (dS^T over
// [128,192), then dQ^T), dV [256,384), dK [384,512).
constexpr int kFusedThreads = 512;
constexpr int kFusedRegsLaunch = 128;
constexpr uint32_t kFusedRegsWG0 = 120, kFusedRegsRows = 216, kFusedRegsDq = 88;
static_assert(128 * (kFusedRegsWG0 + kFusedRegsRows + 2 * kFusedRegsDq) == kFusedThreads * kFusedRegsLaunch,
              "register split");

struct FCfg {
  static constexpr int D = 128;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kOffDS = 6 * kTileBytes;
  static constexpr int kOffVec = 7 * kTileBytes;
  static constexpr int kOffCtl = kOffVec + kBwdStages * BCfg<D>::kVecBytes;
  static constexpr int kSmemBytes = kOffCtl + 512;
  static constexpr uint32_t kIdescQT = idesc_bf16_f32_mn(128, 128);  // A = K^T and B = dS^T, both MN-major
};
static_assert(FCfg::kSmemBytes <= 232448, "fused pass shared memory");

__global__ void __launch_bounds__(kFusedThreads, 1)
    k_bwd_fused(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO, const BwdParams p) {
  constexpr int D = FCfg::D;
  using C = BCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_fused[];
  // the swizzled tiles need 1024-byte alignment, which the declaration asks for;
  // a block that does not get it reports and does nothing
  if (smem_u32(smem_fused) & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.plan.err, DEVERR_BOUNDS);
    return;
  }
  uint8_t* const sK = smem_fused;
  uint8_t* const sV = smem_fused + C::kTileBytes;
  uint8_t* const sQ0 = smem_fused + 2 * C::kTileBytes;  // + 2 st tiles: Q(st), dO(st)
  uint8_t* const sdS = smem_fused + FCfg::kOffDS;
  float* const sVec0 = reinterpret_cast<float*>(smem_fused + FCfg::kOffVec);
  // BKV: K and V.  BF / BE [2]: Q, dO and the query vectors of a step full /
  // free.  BS1 / BS2: S^T / dP^T ready.  BP1 [4]: P^T of one 32-query chunk
  // written, BP2: dS^T written (TMEM and shared memory; 4 warps each).  BQ: dQ^T
  // ready, BQR: dQ^T read out (8 warps).  BO: every product done.
  enum { BKV = 0, BF = 1, BE = 3, BS1 = 5, BS2 = 6, BP1 = 7, BP2 = 11, BQ = 12, BQR = 13, BO = 14, BDONE = 15, NBAR = 16 };
  uint64_t* const bars = reinterpret_cast<uint64_t*>(smem_fused + FCfg::kOffCtl);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(bars + NBAR);
  int* const abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  KvWork* const wk_s = reinterpret_cast<KvWork*>(bars + NBAR + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  auto sQ = [&](int st) { return sQ0 + (2 * st) * C::kTileBytes; };
  auto sdO = [&](int st) { return sQ0 + (2 * st + 1) * C::kTileBytes; };
  auto sVec = [&](int st) { return sVec0 + st * 2 * kTile; };  // [lse2 x 128][D x 128]

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), (i >= BP1 && i <= BP2) ? 4 : (i == BQR ? 8 : 1));
    fence_barrier_init();
    int i, jk;
    chunked_decode(blockIdx.x, p.n_cols, p.rep_kv, p.kv_chunk, i, jk);
    uint32_t* const err = p.plan.err;
    (void)err;
    const int c = static_cast<int>(BFA_IDX(p.col_order[BFA_IDX(i, p.n_cols, err)], p.n_cols, err));
    const int grp = static_cast<int>(BFA_IDX(p.col_group[c], p.plan.n_groups, err));
    KvWork w;
    w.g = p.plan.groups[grp];
    w.kt = c - p.col0[grp];
    w.e0 = p.col_ptr[c];
    w.nq = p.col_ptr[c + 1] - w.e0;
#ifdef BFA_CHECKED
    if (!(w.nq >= 0 && w.nq <= w.g.nqt && w.e0 >= 0 && w.e0 + w.nq <= p.plan.cap_tiles && w.kt >= 0 &&
          w.kt < w.g.nkt && jk >= 0 && jk < p.rep_kv)) {
      atomicOr(err, DEVERR_BOUNDS);
      w.e0 = 0;
      w.nq = 0;
    }
#endif
    w.nh = p.pack_g > 1 ? 1 : p.H / p.Hkv;  // packed tiles hold every head of the kv head
    kv_replica_bh(p, w.g, jk, w.b, w.hk);
    w.steps = w.nq * w.nh;
    *wk_s = w;
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const KvWork& wk = *wk_s;
  const uint64_t cap = p.wait_ns;
  const int steps = wk.steps;
  auto step_head = [&](int s) { return (wk.hk * wk.nh + s / wk.nq) << p.pack_shift; };
  auto step_entry = [&](int s) { return wk.e0 + s % wk.nq; };

  if (warp < 4) {
    regs_dec<kFusedRegsWG0>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0 && steps > 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmdO);
        const int ks = wk.g.k_off + wk.kt * kTile;
        mbar_expect_tx(bar(BKV), 2 * C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn) {
          tma_load_4d(smem_u32(sK + pn * 16384), &tmK, bar(BKV), pn * 64, wk.hk, ks, wk.b);
          tma_load_4d(smem_u32(sV + pn * 16384), &tmV, bar(BKV), pn * 64, wk.hk, ks, wk.b);
        }
        int last[kBwdStages] = {-1, -1};
        for (int s = 0; s < steps; ++s) {
          const int st = s & 1;
          if (s >= kBwdStages && !mbar_wait_fast(bar(BE + st), ((s >> 1) - 1) & 1, cap, abort_flag)) break;
          const int h = step_head(s);
          const int qt = p.q_tile[step_entry(s)];
          BFA_CHECK(qt >= 0 && qt < wk.g.nqt, p.plan.err);
          const int r = wk.g.row0 + qt;
          const int64_t wi = (static_cast<int64_t>(replica_of(p, wk.g, wk.b, h)) * p.plan.n_rows + r) * kTile;
          BFA_CHECK(wi >= 0 && wi + kTile <= static_cast<int64_t>(p.rep) * p.plan.n_rows * kTile, p.plan.err);
          const uint32_t f = bar(BF + st);
          mbar_expect_tx(f, 2 * C::kTileBytes + C::kVecBytes);
          const int qs = wk.g.q_off + qt * kTile;
          load_q_tile<C::kPanels>(p, &tmQ, sQ(st), f, h, wk.hk, qs, wk.b);
          load_q_tile<C::kPanels>(p, &tmdO, sdO(st), f, h, wk.hk, qs, wk.b);
          bulk_load(smem_u32(sVec(st)), p.ws_lse2 + wi, kTile * 4, f);
          bulk_load(smem_u32(sVec(st) + kTile), p.ws_d + wi, kTile * 4, f);
          last[st] = s;
        }
        mbar_drain(bar(BKV), 0, abort_flag);
        for (int st = 0; st < kBwdStages; ++st)
          if (last[st] >= 0) mbar_drain(bar(BF + st), (last[st] >> 1) & 1, abort_flag);
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      // Pipe order: dV(s), S^T(s+1), dK(s), dQ^T(s), dP^T(s+1), dV(s+1), ...
      // dQ^T(s) goes over dS^T(s) once dK(s) is issued; dP^T(s+1) waits until
      // the dQ warps hold dQ^T(s) in registers.
      if (lane == 0 && steps > 0) {
        const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;
        bool ok = mbar_wait_fast(bar(BKV), 0, cap, abort_flag);
        if (ok) ok = mbar_wait_fast(bar(BF), 0, cap, abort_flag);
        if (ok) {
          tc_fence_after();
          issue_nn<D>(tS, sK, sQ(0));  // S^T = K Q^T
          umma_commit(bar(BS1));
          issue_nn<D>(tdP, sV, sdO(0));  // dP^T = V dO^T
          umma_commit(bar(BS2));
        }
        for (int s = 0; ok && s < steps; ++s) {
          const int st = s & 1, st1 = st ^ 1;
          // dV += P^T dO, chunk by chunk as the rows write P^T
          for (int cc = 0; cc < 4; ++cc) {
            if (!mbar_wait_fast(bar(BP1 + cc), s & 1, cap, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint64_t ddo = mn_desc(sdO(st));
#pragma unroll
            for (int kk = 2 * cc; kk < 2 * cc + 2; ++kk)
              umma_ts(tdV, tS + kk * 8, ddo + kk * (2048 >> 4), C::kIdescD, (s > 0 || kk > 0) ? 1u : 0u);
          }
          if (!ok) break;
          if (s + 1 < steps) {
            if (!mbar_wait_fast(bar(BF + st1), ((s + 1) >> 1) & 1, cap, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_nn<D>(tS, sK, sQ(st1));
            umma_commit(bar(BS1));
          }
          // dK += dS^T Q, then dQ^T = K^T dS^T (both operands MN-major in shared memory)
          if (!mbar_wait_fast(bar(BP2), s & 1, cap, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dq = mn_desc(sQ(st));
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ts(tdK, tdP + kk * 8, dq + kk * (2048 >> 4), C::kIdescD, (s > 0 || kk > 0) ? 1u : 0u);
          const uint64_t dkt = mn_desc(sK), dds = mn_desc(sdS);
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ss(tdP, dkt + kk * (2048 >> 4), dds + kk * (2048 >> 4), FCfg::kIdescQT, kk > 0 ? 1u : 0u);
          umma_commit(bar(BQ));
          umma_commit(bar(BE + st));
          if (s + 1 < steps) {
            if (!mbar_wait_fast(bar(BQR), s & 1, cap, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_nn<D>(tdP, sV, sdO(st1));
            umma_commit(bar(BS2));
          }
        }
        if (ok) umma_commit(bar(BO));
        umma_commit(bar(BDONE));
        mbar_drain(bar(BDONE), 0, abort_flag);
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ P^T, dS^T rows (one key per thread)
    regs_inc<kFusedRegsRows>();
    const int quarter = warp & 3;
    const int krow = quarter * 32 + lane;
    const int kpos = wk.kt * kTile + krow;
    const uint32_t tLane = tmem_addr(tmem, quarter * 32, 0);
    // row krow of the dS^T tile with its swizzle folded in: the row starts on a
    // 128-byte boundary, so chunk c16 of the row sits at (row ^ (c16 << 4))
    const uint32_t sdS_row = (smem_u32(sdS) + krow * 128) | ((krow & 7) << 4);
    const GroupCtx ctx = group_ctx(wk.g);
    const float c = p.scale_log2;
    const uint64_t c2 = f2_pack(c, c);
    // Key rows past the group's keys hold other tokens (the next sequence of a
    // packed batch); their dS^T must be 0 here, since dQ^T sums over every key
    // row of the tile.  A tile that runs past the keys is masked on every step.
    const bool kedge = (wk.kt + 1) * kTile > wk.g.k_len;
    const bool kout = kpos >= wk.g.k_len;
    bool ok = true;
    for (int s = 0; s < steps; ++s) {
      const int st = s & 1;
      const int e = step_entry(s);
      const int qt = p.q_tile[e], part = p.tpart[e];
      BFA_CHECK(qt >= 0 && qt < wk.g.nqt, p.plan.err);
      uint32_t am[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      const bool masked = part >= 0 || (qt + 1) * kTile > wk.g.q_len || kedge;
      if (masked) {
        col_mask_words(p.plan, ctx, kpos, krow, qt, part, am);
        if (kout) am[0] = am[1] = am[2] = am[3] = 0u;
      }
      const bool gv = mbar_wait(bar(BF + st), (s >> 1) & 1, cap, abort_flag);
      const bool gs = gv && mbar_wait(bar(BS1), s & 1, cap, abort_flag);
      if (__any_sync(0xffffffffu, !gs)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sLse = smem_u32(sVec(st)), sDv = smem_u32(sVec(st) + kTile);
      // phase 1: P^T = 2^(scale log2(e) S^T - LSE log2(e)), kept in fp32 for
      // phase 2 and written as bf16 over S^T, 32 queries at a time
      uint64_t pv[64];
      {
        uint32_t sA[32], sB[32];
        tmem_ld_32x32b_x32(tLane, sA);
        tmem_wait_ld();
        reg_fence(sA);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t(&sv)[32] = (cc & 1) ? sB : sA;
          if (cc + 1 < 4) tmem_ld_32x32b_x32(tLane + (cc + 1) * 32, (cc & 1) ? sA : sB);
          if (masked) {
            const uint32_t bits = am[cc];
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (!((bits >> j) & 1u)) sv[j] = __float_as_uint(-INFINITY);
          }
          uint32_t pkp[16];
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 L = ld_shared_f4(sLse + (cc * 32 + q4 * 4) * 4);
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int col = q4 * 4 + 2 * h2;
              const float s0 = __uint_as_float(sv[col]), s1 = __uint_as_float(sv[col + 1]);
              const uint64_t nl = h2 ? f2_pack(L.z, L.w) : f2_pack(L.x, L.y);
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(s0, s1), c2, nl), x0, x1);
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              pv[cc * 16 + 2 * q4 + h2] = f2_pack(p0, p1);
              pkp[2 * q4 + h2] = pack_bf16x2(p0, p1);
            }
          }
          tmem_st_32x32b_x16(tLane + cc * 16, pkp);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BP1 + cc));
          if (cc + 1 < 4) {
            tmem_wait_ld();
            reg_fence((cc & 1) ? sA : sB);
          }
        }
      }
      // phase 2: dS^T = P^T * (dP^T - D), as bf16 over dP^T (A operand of dK) and
      // into shared memory (B operand of dQ^T: row krow, queries contiguous, in
      // the 128-byte swizzled layout of a tile); the buffer is free: dQ^T of the
      // previous step was done before dP^T of this one was issued
      const bool gd = mbar_wait(bar(BS2), s & 1, cap, abort_flag);
      if (__any_sync(0xffffffffu, !gd)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t dA[32], dB[32];
        tmem_ld_32x32b_x32(tLane + 128, dA);
        tmem_wait_ld();
        reg_fence(dA);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t(&dp)[32] = (cc & 1) ? dB : dA;
          if (cc + 1 < 4) tmem_ld_32x32b_x32(tLane + 128 + (cc + 1) * 32, (cc & 1) ? dA : dB);
          uint32_t pks[16];
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 Dv = ld_shared_f4(sDv + (cc * 32 + q4 * 4) * 4);
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int col = q4 * 4 + 2 * h2;
              const uint64_t nd = h2 ? f2_pack(Dv.z, Dv.w) : f2_pack(Dv.x, Dv.y);
              float d0, d1;
              f2_unpack(f2_mul(pv[cc * 16 + 2 * q4 + h2],
                               f2_add(f2_pack(__uint_as_float(dp[col]), __uint_as_float(dp[col + 1])), nd)),
                        d0, d1);
              pks[2 * q4 + h2] = pack_bf16x2(d0, d1);
            }
          }
          tmem_st_32x32b_x16(tLane + 128 + cc * 16, pks);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c16 = (cc & 1) * 4 + j;  // 16-byte chunk of the row inside its 64-query panel
            st_shared_v4((sdS_row ^ (c16 << 4)) + (cc >> 1) * 16384, pks[4 * j], pks[4 * j + 1], pks[4 * j + 2],
                         pks[4 * j + 3]);
          }
          if (cc + 1 < 4) {
            tmem_wait_ld();
            reg_fence((cc & 1) ? dA : dB);
          }
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BP2));
    }
    bool done = ok;
    if (ok && steps > 0) {
      const bool got = mbar_wait(bar(BO), 0, cap, abort_flag);
      done = !__any_sync(0xffffffffu, !got);
    }
    tc_fence_after();
    if (done) {
      const bool store = kpos < wk.g.k_len;
      const int64_t tok = static_cast<int64_t>(wk.g.k_off) + kpos;
      __nv_bfloat16* dvp =
          p.dv + static_cast<int64_t>(wk.b) * p.dv_sb + tok * p.dv_ss + static_cast<int64_t>(wk.hk) * p.dv_sh;
      __nv_bfloat16* dkp =
          p.dk + static_cast<int64_t>(wk.b) * p.dk_sb + tok * p.dk_ss + static_cast<int64_t>(wk.hk) * p.dk_sh;
      store_row<D>(tLane + 256, steps > 0, 1.f, dvp, store);
      store_row<D>(tLane + 256 + D, steps > 0, p.scale, dkp, store);
    }
  } else {
    // ------------------------------------------------------------ dQ rows (one head dimension per thread)
    // A warp reads its 64 queries of dQ^T(s) out of TMEM, releases the columns
    // to dP^T(s+1), then sums them into the workspace: for each query, the 32
    // lanes add 32 consecutive floats (one 128-byte line).
    regs_dec<kFusedRegsDq>();
    const int quarter = warp & 3;
    const int q0 = warp >= 12 ? 64 : 0;
    const int dim = quarter * 32 + lane;
    const uint32_t tQT = tmem_addr(tmem + 128 + q0, quarter * 32, 0);
    for (int s = 0; s < steps; ++s) {
      const int h = step_head(s);
      const int qt = p.q_tile[step_entry(s)];
      BFA_CHECK(qt >= 0 && qt < wk.g.nqt, p.plan.err);
      const int64_t wi =
          (static_cast<int64_t>(replica_of(p, wk.g, wk.b, h)) * p.plan.n_rows + wk.g.row0 + qt) * kTile;
      BFA_CHECK(wi >= 0 && wi + kTile <= static_cast<int64_t>(p.rep) * p.plan.n_rows * kTile, p.plan.err);
      const int nvalid = min(kTile, wk.g.q_len - qt * kTile) - q0;  // rows past the sequence stay 0
      float* const dst = p.dq_acc + (wi + q0) * D + dim;
      const bool got = mbar_wait(bar(BQ), s & 1, cap, abort_flag);
      if (__any_sync(0xffffffffu, !got)) break;
      tc_fence_after();
      uint32_t v[64];
      tmem_ld_32x32b_x32(tQT, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_ld_32x32b_x32(tQT + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_wait_ld();
      reg_fence(v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BQR));
#ifdef BFA_CHECKED
      if (!(wi >= 0 && wi + kTile <= static_cast<int64_t>(p.rep) * p.plan.n_rows * kTile)) continue;
#endif
      if (nvalid >= 64) {
#pragma unroll
        for (int q = 0; q < 64; ++q) red_add_f32(dst + q * D, __uint_as_float(v[q]));
      } else {
#pragma unroll
        for (int q = 0; q < 64; ++q)
          if (q < nvalid) red_add_f32(dst + q * D, __uint_as_float(v[q]));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*static_cast<volatile int*>(abort_flag) && threadIdx.x == 0) atomicOr(p.plan.err, DEVERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// dQ = scale * (the fused pass's fp32 sums) as bf16, per (replica, plan row):
// a warp converts 32 rows, one 512-byte row per step (4 floats a lane)
__global__ void __launch_bounds__(128) k_bwd_dq_store(const BwdParams p) {
  constexpr int D = FCfg::D;
  const int64_t blk = blockIdx.x;
  const int r = static_cast<int>(blk % p.plan.n_rows);
  const int j = static_cast<int>(blk / p.plan.n_rows);
  const GroupInfo g = p.plan.groups[p.plan.row_group[r]];
  int b, h;
  replica_bh(p, g, j, b, h);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t wi = (static_cast<int64_t>(j) * p.plan.n_rows + r) * kTile;
  __nv_bfloat16* const base = p.dq + static_cast<int64_t>(b) * p.dq_sb;
#pragma unroll 4
  for (int i = 0; i < 32; ++i) {
    const int row = warp * 32 + i;
    const int qpos = (r - g.row0) * kTile + row;
    if (qpos >= g.q_len) break;
    const float4 a = *reinterpret_cast<const float4*>(p.dq_acc + (wi + row) * D + lane * 4);
    int prow, hrow;
    row_pos_head(p, qpos, h, prow, hrow);
    const int64_t tok = static_cast<int64_t>(g.q_off) + prow;
    uint2 o;
    o.x = pack_bf16x2(a.x * p.scale, a.y * p.scale);
    o.y = pack_bf16x2(a.z * p.scale, a.w * p.scale);
    *reinterpret_cast<uint2*>(base + tok * p.dq_ss + static_cast<int64_t>(hrow) * p.dq_sh + lane * 4) = o;
  }
}

// ----------------------------------------------------------------------------
// launchers (host)
// ----------------------------------------------------------------------------
int bwd_smem_bytes(int D) {
  return D == 64 ? max(BCfg<64>::kSmemBytes, BCfg<64>::kDqSmemBytes) : FCfg::kSmemBytes;
}

cudaError_t launch_bwd_prep(const BwdParams& p, cudaStream_t s) {
  const int64_t blocks = static_cast<int64_t>(p.rep) * p.plan.n_rows;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (p.D == 64) k_bwd_prep<64><<<static_cast<unsigned>(blocks), 128, 0, s>>>(p);
  else k_bwd_prep<128><<<static_cast<unsigned>(blocks), 128, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename K>
static cudaError_t bwd_prepare(K kernel, int smem) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

cudaError_t launch_bwd_dq(int D, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                          const CUtensorMap& tv, const BwdParams& p, int64_t n_work, cudaStream_t s) {
  if (n_work <= 0) return cudaSuccess;
  if (n_work > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (D == 64) {
    static cudaError_t ready = bwd_prepare(k_bwd_dq<64>, BCfg<64>::kDqSmemBytes);
    if (ready != cudaSuccess) return ready;
    k_bwd_dq<64><<<static_cast<unsigned>(n_work), kDqThreads, BCfg<64>::kDqSmemBytes, s>>>(tq, tdo, tk, tv, p);
  } else {
    static cudaError_t ready = bwd_prepare(k_bwd_dq<128>, BCfg<128>::kDqSmemBytes);
    if (ready != cudaSuccess) return ready;
    k_bwd_dq<128><<<static_cast<unsigned>(n_work), kDqThreads, BCfg<128>::kDqSmemBytes, s>>>(tq, tdo, tk, tv, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_fused(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                             const CUtensorMap& tdo, const BwdParams& p, int64_t n_work, cudaStream_t s) {
  if (n_work <= 0) return cudaSuccess;
  if (n_work > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  // the setmaxnreg split is only safe with exactly kFusedRegsLaunch registers a thread
  static cudaError_t ready = []() {
    cudaFuncAttributes a;
    cudaError_t e = cudaFuncGetAttributes(&a, k_bwd_fused);
    if (e != cudaSuccess) return e;
    if (a.numRegs != kFusedRegsLaunch) return cudaErrorInvalidKernelImage;
    return bwd_prepare(k_bwd_fused, FCfg::kSmemBytes);
  }();
  if (ready != cudaSuccess) return ready;
  k_bwd_fused<<<static_cast<unsigned>(n_work), kFusedThreads, FCfg::kSmemBytes, s>>>(tk, tv, tq, tdo, p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq_store(const BwdParams& p, cudaStream_t s) {
  const int64_t blocks = static_cast<int64_t>(p.rep) * p.plan.n_rows;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  k_bwd_dq_store<<<static_cast<unsigned>(blocks), 128, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dkdv(int D, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                            const CUtensorMap& tdo, const BwdParams& p, int64_t n_work, cudaStream_t s) {
  if (n_work <= 0) return cudaSuccess;
  if (n_work > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (D == 64) {
    static cudaError_t ready = bwd_prepare(k_bwd_dkdv<64>, BCfg<64>::kSmemBytes);
    if (ready != cudaSuccess) return ready;
    k_bwd_dkdv<64><<<static_cast<unsigned>(n_work), kBwdThreads, BCfg<64>::kSmemBytes, s>>>(tk, tv, tq, tdo, p);
  } else {
    static cudaError_t ready = bwd_prepare(k_bwd_dkdv<128>, BCfg<128>::kSmemBytes);
    if (ready != cudaSuccess) return ready;
    k_bwd_dkdv<128><<<static_cast<unsigned>(n_work), kBwdThreads, BCfg<128>::kSmemBytes, s>>>(tk, tv, tq, tdo, p);
  }
  return cudaGetLastError();
}

}  // namespace bfa
