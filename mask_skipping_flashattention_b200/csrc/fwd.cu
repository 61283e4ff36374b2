// Fused mask-aware attention forward for sm_100a.
//
// One CTA computes one 128-row query tile of one (batch, head) against the key
// tiles its plan row lists (BinFlash: iterate a pre-sorted list of non-empty key
// blocks, run all-True blocks with no mask loads, apply the mask on partial
// blocks only, skip all-False blocks).  Work items are taken in the plan's
// longest-first row order, so the hardware's in-order CTA dispatch balances SMs
// by the number of non-empty tiles.
//
// Warp roles (256 threads, two CTAs per SM):
//   warp 0      TMA producer: Q once, then K_u / V_u of every listed tile u
//   warp 1      TMEM owner and single-thread tcgen05.mma issuer:
//                 S_u = Q K_u^T   (SS: both operands in shared memory, K-major)
//                 O  += P_u V_u   (TS: P_u read from TMEM, V_u MN-major in smem)
//   warps 2..3  idle (they give their registers to the softmax warpgroup)
//   warps 4..7  softmax: one query row per thread, the whole S row in registers;
//               mask on partial and edge tiles only, online base-2 softmax in
//               fp32, P_u written back to TMEM over S_u as packed bf16, lazy
//               rescale of O in TMEM; epilogue O / l -> bf16 and LSE.
//
// TMEM (256 columns): S / P at columns [0, 128), O at [128, 128 + D).
// Shared memory: Q, K, V tiles (128 x D bf16 each) in 64-column panels with the
// 128-byte swizzle that both TMA and the tensor core use.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fwd_params.cuh"
#include "plan_types.cuh"
#include "ptx.cuh"

namespace bfa {

using namespace ptx;



// 256 threads: warpgroup 0 = warp 0 TMA producer, warp 1 MMA issuer (warps 2-3
// idle), warpgroup 1 = softmax.  Two CTAs per SM: 128 registers per thread at
// launch, redistributed so the softmax holds a whole S row in registers.  The
// split must add up to the launch allocation: 128 * kRegsWG0 + 128 * kRegsWG1 ==
// 256 * kRegsLaunch (checked against the compiled kernel before launching).
constexpr int kThreads = 256;
constexpr int kRegsLaunch = 128;
constexpr uint32_t kRegsWG0 = 56;
constexpr uint32_t kRegsWG1 = 200;
static_assert(128 * kRegsWG0 + 128 * kRegsWG1 == kThreads * kRegsLaunch, "register split");
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled only when the max grows by > 2^8

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kSmemBytes = 3 * kTileBytes + 1024;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColO = 128;
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 1);
};

struct Work {
  int32_t e0, n;        // first listed tile and count
  int32_t b, h, hk;
  int32_t qt;           // query tile inside the group
  int32_t q_off, q_len, k_off, k_len;
  int32_t qid_off, kid_off, kbit_off;
};

__device__ __forceinline__ void decode_work(const FwdParams& p, int w, Work& wk) {
  const int64_t R = p.plan.n_rows;
  const int64_t chunk = p.head_chunk;
  const int64_t hg = w / (R * chunk);
  const int64_t rem = w - hg * R * chunk;
  const int64_t gs = min(chunk, static_cast<int64_t>(p.rep) - hg * chunk);
  const int i = static_cast<int>(rem / gs);
  const int j = static_cast<int>(hg * chunk + rem % gs);
  const int row = p.plan.order[i];
  const GroupInfo g = p.plan.groups[p.plan.row_group[row]];
  wk.e0 = p.plan.row_ptr[row];
  wk.n = p.plan.row_ptr[row + 1] - wk.e0;
  wk.qt = row - g.row0;
  if (p.plan.kind == 1 /*BFA_PLAN_DENSE*/) {
    wk.b = j / p.H;
    wk.h = j % p.H;
  } else if (p.plan.kind == 4 /*BFA_PLAN_BSR*/) {
    wk.b = g.b;
    wk.h = g.hkv * (p.H / p.Hkv) + j;
  } else {
    wk.b = p.varlen ? 0 : g.b;
    wk.h = j;
  }
  wk.hk = wk.h / (p.H / p.Hkv);
  wk.q_off = g.q_off;
  wk.q_len = g.q_len;
  wk.k_off = g.k_off;
  wk.k_len = g.k_len;
  wk.qid_off = g.qid_off;
  wk.kid_off = g.kid_off;
  wk.kbit_off = g.kbit_off;
}

// attend-bits of one query row against the 128 columns of key tile `kt`
__device__ __forceinline__ void row_mask_words(const FwdParams& p, const Work& wk, int row, int kt, int part,
                                               uint32_t (&am)[4]) {
  const int ncols = wk.k_len - kt * kTile;  // in-range columns (may exceed 128)
  const int qpos = wk.qt * kTile + row;     // position of the row inside its group
  if (p.plan.mask_mode == MASK_BITS) {
    if (part >= 0) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.plan.fine + static_cast<int64_t>(part) * kFineWordsPerTile +
                                                           row * kWordsPerTileRow));
      am[0] = v.x; am[1] = v.y; am[2] = v.z; am[3] = v.w;
    } else {
      am[0] = am[1] = am[2] = am[3] = 0xffffffffu;
    }
  } else if (p.plan.mask_mode == MASK_BLOCKID) {
    if (part >= 0) {
      const int32_t qb = p.plan.qid[wk.qid_off + qpos];
      const bool qv = p.plan.qvalid[wk.qid_off + qpos] != 0;
      const int4* kb4 = reinterpret_cast<const int4*>(p.plan.kid + wk.kid_off + kt * kTile);
      const uint4 kv = __ldg(reinterpret_cast<const uint4*>(p.plan.kbits + wk.kbit_off + kt * kWordsPerTileRow));
      const uint32_t kvw[4] = {kv.x, kv.y, kv.z, kv.w};
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
    } else {
      am[0] = am[1] = am[2] = am[3] = 0xffffffffu;
    }
  } else {  // MASK_POS: causal kv_pos <= q_pos, optional window q_pos - kv_pos < W
    int hi = p.plan.causal ? (qpos - kt * kTile) : 127;            // last attended column
    int lo = (p.plan.window >= 0) ? (qpos - kt * kTile - p.plan.window + 1) : 0;  // first attended column
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

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    bfa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::kTileBytes;
  uint8_t* sV = smem + 2 * C::kTileBytes;

  enum { BQ = 0, BKF, BKE, BVF, BVE, BS, BP, BO, BDONE, NBAR };
  __shared__ __align__(8) uint64_t bars[NBAR];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ Work wk_s;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(bar(BQ), 1);
    mbar_init(bar(BKF), 1);
    mbar_init(bar(BKE), 1);
    mbar_init(bar(BVF), 1);
    mbar_init(bar(BVE), 1);
    mbar_init(bar(BS), 1);
    mbar_init(bar(BP), 4);
    mbar_init(bar(BO), 1);
    mbar_init(bar(BDONE), 1);
    fence_barrier_init();
    decode_work(p, blockIdx.x, wk_s);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const Work wk = wk_s;
  const uint64_t cap = p.wait_ns;

  if (warp < 4) {
    // ============================================================ warpgroup 0
    regs_dec<kRegsWG0>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0 && wk.n > 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        const int qs = wk.q_off + wk.qt * kTile;
        mbar_expect_tx(bar(BQ), C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_4d(smem_u32(sQ + pn * 16384), &tmQ, bar(BQ), pn * 64, wk.h, qs, wk.b);
        int last_k = -1, last_v = -1;  // last issued phase of each full barrier
        for (int u = 0; u < wk.n; ++u) {
          const int kt = p.plan.kv_tile[wk.e0 + u];
          const int ks = wk.k_off + kt * kTile;
          if (u > 0 && !mbar_wait(bar(BKE), (u - 1) & 1, cap, &abort_flag)) break;
          mbar_expect_tx(bar(BKF), C::kTileBytes);
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_4d(smem_u32(sK + pn * 16384), &tmK, bar(BKF), pn * 64, wk.hk, ks, wk.b);
          last_k = u;
          if (u > 0 && !mbar_wait(bar(BVE), (u - 1) & 1, cap, &abort_flag)) break;
          mbar_expect_tx(bar(BVF), C::kTileBytes);
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_4d(smem_u32(sV + pn * 16384), &tmV, bar(BVF), pn * 64, wk.hk, ks, wk.b);
          last_v = u;
        }
        // every copy this CTA issued must land before it can exit (bounded; on the
        // normal path these phases completed long ago)
        volatile int no_abort = 0;
        mbar_wait(bar(BQ), 0, cap, &no_abort);
        if (last_k >= 0) mbar_wait(bar(BKF), last_k & 1, cap, &no_abort);
        if (last_v >= 0) mbar_wait(bar(BVF), last_v & 1, cap, &no_abort);
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0 && wk.n > 0) {
        const uint32_t tS = tmem + C::kColS, tO = tmem + C::kColO;
        bool ok = mbar_wait(bar(BQ), 0, cap, &abort_flag);
        for (int u = 0; ok && u < wk.n; ++u) {
          if (!mbar_wait(bar(BKF), u & 1, cap, &abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_ss(tS, smem_desc(smem_u32(sQ + off), 16, 1024), smem_desc(smem_u32(sK + off), 16, 1024),
                    C::kIdescQK, kk > 0);
          }
          umma_commit(bar(BS));
          umma_commit(bar(BKE));
          if (!mbar_wait(bar(BP), u & 1, cap, &abort_flag)) { ok = false; break; }
          if (!mbar_wait(bar(BVF), u & 1, cap, &abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ts(tO, tS + kk * 8, smem_desc(smem_u32(sV + kk * 2048), 16384, 1024), C::kIdescPV,
                    (u > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar(BVE));
        }
        if (ok) umma_commit(bar(BO));
        // every MMA issued must be finished before TMEM is released (bounded)
        umma_commit(bar(BDONE));
        volatile int no_abort = 0;
        mbar_wait(bar(BDONE), 0, cap, &no_abort);
      }
    }
  } else {
    // ============================================================ warpgroup 1: softmax
    regs_inc<kRegsWG1>();
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t tS = tmem_addr(tmem + C::kColS, quarter * 32, 0);
    const uint32_t tO = tmem_addr(tmem + C::kColO, quarter * 32, 0);
    const float c = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    int kt_next = wk.n > 0 ? p.plan.kv_tile[wk.e0] : 0;
    int part_next = wk.n > 0 ? p.plan.part[wk.e0] : -1;
    for (int u = 0; u < wk.n; ++u) {
      const int kt = kt_next, part = part_next;
      if (u + 1 < wk.n) {  // next list entry, off the critical path
        kt_next = p.plan.kv_tile[wk.e0 + u + 1];
        part_next = p.plan.part[wk.e0 + u + 1];
      }
      const bool masked = part >= 0 || (kt + 1) * kTile > wk.k_len;
      uint32_t am[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      if (masked) row_mask_words(p, wk, row, kt, part, am);

      const bool got = mbar_wait(bar(BS), u & 1, cap, &abort_flag);
      if (__any_sync(0xffffffffu, !got)) { ok = false; break; }  // warp-uniform exit
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
      // row max, 8 independent chains
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
      for (int j = 8; j < 128; ++j) mx8[j & 7] = fmaxf(mx8[j & 7], s[j]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float mnew = fmaxf(m, mx * c);
      // The reference max m only moves when some row of the warp grew by more
      // than 2^8; then every row of the warp moves to its true running max (alpha
      // is 1 for rows that did not grow).  The decision is warp-uniform because
      // the O rescale uses whole-warp TMEM loads and stores.
      if (__any_sync(0xffffffffu, mnew > m + kRescaleThreshold)) {
        const float alpha = (mnew == m) ? 1.f : ex2_approx(m - mnew);  // 0 when m = -inf
        l *= alpha;
        if (u > 0) {
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
      const float mref = (m == -INFINITY) ? 0.f : m;
      // p = 2^(s*c - m), 4 independent row-sum chains; packed bf16 pairs go to
      // the first 64 columns of S (the A operand of the P V product)
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const float p0 = ex2_approx(fmaf(s[2 * j], c, -mref));
        const float p1 = ex2_approx(fmaf(s[2 * j + 1], c, -mref));
        rs[j & 3] += p0 + p1;
        pk[j] = pack_bf16x2(p0, p1);
      }
      l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
      tmem_st_32x32b_x32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      tmem_st_32x32b_x32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BP));
    }
    // ---------------------------------------------------------- epilogue
    if (ok && wk.n > 0) {
      const bool got = mbar_wait(bar(BO), 0, cap, &abort_flag);
      ok = !__any_sync(0xffffffffu, !got);
    }
    tc_fence_after();
    const int qpos = wk.qt * kTile + row;
    const bool store = qpos < wk.q_len;  // TMEM loads below stay whole-warp; only stores are per row
    if (ok) {
      const int64_t tok = static_cast<int64_t>(wk.q_off) + qpos;
      __nv_bfloat16* op = p.out + static_cast<int64_t>(wk.b) * p.o_sb + tok * p.o_ss + static_cast<int64_t>(wk.h) * p.o_sh;
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        if (wk.n > 0) {
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
          for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pkd[4 * j], pkd[4 * j + 1], pkd[4 * j + 2], pkd[4 * j + 3]);
        }
      }
      if (p.lse && store) {
        const float lse = (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        const int64_t li = p.varlen ? static_cast<int64_t>(wk.h) * p.Sq_lse + tok
                                    : (static_cast<int64_t>(wk.b) * p.H + wk.h) * p.Sq_lse + qpos;
        p.lse[li] = lse;
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
static cudaError_t check_regs(K kernel) {
  cudaFuncAttributes a;
  cudaError_t e = cudaFuncGetAttributes(&a, kernel);
  if (e != cudaSuccess) return e;
  return a.numRegs == kRegsLaunch ? cudaSuccess : cudaErrorInvalidKernelImage;
}

cudaError_t launch_fwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdParams& p, int64_t n_work, cudaStream_t s) {
  if (n_work <= 0) return cudaSuccess;
  if (n_work > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (D == 64) {
    static bool set = false;
    if (!set) {
      cudaError_t e = check_regs(bfa_fwd_kernel<64>);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(bfa_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<64>::kSmemBytes);
      if (e != cudaSuccess) return e;
      set = true;
    }
    bfa_fwd_kernel<64><<<static_cast<unsigned>(n_work), kThreads, Cfg<64>::kSmemBytes, s>>>(tq, tk, tv, p);
  } else {
    static bool set = false;
    if (!set) {
      cudaError_t e = check_regs(bfa_fwd_kernel<128>);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(bfa_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg<128>::kSmemBytes);
      if (e != cudaSuccess) return e;
      set = true;
    }
    bfa_fwd_kernel<128><<<static_cast<unsigned>(n_work), kThreads, Cfg<128>::kSmemBytes, s>>>(tq, tk, tv, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(uint32_t* err, uint64_t cap, cudaStream_t s) {
  k_wait_selftest<<<1, 32, 0, s>>>(err, cap);
  return cudaGetLastError();
}

cudaError_t probe_fwd_kernels() {
  cudaFuncAttributes a;
  cudaError_t e = cudaFuncGetAttributes(&a, bfa_fwd_kernel<128>);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, bfa_fwd_kernel<64>);
  return e;
}

}  // namespace bfa
