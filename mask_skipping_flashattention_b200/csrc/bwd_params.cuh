// Parameters of the backward kernels (filled on the host, passed by value).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "plan_types.cuh"

namespace bfa {

struct BwdParams {
  PlanDev plan;
  int32_t B, H, Hkv, D;
  int32_t rep;         // (batch, head) replicas that share one plan row (as in the forward)
  int32_t rep_kv;      // (batch, kv head) replicas that share one key-tile column
  int32_t head_chunk;  // replicas kept together in the dQ work order (L2 reuse)
  int32_t kv_chunk;    // kv replicas kept together in the dK/dV work order
  int32_t varlen;
  int32_t Sq_lse;      // batched: per-batch query length (lse row pitch); varlen: total_q
  float scale;         // softmax scale
  float scale_log2;    // scale * log2(e)
  const __nv_bfloat16* out;
  int64_t o_sb, o_ss, o_sh;
  const __nv_bfloat16* dout;
  int64_t do_sb, do_ss, do_sh;
  const float* lse;
  __nv_bfloat16* dq;
  int64_t dq_sb, dq_ss, dq_sh;
  __nv_bfloat16* dk;
  int64_t dk_sb, dk_ss, dk_sh;
  __nv_bfloat16* dv;
  int64_t dv_sb, dv_ss, dv_sh;
  // per (replica, plan row, row of the tile), negated: -LSE * log2(e) and
  // -D = -dO . O, with rows past a sequence (and rows that attend nothing) 0
  float* ws_lse2;
  float* ws_d;
  // fused pass (D = 128): fp32 dQ / scale per (replica, plan row, row of the
  // tile), D values a row; zeroed by the preprocess, summed into by every key
  // tile of the row's list, then scaled into dq.  nullptr for the two-pass form.
  float* dq_acc;
  // GQA-packed query tiles (bfa_plan_bsr_packed): plan row t of a tile is query
  // position t >> pack_shift of head (kv head << pack_shift) + (t & (pack_g - 1));
  // Q and dO move through 5-D maps.  pack_g = 1: rows are positions of one head.
  int32_t pack_g;
  int32_t pack_shift;
  // transposed lists of the plan
  const int32_t* col0;
  const int32_t* col_group;
  const int32_t* col_ptr;
  const int32_t* q_tile;
  const int32_t* tpart;
  const int32_t* col_order;
  int32_t n_cols;
  uint64_t wait_ns;
};

cudaError_t launch_bwd_prep(const BwdParams& p, cudaStream_t s);
cudaError_t launch_bwd_dq(int D, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                          const CUtensorMap& tv, const BwdParams& p, int64_t n_work, cudaStream_t s);
cudaError_t launch_bwd_dkdv(int D, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                            const CUtensorMap& tdo, const BwdParams& p, int64_t n_work, cudaStream_t s);
cudaError_t launch_bwd_fused(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                             const CUtensorMap& tdo, const BwdParams& p, int64_t n_work, cudaStream_t s);
cudaError_t launch_bwd_dq_store(const BwdParams& p, cudaStream_t s);
int bwd_smem_bytes(int D);

}  // namespace bfa
