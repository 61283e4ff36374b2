// Parameters of the fused forward kernel (filled on the host, passed by value).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "plan_types.cuh"

namespace bfa {

struct FwdParams {
  PlanDev plan;
  int32_t B, H, Hkv, D;
  int32_t rep;          // (batch, head) replicas that share one plan row
  int32_t pair_heads;   // 1: a CTA runs two heads of one kv head on one row; 0: two rows of one head
  int32_t head_chunk;   // replica units kept together in the work order (K/V reuse in L2)
  int32_t varlen;
  int32_t Sq_lse;       // batched: per-batch query length (lse row pitch); varlen: total_q
  float scale_log2;     // softmax scale * log2(e)
  __nv_bfloat16* out;
  int64_t o_sb, o_ss, o_sh;
  float* lse;
  uint64_t wait_ns;
  // paged keys / values (0 = contiguous): key token t of sequence s lives at row
  // block_table[s * pages_per_seq + t / page_size] * page_size + t % page_size of
  // the cache viewed as one token axis
  const int32_t* block_table;
  int32_t page_size;
  int32_t pages_per_seq;
  // approximate mode: a tile whose scores all lie more than skip_log2 (log2 units)
  // below the rows' running maxima is dropped; <= 0 keeps the exact computation
  float skip_log2;
  // GQA-packed query tiles: row t of a plan tile is query position t >> pack_shift
  // of head (kv head << pack_shift) + (t & (pack_g - 1)); Q and O move through
  // 5-D maps.  pack_g = 1: rows are positions of one head.
  int32_t pack_g;
  int32_t pack_shift;
};

int fwd_smem_bytes(int D);
cudaError_t launch_fwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdParams& p, int64_t n_work, cudaStream_t s);
cudaError_t launch_wait_selftest(uint32_t* err, uint64_t cap, cudaStream_t s);
cudaError_t probe_fwd_kernels();

}  // namespace bfa
