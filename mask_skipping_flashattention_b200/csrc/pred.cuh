// Position-term predicates: attend(i, j) = OR over terms of
//   diag_lo <= i - j <= diag_hi  AND  q_lo <= i < q_hi  AND  k_lo <= j < k_hi
// (positions local to the sequence; INT32_MIN / INT32_MAX mean unbounded).
// For a fixed query row each term keeps one interval of keys, so the attend-bits
// of a row over a 128-key tile are an OR of interval masks.  The planner counts
// these bits to classify tiles exactly and the forward kernel masks its partial
// tiles with them: both use this one function.
#pragma once

#include <cstdint>

namespace bfa {

constexpr int kTermInts = 6;  // diag_lo, diag_hi, q_lo, q_hi, k_lo, k_hi

// bits c of the word covering keys c0 .. c0 + 31 that lie in [lo, hi]
__device__ __forceinline__ uint32_t interval_word(int64_t lo, int64_t hi, int64_t c0) {
  const int64_t a = lo - c0, z = hi - c0;
  if (z < 0 || a > 31 || a > z) return 0u;
  const uint32_t m_hi = (z >= 31) ? 0xffffffffu : ((2u << z) - 1u);
  const uint32_t m_lo = (a <= 0) ? 0xffffffffu : ~((1u << a) - 1u);
  return m_hi & m_lo;
}

// attend-bits of query position i against the 128 keys of key tile kt
// (keys beyond k_len never attend)
__device__ __forceinline__ void pred_words(const int32_t* __restrict__ terms, int n_terms, int i, int kt, int k_len,
                                           uint32_t (&am)[4]) {
  am[0] = am[1] = am[2] = am[3] = 0u;
  const int64_t c0 = static_cast<int64_t>(kt) * 128;
  for (int t = 0; t < n_terms; ++t) {
    const int32_t* T = terms + t * kTermInts;
    if (i < T[2] || i >= T[3]) continue;
    int64_t lo = static_cast<int64_t>(i) - T[1];          // i - j <= diag_hi
    int64_t hi = static_cast<int64_t>(i) - T[0];          // i - j >= diag_lo
    lo = lo > T[4] ? lo : static_cast<int64_t>(T[4]);     // j >= k_lo
    hi = hi < static_cast<int64_t>(T[5]) - 1 ? hi : static_cast<int64_t>(T[5]) - 1;  // j < k_hi
    lo = lo > 0 ? lo : 0;
    hi = hi < static_cast<int64_t>(k_len) - 1 ? hi : static_cast<int64_t>(k_len) - 1;
#pragma unroll
    for (int w = 0; w < 4; ++w) am[w] |= interval_word(lo, hi, c0 + 32 * w);
  }
}

// attend-bits of key position j against the 128 queries of query tile qt, the
// transposed form for the backward's key-tile pass (queries beyond q_len never
// attend): for a fixed key each term keeps one interval of queries
__device__ __forceinline__ void pred_words_col(const int32_t* __restrict__ terms, int n_terms, int j, int qt,
                                               int q_len, uint32_t (&am)[4]) {
  am[0] = am[1] = am[2] = am[3] = 0u;
  const int64_t r0 = static_cast<int64_t>(qt) * 128;
  for (int t = 0; t < n_terms; ++t) {
    const int32_t* T = terms + t * kTermInts;
    if (j < T[4] || j >= T[5]) continue;
    int64_t lo = static_cast<int64_t>(j) + T[0];          // i - j >= diag_lo
    int64_t hi = static_cast<int64_t>(j) + T[1];          // i - j <= diag_hi
    lo = lo > T[2] ? lo : static_cast<int64_t>(T[2]);     // i >= q_lo
    hi = hi < static_cast<int64_t>(T[3]) - 1 ? hi : static_cast<int64_t>(T[3]) - 1;  // i < q_hi
    lo = lo > 0 ? lo : 0;
    hi = hi < static_cast<int64_t>(q_len) - 1 ? hi : static_cast<int64_t>(q_len) - 1;
#pragma unroll
    for (int w = 0; w < 4; ++w) am[w] |= interval_word(lo, hi, r0 + 32 * w);
  }
}

}  // namespace bfa
