// N:M selection inside one 32-entry word of a row ("Motivating Next-Gen
// Accelerators with Flexible (N:M) Activation Sparsity ...", Methodology: in
// every block of M consecutive entries the N of largest magnitude are kept;
// Block Q-Sparse in the "Q-Sparse ..." rebuttal, A2).  M divides 32, so blocks
// never straddle a word.  Entries are ranked by the unique composite
// (magnitude key << 5 | (31 - position in block)): larger magnitude first,
// lower index first among equal magnitudes, NaN lowest.
#pragma once

#include "common.cuh"

namespace sig {

// One bitonic stage (K = run length, J = partner distance) and the ones after
// it; template recursion keeps every index a compile-time constant.  T is an
// unsigned composite type (uint32_t or uint64_t).
template <int M, int K, int J, typename T>
__device__ __forceinline__ void bitonic_stage(T (&s)[M]) {
#pragma unroll
  for (int i = 0; i < M; ++i) {
    const int l = i ^ J;
    if (l > i) {
      const T a = s[i], b = s[l];
      const T hi = a > b ? a : b, lo = a > b ? b : a;
      const bool desc = (i & K) == 0;      // the final merge leaves s descending
      s[i] = desc ? hi : lo;
      s[l] = desc ? lo : hi;
    }
  }
  if constexpr (J > 1) bitonic_stage<M, K, J / 2>(s);
  else if constexpr (K < M) bitonic_stage<M, K * 2, K>(s);
}

// Bits of the n largest composites among M unique composites (bit j for c[j]).
// M <= 8: count, for each entry, the entries ranked above it.  M >= 16: sort a
// copy descending with a bitonic network; the n-th largest is the minimum of
// the first n, and an entry is kept when it is at least that.
template <int M, typename T>
__device__ __forceinline__ uint32_t select_top_n(const T (&c)[M], int n) {
  uint32_t bits = 0;
  if constexpr (M <= 8) {
#pragma unroll
    for (int j = 0; j < M; ++j) {
      int rank = 0;
#pragma unroll
      for (int l = 0; l < M; ++l) rank += c[l] > c[j] ? 1 : 0;
      bits |= (rank < n ? 1u : 0u) << j;
    }
  } else {
    T s[M];
#pragma unroll
    for (int j = 0; j < M; ++j) s[j] = c[j];
    bitonic_stage<M, 2, 1>(s);
    T thr = ~T(0);
#pragma unroll
    for (int j = 0; j < M; ++j) thr = (j < n && s[j] < thr) ? s[j] : thr;
#pragma unroll
    for (int j = 0; j < M; ++j) bits |= (c[j] >= thr ? 1u : 0u) << j;
  }
  return bits;
}

// Keep-bits of a 32-entry word held as four 16-byte vectors (entry e of the
// word is half e & 7 of q[e >> 3]); only the first `cnt` entries (a multiple
// of M) are ranked.
template <int M>
__device__ __forceinline__ uint32_t nm_word_bits(const uint4 (&q)[4], int n, int cnt = 32) {
  uint32_t bits = 0;
#pragma unroll
  for (int b0 = 0; b0 < 32; b0 += M) {
    if (b0 < cnt) {
      uint32_t comp[M];
#pragma unroll
      for (int j = 0; j < M; ++j)
        comp[j] = (mag_key(lane_half(q[(b0 + j) >> 3], (b0 + j) & 7)) << 5) | (uint32_t)(31 - j);
      bits |= select_top_n<M>(comp, n) << b0;
    }
  }
  return bits;
}

// Keep-bits of the 8 entries of one 16-byte vector, for M dividing 8 (blocks
// never straddle the vector).
template <int M>
__device__ __forceinline__ uint32_t nm_vec_bits(const uint4& v, int n) {
  uint32_t bits = 0;
#pragma unroll
  for (int b0 = 0; b0 < 8; b0 += M) {
    uint32_t comp[M];
#pragma unroll
    for (int j = 0; j < M; ++j) comp[j] = (mag_key(lane_half(v, b0 + j)) << 5) | (uint32_t)(31 - j);
    bits |= select_top_n<M>(comp, n) << b0;
  }
  return bits;
}

// The 16-byte vector `v` (entries 8i .. 8i+7 of the word) with the entries
// whose keep-bit is clear set to +0.
__device__ __forceinline__ uint4 nm_apply(const uint4& v, uint32_t bits, int i) {
  const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
  uint32_t p[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int a = i * 8 + 2 * k;
    const uint32_t lo = ((bits >> a) & 1u) ? (wv[k] & 0xffffu) : 0u;
    const uint32_t hi = ((bits >> (a + 1)) & 1u) ? (wv[k] & 0xffff0000u) : 0u;
    p[k] = lo | hi;
  }
  return make_uint4(p[0], p[1], p[2], p[3]);
}

}  // namespace sig
