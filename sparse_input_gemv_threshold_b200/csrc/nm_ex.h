// Host-side interface of the N:M selection and mitigation variants (per-token
// shift, weight-aware score, variance correction) and of the GEMM that adds
// the shift back.
#pragma once

#include "internal.h"

namespace sig {

// Masked, optionally shifted and rescaled activation block (one warp per row).
cudaError_t launch_nm_ex(const uint16_t* X, int64_t rows, int d, int n, int m, const float* shift,
                         const float* norms, bool var, uint16_t* X_masked, uint32_t* mask_bits,
                         float* gamma_out, cudaStream_t stream);

// sums[j] = sum_i WT[i, j], accumulated in float64, rounded once to float32.
cudaError_t launch_col_sums(const uint16_t* WT, int64_t rows, int cols, float* sums,
                            cudaStream_t stream);

// Y = A WT (+ shift[row] * colsum[col] when shift is not NULL), tcgen05.
cudaError_t launch_gemm_f16_shift(const uint16_t* A, const uint16_t* WT, uint16_t* Y, int M, int N,
                                  int K, const float* shift, const float* colsum,
                                  cudaStream_t stream);

}  // namespace sig
