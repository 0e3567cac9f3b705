// Host-side interface of the weight-quantised sparse GEMV (int8 or fp8 e4m3
// weights, one float32 scale per output column).
#pragma once

#include "internal.h"

namespace sig {

constexpr int kQ8Tile = 512;   // output columns per CTA: 32 lanes x 16 8-bit weights
constexpr int kFmtInt8 = 0;    // two's-complement int8
constexpr int kFmtE4M3 = 1;    // fp8 e4m3 (OCP E4M3)

GemvPlan plan_gemv_q8(int64_t d_in, int64_t d_out);
cudaError_t launch_gemv_q8(const GemvPlan& p, int fmt, const uint8_t* QT, const float* scale,
                           const uint16_t* x, float t, uint16_t* y, int d_in, int d_out, void* ws,
                           cudaStream_t stream);

}  // namespace sig
