// Internal host-side interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

namespace sig {

constexpr int kNumSMs = 148;         // B200: 2 dies x 74 SMs
constexpr int kGemvThreads = 256;    // 8 warps
constexpr int kGemvCtasPerSM = 4;    // residency the grid is sized for
constexpr int kGemvTile = 256;       // output columns per CTA (one warp spans them)
constexpr int kGemvMaxSplits = 64;   // K-splits per column tile (32 unless fewer than 16 tiles)
constexpr int kIdxCap = 4096;        // rows of a slice staged in shared memory at once
constexpr int kGemvMaxMat = 4;       // weights that can share one input in one launch
constexpr int kMaxDIn = 131072;
constexpr int kMaxTopkD = 131072;    // top-k stages its keys in the cluster's shared memory

// How the rows of a sparse GEMV are chosen.
enum MaskMode : int {
  MASK_THRESH = 0,         // |x_i| >= t, computed in the prologue
  MASK_THRESH_SCALED = 1,  // |x_i| * scale_i >= t (RaNA Eqn. 12 with scale = norms)
  MASK_IDX = 2,            // rows idx[0 .. *nnz) given by the caller
  MASK_DENSE = 3,          // every row
  MASK_SQUARE = 4          // x_i * x_i >= t (RaNA rank adapter masker, one float32 multiply)
};

// What happens to a finished output column, and the weight format it implies.
enum Epilogue : int {
  EPI_STORE = 0,      // fp16 weights: y_j = fp16(sum)
  EPI_SILU_MUL = 1,   // fp16 weights, dual product (g, u): h_j = fp16(SiLU(g_j) * u_j)
  EPI_SCALE_I8 = 2,   // int8 weights: y_j = fp16(s_j * sum)
  EPI_SCALE_E4M3 = 3, // fp8 e4m3 weights: y_j = fp16(s_j * sum)
  EPI_SCALE_I4 = 4    // int4 weights, two per byte: y_j = fp16(s_j * sum)
};

// Launch `kernel` with programmatic stream serialization (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

struct GemvPlan {
  int C;              // column tiles
  int S;              // K-splits (slices of the kept-row list), <= kGemvMaxSplits
  int chunk;          // rows of a slice staged in shared memory at once
  size_t smem;        // dynamic shared memory per CTA
  size_t counters;    // workspace bytes for one word per column tile (arrival
                      // counter, or epoch of the fp16 GEMV's tagged partials)
  size_t partials;    // workspace bytes for the slices' partial sums (float32;
                      // 64-bit {value, tag} words in the fp16 GEMV)
  size_t ws_bytes() const { return counters + partials; }
};

GemvPlan plan_gemv(int64_t d_in, int64_t d_out, bool dual);
GemvPlan plan_gemv_multi(int64_t d_in, const int64_t* d_out, int n_mat, bool dual);

// Workspace layout of the gated MLP: the dual (gate, up) product's counters and
// partials, then the down product's, then the fp16 hidden vector h.
struct GatedPlan {
  GemvPlan up, down;
  size_t off_down, off_h, total;
};

inline GatedPlan plan_gated(int64_t d_model, int64_t d_ff) {
  auto up256 = [](size_t v) { return (v + 255) / 256 * 256; };
  GatedPlan g;
  g.up = plan_gemv(d_model, d_ff, true);
  g.down = plan_gemv(d_ff, d_model, false);
  g.off_down = up256(g.up.ws_bytes());
  g.off_h = g.off_down + up256(g.down.ws_bytes());
  g.total = g.off_h + up256((size_t)d_ff * 2);
  return g;
}

// A few tokens with their own threshold masks through one weight (B <= 16).
constexpr int kGemvMaxBatch = 16;
GemvPlan plan_gemv_batch(int64_t d_in, int64_t d_out, int B);
cudaError_t launch_gemv_batch(const GemvPlan& p, const uint16_t* WT, const uint16_t* X, uint16_t* Y,
                              int B, int d_in, int d_out, float t, void* ws, cudaStream_t stream);

// Rank adapter y = A (m . v), v = fp16(B x): a dense GEMV into v, then the
// masked GEMV on A; one workspace holds both plans' scratch and v.
struct RankPlan {
  GemvPlan in, out;
  size_t off_out, off_v, total;
};

inline RankPlan plan_rank(int64_t d_in, int64_t r, int64_t d_out) {
  auto up256 = [](size_t v) { return (v + 255) / 256 * 256; };
  RankPlan g;
  g.in = plan_gemv(d_in, r, false);
  g.out = plan_gemv(r, d_out, false);
  g.off_out = up256(g.in.ws_bytes());
  g.off_v = g.off_out + up256(g.out.ws_bytes());
  g.total = g.off_v + up256((size_t)r * 2);
  return g;
}

struct GemvLaunch {
  int n_mat = 1;                         // weights sharing the input and its mask
  const uint16_t* WT[kGemvMaxMat] = {};  // each d_in x d_out[i], row-major
  uint16_t* y[kGemvMaxMat] = {};         // outputs (y, or h for EPI_SILU_MUL)
  int d_out[kGemvMaxMat] = {};
  const uint16_t* WT2 = nullptr;         // second weight of the dual (gate, up) product
  const uint16_t* x = nullptr;
  const float* scale = nullptr;          // MASK_THRESH_SCALED
  const float* col_scale = nullptr;      // EPI_SCALE_*: one float32 per output column
  const uint8_t* QT = nullptr;           // EPI_SCALE_*: the 8-bit weight (d_in x d_out bytes)
  const int32_t* idx = nullptr;          // MASK_IDX
  const int32_t* nnz = nullptr;          // MASK_IDX
  float t = 0.f;
  int d_in = 0;
  uint32_t* mask_out = nullptr;          // nullable: written by one CTA
  void* ws = nullptr;                    // plan.ws_bytes() bytes, counters zero on entry
};

cudaError_t launch_gemv(int mode, int epi, const GemvPlan& plan, const GemvLaunch& a,
                        cudaStream_t stream);

// Mask kernels (mask.cu).
cudaError_t launch_threshold_compact(const uint16_t* x, int d, float t, uint32_t* mask_bits,
                                     int32_t* idx, int32_t* nnz, cudaStream_t stream);
cudaError_t launch_topk(const uint16_t* x, int d, int k, uint32_t* mask_bits, int32_t* idx,
                        int32_t* nnz, cudaStream_t stream);
cudaError_t launch_nm_mask(const uint16_t* X, int64_t rows, int d, int n, int m,
                           uint16_t* X_masked, uint32_t* mask_bits, cudaStream_t stream);
cudaError_t launch_row_norms(const uint16_t* WT, int64_t rows, int cols, float* norms,
                             cudaStream_t stream);

// Tensor-core GEMM (nm_gemm.cu): Y = A * B, A [M x K] fp16 row-major,
// B given as WT [K x N] fp16 row-major, Y [M x N] fp16.
cudaError_t read_device_error(unsigned* out, cudaStream_t stream);   // GEMM word (gemm .cu)
cudaError_t read_gemv_error(unsigned* out, cudaStream_t stream);     // split-K finish word
cudaError_t set_wait_limit(long long cycles);   // <= 0: the default (~2 s)

cudaError_t launch_gemm_f16(const uint16_t* A, const uint16_t* WT, uint16_t* Y, int M, int N,
                            int K, cudaStream_t stream);

// 2:4 sparse-operand GEMM (nm_gemm.cu): Y = A WT with A given packed (vals
// [M x K/2] fp16, the two kept values of every block of four; meta the
// tensor-core metadata, 2048 bytes per 128 x 128 block, see sparsify_nm).
// M % 128 == 0, K % 128 == 0, N % 128 == 0.
cudaError_t launch_gemm_sp(const uint16_t* vals, const uint8_t* meta, const uint16_t* WT,
                           uint16_t* Y, int M, int N, int K, cudaStream_t stream);

// Packed 2:4 operand of X (mask.cu): n = 2 keeps the two largest |x| of every
// block of four, n = 1 the largest plus a zero at the block's smallest other
// position.  rows % 128 == 0, d % 128 == 0.
cudaError_t launch_nm_pack(const uint16_t* X, int64_t rows, int d, int n, uint16_t* vals,
                           uint8_t* meta, cudaStream_t stream);

}  // namespace sig
