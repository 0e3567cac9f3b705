// C ABI of libsig.so (declared in include/sig.h).  Every entry point checks its
// arguments on the host and returns a status without launching anything when
// a check fails; otherwise it enqueues its kernels on the caller's stream and
// returns at once.
#include "../../include/sig.h"
#include "internal.h"
#include "nm_ex.h"

#include <cuda_runtime.h>

#include <algorithm>

using namespace sig;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
// Natural alignment of a 32-bit buffer (uint32 masks, int32 indices and
// counts, float32 vectors); NULL passes.
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? SIG_OK : SIG_ERR_CUDA; }

int check_gemv_shape(int64_t d_in, int64_t d_out) {
  if (d_in < 1 || d_in > kMaxDIn) return SIG_ERR_SHAPE;
  if (d_out < 8 || d_out % 8 != 0 || d_out > (int64_t)1 << 30) return SIG_ERR_SHAPE;
  if (d_in * d_out > ((int64_t)1 << 40)) return SIG_ERR_SHAPE;
  return SIG_OK;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool nm_pattern_ok(int n, int m) {
  const bool pow2 = m == 1 || m == 2 || m == 4 || m == 8 || m == 16 || m == 32;
  return pow2 && n >= 1 && n <= m;
}

}  // namespace

extern "C" {

const char* sig_status_string(int status) {
  switch (status) {
    case SIG_OK: return "ok";
    case SIG_ERR_NULL: return "a required pointer is NULL";
    case SIG_ERR_SHAPE: return "a size is out of range or inconsistent";
    case SIG_ERR_ALIGN: return "a pointer is not aligned as required";
    case SIG_ERR_WORKSPACE: return "workspace missing or too small";
    case SIG_ERR_CUDA: return "CUDA runtime error";
    case SIG_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    case SIG_ERR_ARG: return "an argument is out of range";
  }
  return "unknown status";
}

int sig_abi_version(void) { return 2; }

size_t sig_workspace_bytes(int op, int64_t d_in, int64_t d_out, int64_t rows) {
  switch (op) {
    case SIG_OP_SPARSE_GEMV:
      if (check_gemv_shape(d_in, d_out) != SIG_OK) return 0;
      return plan_gemv(d_in, d_out, false).ws_bytes();
    case SIG_OP_TOPK:
      return 0;
    case SIG_OP_GATED_MLP:
      if (check_gemv_shape(d_in, d_out) != SIG_OK || check_gemv_shape(d_out, d_in) != SIG_OK)
        return 0;
      return plan_gated(d_in, d_out).total;
    case SIG_OP_RANK_ADAPTER:
      if (check_gemv_shape(d_in, rows) != SIG_OK || check_gemv_shape(rows, d_out) != SIG_OK)
        return 0;
      return plan_rank(d_in, rows, d_out).total;
    case SIG_OP_SPARSE_GEMV_BATCH:
      if (check_gemv_shape(d_in, d_out) != SIG_OK || d_in % 8 != 0 || rows < 1 ||
          rows > kGemvMaxBatch)
        return 0;
      return plan_gemv_batch(d_in, d_out, (int)rows).ws_bytes();
    case SIG_OP_SPARSE_GEMV_Q8:
    case SIG_OP_SPARSE_GEMV_F8:
    case SIG_OP_SPARSE_GEMV_Q4:
      if (check_gemv_shape(d_in, d_out) != SIG_OK) return 0;
      return plan_gemv(d_in, d_out, false).ws_bytes();
    case SIG_OP_NM_GEMM:
      if (rows < 1 || d_in < 1) return 0;
      return round_up((size_t)rows * (size_t)d_in * 2, 256);   // the masked activation block
  }
  return 0;
}

int sig_workspace_init(void* ws, size_t ws_bytes, sig_stream_t stream) {
  if (ws_bytes == 0) return SIG_OK;
  if (ws == nullptr) return SIG_ERR_NULL;
  if (!aligned256(ws)) return SIG_ERR_ALIGN;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream));
}

int sparsify_threshold(const uint16_t* x, int64_t d, float t, uint32_t* mask_bits, int32_t* idx,
                       int32_t* nnz, sig_stream_t stream) {
  if (x == nullptr || mask_bits == nullptr) return SIG_ERR_NULL;
  if (d < 1 || d > kMaxDIn) return SIG_ERR_SHAPE;
  if (!aligned16(x) || !aligned4(mask_bits) || !aligned4(idx) || !aligned4(nnz)) return SIG_ERR_ALIGN;
  return cuda_status(launch_threshold_compact(x, (int)d, t, mask_bits, idx, nnz,
                                              (cudaStream_t)stream));
}

int sparsify_topk(const uint16_t* x, int64_t d, int64_t k, uint32_t* mask_bits, int32_t* idx,
                  int32_t* nnz, void* ws, size_t ws_bytes, sig_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  if (x == nullptr || mask_bits == nullptr || idx == nullptr || nnz == nullptr)
    return SIG_ERR_NULL;
  if (d < 1 || d > kMaxTopkD) return SIG_ERR_SHAPE;
  if (k < 0 || k > d) return SIG_ERR_ARG;
  if (!aligned16(x) || !aligned4(mask_bits) || !aligned4(idx) || !aligned4(nnz)) return SIG_ERR_ALIGN;
  return cuda_status(launch_topk(x, (int)d, (int)k, mask_bits, idx, nnz, (cudaStream_t)stream));
}

size_t sig_nm_packed_bytes(int64_t rows, int64_t d) {
  if (rows < 128 || rows % 128 != 0 || d < 128 || d % 128 != 0 || rows > (1 << 24) ||
      d > (1 << 20))
    return 0;
  return (size_t)rows * (size_t)d / 8 * 9;   // d/2 fp16 values + d/8 metadata bytes per row
}

int sparsify_nm(const uint16_t* X, int64_t rows, int64_t d, int n, int m, uint16_t* X_masked,
                uint32_t* mask_bits, void* packed, sig_stream_t stream) {
  if (!nm_pattern_ok(n, m)) return SIG_ERR_ARG;
  if (packed != nullptr && !(m == 4 && (n == 2 || n == 1))) return SIG_ERR_ARG;
  if (rows < 0 || d < 1 || d % m != 0 || d > ((int64_t)1 << 30)) return SIG_ERR_SHAPE;
  if (rows == 0) return SIG_OK;  // an empty batch: nothing to read or write
  if (X == nullptr || (X_masked == nullptr && mask_bits == nullptr && packed == nullptr))
    return SIG_ERR_NULL;
  if (packed != nullptr && sig_nm_packed_bytes(rows, d) == 0) return SIG_ERR_SHAPE;
  if (d % 8 != 0 || !aligned16(X) || (X_masked != nullptr && !aligned16(X_masked)) ||
      !aligned4(mask_bits) || !aligned16(packed))
    return SIG_ERR_ALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  if (X_masked != nullptr || mask_bits != nullptr) {
    const cudaError_t e = launch_nm_mask(X, rows, (int)d, n, m, X_masked, mask_bits, st);
    if (e != cudaSuccess) return SIG_ERR_CUDA;
  }
  if (packed != nullptr) {
    uint16_t* vals = static_cast<uint16_t*>(packed);
    uint8_t* meta = static_cast<uint8_t*>(packed) + (size_t)rows * (size_t)d;
    return cuda_status(launch_nm_pack(X, rows, (int)d, n, vals, meta, st));
  }
  return SIG_OK;
}

int sparse_gemv(const uint16_t* WT, int64_t d_in, int64_t d_out, const uint16_t* x, float t,
                const int32_t* idx, const int32_t* nnz, uint16_t* y, void* ws, size_t ws_bytes,
                sig_stream_t stream) {
  if (WT == nullptr || x == nullptr || y == nullptr) return SIG_ERR_NULL;
  if (idx != nullptr && nnz == nullptr) return SIG_ERR_NULL;
  const int sh = check_gemv_shape(d_in, d_out);
  if (sh != SIG_OK) return sh;
  if (!aligned16(WT) || !aligned16(x) || !aligned16(y) || !aligned4(idx) || !aligned4(nnz))
    return SIG_ERR_ALIGN;
  const GemvPlan p = plan_gemv(d_in, d_out, false);
  if (p.ws_bytes() > 0 && (ws == nullptr || ws_bytes < p.ws_bytes())) return SIG_ERR_WORKSPACE;
  if (ws != nullptr && !aligned256(ws)) return SIG_ERR_ALIGN;
  GemvLaunch a{};
  a.WT[0] = WT; a.y[0] = y; a.d_out[0] = (int)d_out;
  a.x = x; a.t = t; a.idx = idx; a.nnz = nnz; a.d_in = (int)d_in; a.ws = ws;
  return cuda_status(launch_gemv(idx == nullptr ? MASK_THRESH : MASK_IDX, EPI_STORE, p, a,
                                 (cudaStream_t)stream));
}

int sparse_gemv_batch(const uint16_t* WT, int64_t d_in, int64_t d_out, const uint16_t* X,
                      int64_t B, float t, uint16_t* Y, void* ws, size_t ws_bytes,
                      sig_stream_t stream) {
  if (WT == nullptr || X == nullptr || Y == nullptr) return SIG_ERR_NULL;
  if (B < 1 || B > kGemvMaxBatch) return SIG_ERR_ARG;
  const int sh = check_gemv_shape(d_in, d_out);
  if (sh != SIG_OK) return sh;
  if (d_in % 8 != 0) return SIG_ERR_SHAPE;
  if (!aligned16(WT) || !aligned16(X) || !aligned16(Y)) return SIG_ERR_ALIGN;
  const GemvPlan p = plan_gemv_batch(d_in, d_out, (int)B);
  if (p.ws_bytes() > 0 && (ws == nullptr || ws_bytes < p.ws_bytes())) return SIG_ERR_WORKSPACE;
  if (ws != nullptr && !aligned256(ws)) return SIG_ERR_ALIGN;
  return cuda_status(launch_gemv_batch(p, WT, X, Y, (int)B, (int)d_in, (int)d_out, t, ws,
                                       (cudaStream_t)stream));
}

namespace {

int quantised_gemv(int epi, const uint8_t* QT, const float* scale, int64_t d_in, int64_t d_out,
                   const uint16_t* x, float t, uint16_t* y, void* ws, size_t ws_bytes,
                   sig_stream_t stream) {
  if (QT == nullptr || scale == nullptr || x == nullptr || y == nullptr) return SIG_ERR_NULL;
  const int sh = check_gemv_shape(d_in, d_out);
  if (sh != SIG_OK) return sh;
  if (!aligned16(QT) || !aligned16(x) || !aligned16(y) || !aligned4(scale)) return SIG_ERR_ALIGN;
  const GemvPlan p = plan_gemv(d_in, d_out, false);
  if (p.ws_bytes() > 0 && (ws == nullptr || ws_bytes < p.ws_bytes())) return SIG_ERR_WORKSPACE;
  if (ws != nullptr && !aligned256(ws)) return SIG_ERR_ALIGN;
  GemvLaunch a{};
  a.QT = QT; a.col_scale = scale; a.y[0] = y; a.d_out[0] = (int)d_out;
  a.x = x; a.t = t; a.d_in = (int)d_in; a.ws = ws;
  return cuda_status(launch_gemv(MASK_THRESH, epi, p, a, (cudaStream_t)stream));
}

}  // namespace

int sparse_gemv_q8(const int8_t* QT, const float* scale, int64_t d_in, int64_t d_out,
                   const uint16_t* x, float t, uint16_t* y, void* ws, size_t ws_bytes,
                   sig_stream_t stream) {
  return quantised_gemv(EPI_SCALE_I8, reinterpret_cast<const uint8_t*>(QT), scale, d_in, d_out, x,
                        t, y, ws, ws_bytes, stream);
}

int sparse_gemv_f8(const uint8_t* QT, const float* scale, int64_t d_in, int64_t d_out,
                   const uint16_t* x, float t, uint16_t* y, void* ws, size_t ws_bytes,
                   sig_stream_t stream) {
  return quantised_gemv(EPI_SCALE_E4M3, QT, scale, d_in, d_out, x, t, y, ws, ws_bytes, stream);
}

int sparse_gemv_q4(const uint8_t* QT4, const float* scale, int64_t d_in, int64_t d_out,
                   const uint16_t* x, float t, uint16_t* y, void* ws, size_t ws_bytes,
                   sig_stream_t stream) {
  return quantised_gemv(EPI_SCALE_I4, QT4, scale, d_in, d_out, x, t, y, ws, ws_bytes, stream);
}

size_t sig_workspace_bytes_multi(int n_mat, const int64_t* d_out, int64_t d_in) {
  if (n_mat < 1 || n_mat > kGemvMaxMat || d_out == nullptr) return 0;
  for (int i = 0; i < n_mat; ++i)
    if (check_gemv_shape(d_in, d_out[i]) != SIG_OK) return 0;
  return plan_gemv_multi(d_in, d_out, n_mat, false).ws_bytes();
}

int sparse_gemv_multi(int n_mat, const uint16_t* const* WT, const int64_t* d_out, int64_t d_in,
                      const uint16_t* x, float t, const int32_t* idx, const int32_t* nnz,
                      uint16_t* const* y, void* ws, size_t ws_bytes, sig_stream_t stream) {
  if (WT == nullptr || d_out == nullptr || y == nullptr || x == nullptr) return SIG_ERR_NULL;
  if (idx != nullptr && nnz == nullptr) return SIG_ERR_NULL;
  if (n_mat < 1 || n_mat > kGemvMaxMat) return SIG_ERR_ARG;
  int64_t total = 0;
  for (int i = 0; i < n_mat; ++i) {
    if (WT[i] == nullptr || y[i] == nullptr) return SIG_ERR_NULL;
    const int sh = check_gemv_shape(d_in, d_out[i]);
    if (sh != SIG_OK) return sh;
    if (!aligned16(WT[i]) || !aligned16(y[i])) return SIG_ERR_ALIGN;
    total += d_out[i];
  }
  if (total > ((int64_t)1 << 30)) return SIG_ERR_SHAPE;
  if (!aligned16(x) || !aligned4(idx) || !aligned4(nnz)) return SIG_ERR_ALIGN;
  const GemvPlan p = plan_gemv_multi(d_in, d_out, n_mat, false);
  if (p.ws_bytes() > 0 && (ws == nullptr || ws_bytes < p.ws_bytes())) return SIG_ERR_WORKSPACE;
  if (ws != nullptr && !aligned256(ws)) return SIG_ERR_ALIGN;
  GemvLaunch a{};
  a.n_mat = n_mat;
  for (int i = 0; i < n_mat; ++i) {
    a.WT[i] = WT[i];
    a.y[i] = y[i];
    a.d_out[i] = (int)d_out[i];
  }
  a.x = x; a.t = t; a.idx = idx; a.nnz = nnz; a.d_in = (int)d_in; a.ws = ws;
  return cuda_status(launch_gemv(idx == nullptr ? MASK_THRESH : MASK_IDX, EPI_STORE, p, a,
                                 (cudaStream_t)stream));
}

int gated_mlp_sparse(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                     const uint16_t* WdT, const float* down_norms, int64_t d_model, int64_t d_ff,
                     float t, uint16_t* y, uint16_t* h_out, uint32_t* mask_out, void* ws,
                     size_t ws_bytes, sig_stream_t stream) {
  if (x == nullptr || WgT == nullptr || WuT == nullptr || WdT == nullptr ||
      down_norms == nullptr || y == nullptr)
    return SIG_ERR_NULL;
  int sh = check_gemv_shape(d_model, d_ff);
  if (sh == SIG_OK) sh = check_gemv_shape(d_ff, d_model);
  if (sh != SIG_OK) return sh;
  if (!aligned16(x) || !aligned16(WgT) || !aligned16(WuT) || !aligned16(WdT) || !aligned16(y) ||
      (h_out != nullptr && !aligned16(h_out)) || !aligned4(down_norms) || !aligned4(mask_out))
    return SIG_ERR_ALIGN;
  const GatedPlan g = plan_gated(d_model, d_ff);
  if (ws == nullptr || ws_bytes < g.total) return SIG_ERR_WORKSPACE;
  if (!aligned256(ws)) return SIG_ERR_ALIGN;
  char* base = reinterpret_cast<char*>(ws);
  uint16_t* h = h_out != nullptr ? h_out : reinterpret_cast<uint16_t*>(base + g.off_h);

  GemvLaunch up{};
  up.WT[0] = WgT; up.WT2 = WuT; up.y[0] = h; up.d_out[0] = (int)d_ff;
  up.x = x; up.d_in = (int)d_model; up.ws = base;
  cudaError_t e = launch_gemv(MASK_DENSE, EPI_SILU_MUL, g.up, up, (cudaStream_t)stream);
  if (e != cudaSuccess) return SIG_ERR_CUDA;

  GemvLaunch dn{};
  dn.WT[0] = WdT; dn.y[0] = y; dn.d_out[0] = (int)d_model;
  dn.x = h; dn.scale = down_norms; dn.t = t; dn.d_in = (int)d_ff; dn.mask_out = mask_out;
  dn.ws = base + g.off_down;
  return cuda_status(launch_gemv(MASK_THRESH_SCALED, EPI_STORE, g.down, dn, (cudaStream_t)stream));
}

int teal_mlp_sparse(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                    const uint16_t* WdT, int64_t d_model, int64_t d_ff, float t_x, float t_h,
                    uint16_t* y, uint16_t* h_out, uint32_t* mask_out, void* ws, size_t ws_bytes,
                    sig_stream_t stream) {
  if (x == nullptr || WgT == nullptr || WuT == nullptr || WdT == nullptr || y == nullptr)
    return SIG_ERR_NULL;
  int sh = check_gemv_shape(d_model, d_ff);
  if (sh == SIG_OK) sh = check_gemv_shape(d_ff, d_model);
  if (sh != SIG_OK) return sh;
  if (!aligned16(x) || !aligned16(WgT) || !aligned16(WuT) || !aligned16(WdT) || !aligned16(y) ||
      (h_out != nullptr && !aligned16(h_out)) || !aligned4(mask_out))
    return SIG_ERR_ALIGN;
  const GatedPlan g = plan_gated(d_model, d_ff);
  if (ws == nullptr || ws_bytes < g.total) return SIG_ERR_WORKSPACE;
  if (!aligned256(ws)) return SIG_ERR_ALIGN;
  char* base = reinterpret_cast<char*>(ws);
  uint16_t* h = h_out != nullptr ? h_out : reinterpret_cast<uint16_t*>(base + g.off_h);

  GemvLaunch up{};
  up.WT[0] = WgT; up.WT2 = WuT; up.y[0] = h; up.d_out[0] = (int)d_ff;
  up.x = x; up.t = t_x; up.d_in = (int)d_model; up.ws = base;
  cudaError_t e = launch_gemv(MASK_THRESH, EPI_SILU_MUL, g.up, up, (cudaStream_t)stream);
  if (e != cudaSuccess) return SIG_ERR_CUDA;

  GemvLaunch dn{};
  dn.WT[0] = WdT; dn.y[0] = y; dn.d_out[0] = (int)d_model;
  dn.x = h; dn.t = t_h; dn.d_in = (int)d_ff; dn.mask_out = mask_out;
  dn.ws = base + g.off_down;
  return cuda_status(launch_gemv(MASK_THRESH, EPI_STORE, g.down, dn, (cudaStream_t)stream));
}

int rank_adapter_sparse(const uint16_t* x, const uint16_t* BT, const uint16_t* AT, int64_t d_in,
                        int64_t r, int64_t d_out, float t, uint16_t* y, uint16_t* v_out,
                        uint32_t* mask_out, void* ws, size_t ws_bytes, sig_stream_t stream) {
  if (x == nullptr || BT == nullptr || AT == nullptr || y == nullptr) return SIG_ERR_NULL;
  int sh = check_gemv_shape(d_in, r);
  if (sh == SIG_OK) sh = check_gemv_shape(r, d_out);
  if (sh != SIG_OK) return sh;
  if (!aligned16(x) || !aligned16(BT) || !aligned16(AT) || !aligned16(y) ||
      (v_out != nullptr && !aligned16(v_out)) || !aligned4(mask_out))
    return SIG_ERR_ALIGN;
  const RankPlan g = plan_rank(d_in, r, d_out);
  if (ws == nullptr || ws_bytes < g.total) return SIG_ERR_WORKSPACE;
  if (!aligned256(ws)) return SIG_ERR_ALIGN;
  char* base = reinterpret_cast<char*>(ws);
  uint16_t* v = v_out != nullptr ? v_out : reinterpret_cast<uint16_t*>(base + g.off_v);

  GemvLaunch in{};
  in.WT[0] = BT; in.y[0] = v; in.d_out[0] = (int)r;
  in.x = x; in.d_in = (int)d_in; in.ws = base;
  cudaError_t e = launch_gemv(MASK_DENSE, EPI_STORE, g.in, in, (cudaStream_t)stream);
  if (e != cudaSuccess) return SIG_ERR_CUDA;

  GemvLaunch out{};
  out.WT[0] = AT; out.y[0] = y; out.d_out[0] = (int)d_out;
  out.x = v; out.t = t; out.d_in = (int)r; out.mask_out = mask_out;
  out.ws = base + g.off_out;
  return cuda_status(launch_gemv(MASK_SQUARE, EPI_STORE, g.out, out, (cudaStream_t)stream));
}

int sparsify_nm_ex(const uint16_t* X, int64_t rows, int64_t d, int n, int m, const float* shift,
                   const float* norms, int var, uint16_t* X_masked, uint32_t* mask_bits,
                   float* gamma_out, sig_stream_t stream) {
  if (!nm_pattern_ok(n, m)) return SIG_ERR_ARG;
  if (rows < 0 || d < 1 || d % m != 0 || d > ((int64_t)1 << 30)) return SIG_ERR_SHAPE;
  if (rows == 0) return SIG_OK;
  if (X == nullptr || X_masked == nullptr) return SIG_ERR_NULL;
  if (d % 8 != 0 || !aligned16(X) || !aligned16(X_masked) || (norms != nullptr && !aligned16(norms)) ||
      !aligned4(shift) || !aligned4(mask_bits) || !aligned4(gamma_out))
    return SIG_ERR_ALIGN;
  return cuda_status(launch_nm_ex(X, rows, (int)d, n, m, shift, norms, var != 0, X_masked,
                                  mask_bits, gamma_out, (cudaStream_t)stream));
}

int nm_act_gemm_ex(const uint16_t* X, int64_t rows, int64_t K, const uint16_t* WT, int64_t N,
                   int n, int m, const float* shift, const float* norms, int var,
                   const float* col_sums, uint16_t* Y, void* ws, size_t ws_bytes,
                   sig_stream_t stream) {
  if (X == nullptr || WT == nullptr || Y == nullptr) return SIG_ERR_NULL;
  if (shift != nullptr && col_sums == nullptr) return SIG_ERR_NULL;
  if (!nm_pattern_ok(n, m)) return SIG_ERR_ARG;
  if (rows < 128 || rows % 128 != 0 || K < 64 || K % 64 != 0 || N < 128 || N % 128 != 0 ||
      K % m != 0 || rows > (1 << 24) || K > (1 << 20) || N > (1 << 20))
    return SIG_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(WT) || !aligned16(Y) || (norms != nullptr && !aligned16(norms)) ||
      !aligned4(shift) || !aligned4(col_sums))
    return SIG_ERR_ALIGN;
  const size_t need = sig_workspace_bytes(SIG_OP_NM_GEMM, K, N, rows);
  if (ws == nullptr || ws_bytes < need) return SIG_ERR_WORKSPACE;
  if (!aligned256(ws)) return SIG_ERR_ALIGN;
  uint16_t* Xm = reinterpret_cast<uint16_t*>(ws);
  cudaError_t e = launch_nm_ex(X, rows, (int)K, n, m, shift, norms, var != 0, Xm, nullptr, nullptr,
                               (cudaStream_t)stream);
  if (e != cudaSuccess) return SIG_ERR_CUDA;
  return cuda_status(launch_gemm_f16_shift(Xm, WT, Y, (int)rows, (int)N, (int)K, shift, col_sums,
                                           (cudaStream_t)stream));
}

int sig_col_sums(const uint16_t* WT, int64_t rows, int64_t cols, float* sums,
                 sig_stream_t stream) {
  if (WT == nullptr || sums == nullptr) return SIG_ERR_NULL;
  if (rows < 1 || cols < 1 || cols > ((int64_t)1 << 30)) return SIG_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(WT) & 1u) != 0 || !aligned4(sums)) return SIG_ERR_ALIGN;
  return cuda_status(launch_col_sums(WT, rows, (int)cols, sums, (cudaStream_t)stream));
}

int sig_row_norms(const uint16_t* WT, int64_t rows, int64_t cols, float* norms,
                  sig_stream_t stream) {
  if (WT == nullptr || norms == nullptr) return SIG_ERR_NULL;
  if (rows < 0 || cols < 8 || cols % 8 != 0 || cols > ((int64_t)1 << 30)) return SIG_ERR_SHAPE;
  if (!aligned16(WT) || !aligned4(norms)) return SIG_ERR_ALIGN;
  return cuda_status(launch_row_norms(WT, rows, (int)cols, norms, (cudaStream_t)stream));
}

int nm_act_gemm(const uint16_t* X, int64_t rows, int64_t K, const uint16_t* WT, int64_t N, int n,
                int m, uint16_t* Y, void* ws, size_t ws_bytes, sig_stream_t stream) {
  if (X == nullptr || WT == nullptr || Y == nullptr) return SIG_ERR_NULL;
  if (!nm_pattern_ok(n, m)) return SIG_ERR_ARG;
  if (rows < 128 || rows % 128 != 0 || K < 64 || K % 64 != 0 || N < 128 || N % 128 != 0 ||
      K % m != 0 || rows > (1 << 24) || K > (1 << 20) || N > (1 << 20))
    return SIG_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(WT) || !aligned16(Y)) return SIG_ERR_ALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  if (n == m)   // every entry kept: the plain tensor-core GEMM on X
    return cuda_status(launch_gemm_f16(X, WT, Y, (int)rows, (int)N, (int)K, st));
  const size_t need = sig_workspace_bytes(SIG_OP_NM_GEMM, K, N, rows);
  if (ws == nullptr || ws_bytes < need) return SIG_ERR_WORKSPACE;
  if (!aligned256(ws)) return SIG_ERR_ALIGN;
  if (m == 4 && n <= 2 && K % 128 == 0) {
    // 2:4 (and 1:4 padded to 2:4): packed operand, sparse tensor cores
    uint16_t* vals = reinterpret_cast<uint16_t*>(ws);
    uint8_t* meta = reinterpret_cast<uint8_t*>(ws) + (size_t)rows * (size_t)K;
    if (launch_nm_pack(X, rows, (int)K, n, vals, meta, st) != cudaSuccess) return SIG_ERR_CUDA;
    return cuda_status(launch_gemm_sp(vals, meta, WT, Y, (int)rows, (int)N, (int)K, st));
  }
  uint16_t* Xm = reinterpret_cast<uint16_t*>(ws);
  cudaError_t e = launch_nm_mask(X, rows, (int)K, n, m, Xm, nullptr, st);
  if (e != cudaSuccess) return SIG_ERR_CUDA;
  return cuda_status(launch_gemm_f16(Xm, WT, Y, (int)rows, (int)N, (int)K, st));
}

int nm_act_gemm_packed(const void* packed, int64_t rows, int64_t K, const uint16_t* WT, int64_t N,
                       uint16_t* Y, sig_stream_t stream) {
  if (packed == nullptr || WT == nullptr || Y == nullptr) return SIG_ERR_NULL;
  if (sig_nm_packed_bytes(rows, K) == 0 || N < 128 || N % 128 != 0 || N > (1 << 20))
    return SIG_ERR_SHAPE;
  if (!aligned16(packed) || !aligned16(WT) || !aligned16(Y)) return SIG_ERR_ALIGN;
  const uint16_t* vals = static_cast<const uint16_t*>(packed);
  const uint8_t* meta = static_cast<const uint8_t*>(packed) + (size_t)rows * (size_t)K;
  return cuda_status(launch_gemm_sp(vals, meta, WT, Y, (int)rows, (int)N, (int)K,
                                    (cudaStream_t)stream));
}

int sig_set_wait_limit(long long cycles) {
  return cuda_status(set_wait_limit(cycles));
}

int sig_take_device_error(unsigned* code, sig_stream_t stream) {
  if (code == nullptr) return SIG_ERR_NULL;
  unsigned gemm = 0, gemv = 0;
  if (read_device_error(&gemm, (cudaStream_t)stream) != cudaSuccess) return SIG_ERR_CUDA;
  if (read_gemv_error(&gemv, (cudaStream_t)stream) != cudaSuccess) return SIG_ERR_CUDA;
  *code = gemm | gemv;
  return *code == 0u ? SIG_OK : SIG_ERR_TIMEOUT;
}

}  // extern "C"
