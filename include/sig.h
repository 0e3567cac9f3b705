/*
 * sig.h — C ABI of libsig.so: the activation-sparse linear layer for LLM
 * decoding on one NVIDIA B200 (sm_100a).
 *
 * The layer computes y = W (m . x): a mask m picks the entries of the
 * activation x that survive, and the product reads only the weight columns of
 * the surviving entries.  Sources, by page title and section:
 *   - "Training-Free Activation Sparsity in Large Language Models" (TEAL
 *     README), Abstract: magnitude threshold on the hidden states.
 *   - "Q-Sparse: All Large Language Models can be Fully Sparsely-Activated"
 *     (OpenReview rebuttal), A1 on MoE: top-k by magnitude per token; A2 on
 *     batched inference: Block Q-Sparse with N:M activation sparsity; A3:
 *     FLOPs of the product.
 *   - "Adaptive Rank Allocation: Speeding Up Modern Transformers with RaNA
 *     Adapters" (OpenReview rebuttal), Q3 Eqn. 12: the gated-MLP neuron
 *     masker; Q5.1: the masked product skips the columns of zero mask entries.
 *   - "Motivating Next-Gen Accelerators with Flexible (N:M) Activation
 *     Sparsity ..." (summary), Methodology: N kept in every block of M.
 *
 * Conventions shared by every entry point
 *   - Every pointer named WT, x, X, y, Y, h_out, mask_bits, idx, nnz, ws,
 *     down_norms, norms, packed, X_masked is a DEVICE pointer.  The caller owns
 *     every buffer; the library allocates nothing, keeps no pointer after the
 *     call returns, and never synchronises the device.
 *   - fp16 buffers hold IEEE binary16 bit patterns (uint16_t).
 *   - Weights are stored transposed: WT is d_in x d_out, row-major, so row i
 *     (2*d_out contiguous bytes) holds every weight that multiplies input i.
 *   - Masks are bit-packed: bit (i % 32) of word (i / 32) is m_i.  2-D masks
 *     pack each row on its own, rows padded to whole words.
 *   - Index lists are int32, strictly ascending; the count lives on the device
 *     (int32 *nnz), so no host round trip separates mask and product.
 *   - Magnitude ranking (top-k, N:M): larger |x| first; equal |x| by lower
 *     index first; +v/-v and +0/-0 tie; a NaN ranks below every number.
 *   - All work is enqueued asynchronously on `stream` (NULL = legacy default
 *     stream).  Calls that share a workspace must not overlap on the device.
 *   - Alignment: besides the 16-byte rules each entry point states, every
 *     uint32, int32 and float32 buffer (masks, index lists, counts, norms,
 *     shifts, sums, scales) must be 4-byte aligned and every fp16 buffer
 *     2-byte aligned; otherwise the call returns SIG_ERR_ALIGN.
 *   - Errors: arguments are checked on the host before anything is enqueued,
 *     and a non-zero sig_status comes back with nothing launched.  A launch
 *     failure returns SIG_ERR_CUDA.  Nothing throws across the ABI.
 */
#ifndef SIG_H
#define SIG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported with default visibility; everything else in libsig.so is hidden. */
#if defined(__GNUC__)
#define SIG_API __attribute__((visibility("default")))
#else
#define SIG_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* sig_stream_t;

typedef enum {
  SIG_OK = 0,
  SIG_ERR_NULL = 1,       /* a required pointer is NULL                        */
  SIG_ERR_SHAPE = 2,      /* a size is out of range or inconsistent            */
  SIG_ERR_ALIGN = 3,      /* a pointer is not aligned as required              */
  SIG_ERR_WORKSPACE = 4,  /* workspace NULL or smaller than sig_workspace_bytes */
  SIG_ERR_CUDA = 5,       /* the CUDA runtime reported an error                */
  SIG_ERR_TIMEOUT = 6,    /* a bounded device-side wait gave up                */
  SIG_ERR_ARG = 7         /* another argument is out of range (k, n, m, op)    */
} sig_status;

/* Operation codes for sig_workspace_bytes. */
typedef enum {
  SIG_OP_SPARSE_GEMV = 1,  /* sparse_gemv(d_in, d_out)                 */
  SIG_OP_TOPK = 2,         /* sparsify_topk(d = d_in)                  */
  SIG_OP_GATED_MLP = 3,    /* gated_mlp_sparse(d_model = d_in, d_ff = d_out) */
  SIG_OP_NM_GEMM = 4,      /* nm_act_gemm(K = d_in, N = d_out, rows)   */
  SIG_OP_RANK_ADAPTER = 5, /* rank_adapter_sparse(d_in, d_out, rows = r) */
  SIG_OP_SPARSE_GEMV_BATCH = 6, /* sparse_gemv_batch(d_in, d_out, rows = tokens) */
  SIG_OP_SPARSE_GEMV_Q8 = 7,    /* sparse_gemv_q8(d_in, d_out)              */
  SIG_OP_SPARSE_GEMV_F8 = 8,    /* sparse_gemv_f8(d_in, d_out)              */
  SIG_OP_SPARSE_GEMV_Q4 = 9     /* sparse_gemv_q4(d_in, d_out)              */
} sig_op;

/* Largest activation length the fused mask prologue accepts. */
#define SIG_MAX_D_IN 131072
/* Largest length sparsify_topk accepts (its keys live in shared memory). */
#define SIG_MAX_TOPK_D 131072

/* Human-readable name of a status code (static storage, never NULL). */
SIG_API const char* sig_status_string(int status);

/* ABI version of this header; bumps when a signature changes. */
SIG_API int sig_abi_version(void);

/*
 * Bytes of device workspace an operation needs for the given sizes (0 when
 * the operation needs none).  Returns 0 and sets nothing for an unknown op.
 * It holds split-K partial sums and per-tile epoch or arrival counters; the gated MLP also
 * keeps its fp16 hidden vector there when h_out is NULL, and the N:M GEMM its
 * masked activation block.
 */
SIG_API size_t sig_workspace_bytes(int op, int64_t d_in, int64_t d_out, int64_t rows);

/*
 * Zero a workspace before its first use (asynchronously on `stream`).  A
 * workspace then serves any number of calls of ONE operation at ONE shape
 * (the same sizes and, for sparse_gemv_multi, the same d_out list): the fp16
 * GEMVs tag their split-K partial sums with a per-tile epoch that advances
 * with every call, and the other operations leave their counters at zero.
 * Zero it again before using it for another operation or another shape.
 * ws must be 256-byte aligned.
 */
SIG_API int sig_workspace_init(void* ws, size_t ws_bytes, sig_stream_t stream);

/*
 * Threshold mask (TEAL README, Abstract; comparison ">= t" as in RaNA
 * Eqn. 12):  m_i = |x_i| >= t, compared in float32 (exact for fp16 x).
 *   x          [d] fp16, 16-byte aligned.
 *   t          threshold (float).  A NaN in x is never kept.
 *   mask_bits  [ceil(d/32)] uint32 out.
 *   idx        [d] int32 out, nullable: ascending kept indices (first *nnz valid).
 *   nnz        [1] int32 out, nullable: number of kept entries.
 * Errors: SIG_ERR_NULL (x or mask_bits), SIG_ERR_SHAPE (d < 1 or d > SIG_MAX_D_IN),
 *         SIG_ERR_ALIGN (x not 16-byte aligned, or mask_bits, idx or nnz not
 *         4-byte aligned).
 */
SIG_API int sparsify_threshold(const uint16_t* x, int64_t d, float t,
                       uint32_t* mask_bits, int32_t* idx, int32_t* nnz,
                       sig_stream_t stream);

/*
 * Top-k mask (Q-Sparse rebuttal, A1 on MoE): keep the k entries of largest
 * |x|, ties by lower index; exactly k bits are set.  Selection runs on the
 * 15-bit magnitude code of fp16, so no float comparison decides it.
 *   x          [d] fp16, 16-byte aligned.
 *   k          0 <= k <= d.
 *   mask_bits  [ceil(d/32)] uint32 out.   idx [d] int32 out (first k valid).
 *   nnz        [1] int32 out (= k).
 *   ws         sig_workspace_bytes(SIG_OP_TOPK, d, 0, 0) bytes (may be 0 → ws may be NULL).
 * Errors: SIG_ERR_NULL, SIG_ERR_SHAPE (d < 1 or d > SIG_MAX_TOPK_D), SIG_ERR_ARG (k),
 *         SIG_ERR_ALIGN.
 */
SIG_API int sparsify_topk(const uint16_t* x, int64_t d, int64_t k,
                  uint32_t* mask_bits, int32_t* idx, int32_t* nnz,
                  void* ws, size_t ws_bytes, sig_stream_t stream);

/*
 * N:M activation mask (N:M summary, Methodology; Block Q-Sparse in the
 * Q-Sparse rebuttal, A2): for every row of X and every block of m consecutive
 * entries, keep the n of largest |x| (ties by lower index).
 *   X          [rows x d] fp16 row-major, 16-byte aligned; d % 8 == 0 so that
 *              every row starts 16-byte aligned (else SIG_ERR_ALIGN).
 *   n, m       m in {1, 2, 4, 8, 16, 32}, 1 <= n <= m, d % m == 0.
 *   X_masked   [rows x d] fp16 out, 16-byte aligned, nullable: X with dropped
 *              entries set to +0.
 *   mask_bits  [rows x ceil(d/32)] uint32 out, nullable.
 *   packed     sig_nm_packed_bytes(rows, d) bytes out, 16-byte aligned,
 *              nullable: the 2:4 operand of the sparse tensor cores, for
 *              nm_act_gemm_packed.  Only for 2:4 and 1:4 (n:m = 2:4 or 1:4,
 *              else SIG_ERR_ARG), rows % 128 == 0 and d % 128 == 0 (else
 *              SIG_ERR_SHAPE).  1:4 is padded to 2:4: the block's second slot
 *              holds +0 at the smallest position that is not kept.  Layout:
 *                values  [rows x d/2] fp16 at byte 0: for row r and block b
 *                        (entries 4b .. 4b+3), the two slots in ascending
 *                        position order at [r, 2b] and [r, 2b+1];
 *                meta    rows*d/8 bytes at byte rows*d: one 2048-byte tile per
 *                        128 x 128 block (row block R, column block C; tile
 *                        R * (d/128) + C).  Byte 16 L + 4 j + 2 s + i of a tile
 *                        (lane L < 128, group j < 4, s and i < 2) holds the
 *                        blocks of row r = 128 R + L % 8 + 8 s + 16 (L / 16),
 *                        entries 128 C + 32 j + 16 ((L / 8) % 2) + 8 i + 4 k
 *                        for k = 0 (low nibble) and k = 1 (high nibble); a
 *                        block's nibble is p0 | p1 << 2, p0 < p1 the positions
 *                        of its two slots.  This is the order in which a
 *                        128x128b tensor-memory copy hands a 128 x 128 block of
 *                        metadata to the sparse MMA.
 * At least one of X_masked, mask_bits and packed must be non-NULL.  rows == 0
 * is an empty batch: the call returns SIG_OK and touches no pointer.
 * Errors: SIG_ERR_NULL, SIG_ERR_SHAPE (rows < 0, d < 1, d % m), SIG_ERR_ARG (n, m),
 *         SIG_ERR_ALIGN.
 */
SIG_API int sparsify_nm(const uint16_t* X, int64_t rows, int64_t d, int n, int m,
                uint16_t* X_masked, uint32_t* mask_bits, void* packed, sig_stream_t stream);

/* Bytes of sparsify_nm's packed output (rows*d*9/8), or 0 when rows or d is
 * not a positive multiple of 128. */
SIG_API size_t sig_nm_packed_bytes(int64_t rows, int64_t d);

/*
 * Sparse-input GEMV y = W (m . x) (RaNA rebuttal, Q5.1; Q-Sparse A3):
 *   y_j = sum over kept i of WT[i, j] * x_i, accumulated in float32 and
 *   rounded once to fp16.  Only the kept rows of WT are read.
 * Mask source:
 *   idx == NULL: fused threshold |x_i| >= t, computed inside the same launch.
 *   idx != NULL: the rows idx[0 .. *nnz) from a sparsify_* call; t is ignored.
 *                Entries outside [0, d_in) are skipped; *nnz is clamped to [0, d_in].
 *   WT   [d_in x d_out] fp16 row-major, 16-byte aligned, d_out % 8 == 0.
 *   x    [d_in] fp16, 16-byte aligned.       y [d_out] fp16 out, 16-byte aligned.
 *   ws   sig_workspace_bytes(SIG_OP_SPARSE_GEMV, d_in, d_out, 0) bytes, 256-byte
 *        aligned, zeroed by sig_workspace_init (or allocated zeroed) before
 *        its first use and serving this shape only (see sig_workspace_init);
 *        it holds one epoch word per 256-column tile and the split-K slices'
 *        partial sums as 64-bit {float32 value, epoch tag} words.  When the
 *        size is 0 (one slice per tile, which the planner chooses above 296
 *        tiles, i.e. d_out > 75776) ws may be NULL.
 * The split-K finish: every slice stores its partial sums and exits; the
 * tile's last two slices each finish one 128-column half: they wait (bounded,
 * ~2 s; on expiry bit 1 of the device error word is set, see
 * sig_take_device_error) until every slice's word carries this call's tag,
 * then add them in slice order.
 * The result is bit-identical from run to run (fixed-order split-K reduction;
 * no floating-point atomics).  An empty mask writes y = 0.
 * Errors: SIG_ERR_NULL, SIG_ERR_SHAPE (d_in < 1, d_in > SIG_MAX_D_IN, d_out < 8,
 *         d_out % 8), SIG_ERR_ALIGN, SIG_ERR_WORKSPACE, SIG_ERR_CUDA.
 */
SIG_API int sparse_gemv(const uint16_t* WT, int64_t d_in, int64_t d_out,
                const uint16_t* x, float t, const int32_t* idx, const int32_t* nnz,
                uint16_t* y, void* ws, size_t ws_bytes, sig_stream_t stream);

/*
 * Sparse-input GEMV for several weights that read the same input, in one
 * launch: y_p = W_p (m . x) for p < n_mat, with ONE mask m.  In a transformer
 * block the query, key and value projections read the same hidden state, and
 * so do the gate and up projections of the MLP; TEAL thresholds that shared
 * hidden state once (TEAL README, Abstract), and the product is that of
 * sparse_gemv for each weight (RaNA rebuttal, Q5.1).  The mask is computed
 * once per CTA for all the weights and their column tiles share the grid.
 *   n_mat    1 .. 4.
 *   WT, y    HOST arrays of n_mat DEVICE pointers: WT[p] [d_in x d_out[p]]
 *            fp16 row-major, y[p] [d_out[p]] fp16 out; all 16-byte aligned.
 *   d_out    HOST array of n_mat sizes, each a multiple of 8.
 *   x, t, idx, nnz   as sparse_gemv (one mask for all the weights).
 *   ws       sig_workspace_bytes_multi(n_mat, d_out, d_in) bytes, 256-byte
 *            aligned, zeroed before its first use and serving these shapes only
 *            (see sig_workspace_init); it may be NULL when that size is 0.
 * Each y[p] meets the tolerance of sparse_gemv and is bit-identical from run
 * to run.  It can differ in the last bits from a separate sparse_gemv call on
 * W_p, because the grid, and so the split-K order, is planned for all the
 * weights together; with n_mat == 1 it is that call.
 * Errors: SIG_ERR_NULL, SIG_ERR_ARG (n_mat), SIG_ERR_SHAPE, SIG_ERR_ALIGN,
 *         SIG_ERR_WORKSPACE, SIG_ERR_CUDA.
 */
SIG_API int sparse_gemv_multi(int n_mat, const uint16_t* const* WT, const int64_t* d_out,
                              int64_t d_in, const uint16_t* x, float t,
                              const int32_t* idx, const int32_t* nnz,
                              uint16_t* const* y, void* ws, size_t ws_bytes,
                              sig_stream_t stream);

/* Workspace bytes of sparse_gemv_multi (0 for invalid arguments or none needed). */
SIG_API size_t sig_workspace_bytes_multi(int n_mat, const int64_t* d_out, int64_t d_in);

/*
 * Gated MLP with the RaNA neuron masker (RaNA rebuttal, Q3, Eqn. 12):
 *   g = GateProj(x), u = UpProj(x)       (dense GEMVs, float32 accumulation)
 *   h = fp16(SiLU(g) * u)                (SiLU(z) = z / (1 + exp(-z)), float32)
 *   m_i = float32(|h_i|) * down_norms[i] >= t      (one float32 multiply)
 *   y = W_down (m . h)                   (sparse GEMV as in sparse_gemv)
 *   x        [d_model] fp16.   WgT, WuT [d_model x d_ff] fp16.   WdT [d_ff x d_model] fp16.
 *   down_norms [d_ff] float32: ||row i of WdT||_2 (see sig_row_norms).
 *   y        [d_model] fp16 out.  h_out [d_ff] fp16 out, nullable.
 *   mask_out [ceil(d_ff/32)] uint32 out, nullable.
 *   ws       sig_workspace_bytes(SIG_OP_GATED_MLP, d_model, d_ff, 0) bytes.
 * d_model % 8 == 0, d_ff % 8 == 0, d_model and d_ff <= SIG_MAX_D_IN.
 * Errors: as sparse_gemv.
 */
SIG_API int gated_mlp_sparse(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                     const uint16_t* WdT, const float* down_norms,
                     int64_t d_model, int64_t d_ff, float t,
                     uint16_t* y, uint16_t* h_out, uint32_t* mask_out,
                     void* ws, size_t ws_bytes, sig_stream_t stream);

/*
 * A few tokens, each with its own threshold mask, through one weight:
 *   y_b = W (m_b . x_b),  m_b,i = |x_b,i| >= t,  b < B.
 * The product is the single-token one of sparse_gemv (RaNA rebuttal, Q5.1);
 * batches with inconsistent masks are the open case of the same rebuttal (Q6).
 * One launch reads every weight row that any token keeps (the union of the
 * masks) once and applies each token's own mask to it; same tolerance and
 * determinism as sparse_gemv for every token.
 *   WT [d_in x d_out] fp16.  X [B x d_in] fp16, row-major.  Y [B x d_out] fp16 out.
 *   ws sig_workspace_bytes(SIG_OP_SPARSE_GEMV_BATCH, d_in, d_out, B) bytes
 *      (0 means none is needed and ws may be NULL), 256-byte aligned, zeroed
 *      once before first use; every call leaves it ready for the next.
 * 1 <= B <= SIG_MAX_BATCH (16); d_in % 8 == 0 (whole 16-byte groups per token row),
 * d_in <= SIG_MAX_D_IN; d_out % 8 == 0.
 * Errors: SIG_ERR_NULL, SIG_ERR_ARG (B), SIG_ERR_SHAPE, SIG_ERR_ALIGN,
 *         SIG_ERR_WORKSPACE, SIG_ERR_CUDA.
 */
#define SIG_MAX_BATCH 16
SIG_API int sparse_gemv_batch(const uint16_t* WT, int64_t d_in, int64_t d_out,
                              const uint16_t* X, int64_t B, float t, uint16_t* Y,
                              void* ws, size_t ws_bytes, sig_stream_t stream);

/*
 * Weight-quantised sparse GEMV: y = W (m . x), m_i = |x_i| >= t, with the weight
 * held as int8 q and one float32 scale per output column, W[j, i] = s_j q[i, j]:
 *   y_j = fp16( s_j * sum_{i: m_i} q[i, j] x_i )      (float32 accumulation)
 * The pages leave quantised sparse kernels open (TEAL README, Limitations) and
 * call quantisation orthogonal to activation sparsity (Q-Sparse rebuttal, A1 on
 * batched inference); a kept input costs d_out bytes instead of 2 d_out.
 *   QT [d_in x d_out] int8 (transposed: row i multiplies x_i), 16-byte aligned.
 *   scale [d_out] float32.  x [d_in] fp16.  y [d_out] fp16 out.
 *   ws sig_workspace_bytes(SIG_OP_SPARSE_GEMV_Q8, d_in, d_out, 0) bytes
 *      (0 means none is needed), 256-byte aligned, zeroed before first use and
 *      serving this shape only (see sig_workspace_init).
 * d_out % 8 == 0 (whole 8-byte lanes of eight weights), d_in <= SIG_MAX_D_IN.
 * Errors: SIG_ERR_NULL, SIG_ERR_SHAPE, SIG_ERR_ALIGN, SIG_ERR_WORKSPACE, SIG_ERR_CUDA.
 */
SIG_API int sparse_gemv_q8(const int8_t* QT, const float* scale, int64_t d_in, int64_t d_out,
                           const uint16_t* x, float t, uint16_t* y, void* ws, size_t ws_bytes,
                           sig_stream_t stream);

/*
 * The same product with fp8 weights: QT holds OCP E4M3 codes (sign bit 7,
 * exponent bits 6..3 with bias 7, mantissa bits 2..0; no infinities,
 * S.1111.111 is NaN), W[j, i] = s_j e4m3(QT[i, j]):
 *   y_j = fp16( s_j * sum_{i: m_i} e4m3(QT[i, j]) x_i )   (float32 accumulation)
 * Every e4m3 value is exact in fp16, so the hardware converts two codes to an
 * fp16 pair in one instruction.  Arguments, workspace
 * (sig_workspace_bytes(SIG_OP_SPARSE_GEMV_F8, d_in, d_out, 0)), shape rules
 * and errors as sparse_gemv_q8.
 */
SIG_API int sparse_gemv_f8(const uint8_t* QT, const float* scale, int64_t d_in, int64_t d_out,
                           const uint16_t* x, float t, uint16_t* y, void* ws, size_t ws_bytes,
                           sig_stream_t stream);

/*
 * The same product with int4 weights, two to a byte: QT4 is d_in x d_out / 2
 * bytes, row-major; byte b of row i holds q[i, 2b] in bits 0..3 and
 * q[i, 2b + 1] in bits 4..7, each a two's-complement value in [-8, 7];
 * W[j, i] = s_j q[i, j]:
 *   y_j = fp16( s_j * sum_{i: m_i} q[i, j] x_i )      (float32 accumulation)
 * A kept input costs d_out / 2 bytes.  Workspace
 * (sig_workspace_bytes(SIG_OP_SPARSE_GEMV_Q4, d_in, d_out, 0)), shape rules
 * (d_out % 8 == 0: whole 4-byte lanes of eight weights) and errors as
 * sparse_gemv_q8; QT4 16-byte aligned.
 */
SIG_API int sparse_gemv_q4(const uint8_t* QT4, const float* scale, int64_t d_in, int64_t d_out,
                           const uint16_t* x, float t, uint16_t* y, void* ws, size_t ws_bytes,
                           sig_stream_t stream);

/*
 * RaNA linear-layer rank adapter (RaNA rebuttal, Q5.1: Linear(x) ~ A (m(x) . Bx),
 * whose masked product skips the columns of A with a zero mask entry; Q4: the
 * masker squares Bx element-wise against a threshold (eqn. 9); Q2 to the fourth
 * reviewer: one plain GEMV for v = Bx and one masked GEMV):
 *   v = fp16(B x)                        (dense GEMV, float32 accumulation)
 *   m_i = float32(v_i) * float32(v_i) >= t          (one float32 multiply)
 *   y = A (m . v)                        (sparse GEMV as in sparse_gemv)
 *   x [d_in] fp16.  BT [d_in x r] fp16 (B transposed: row i multiplies x_i).
 *   AT [r x d_out] fp16 (A transposed: row i multiplies v_i).
 *   y [d_out] fp16 out.  v_out [r] fp16 out, nullable.
 *   mask_out [ceil(r/32)] uint32 out, nullable.
 *   ws sig_workspace_bytes(SIG_OP_RANK_ADAPTER, d_in, d_out, r) bytes.
 * r % 8 == 0 and d_out % 8 == 0 (they are output widths); d_in and r each
 * in [1, SIG_MAX_D_IN].  Two launches on `stream`; the caller owns every buffer.
 * Errors: as sparse_gemv.
 */
SIG_API int rank_adapter_sparse(const uint16_t* x, const uint16_t* BT, const uint16_t* AT,
                                int64_t d_in, int64_t r, int64_t d_out, float t,
                                uint16_t* y, uint16_t* v_out, uint32_t* mask_out,
                                void* ws, size_t ws_bytes, sig_stream_t stream);

/*
 * N:M activation mask with the selection and error-mitigation variants of
 * "Motivating Next-Gen Accelerators with Flexible (N:M) Activation Sparsity
 * ..." (summary, Methodology: criteria ACT and WT, mitigation PTS and VAR),
 * per row r of X:
 *   x' = fp16(float32(x) - shift[r])            (PTS; shift NULL: x' = x)
 *   score_i = |x'_i|                            (ACT, norms NULL)
 *           = float32(|x'_i|) * norms[i]        (WT: one float32 multiply;
 *                                                norms = ||W_i||, see sig_row_norms)
 *   m: in each block of m, the n of largest score (lower index first among
 *      equals, NaN last), as sparsify_nm
 *   X_masked = fp16(gamma_r * m . x')           (VAR: gamma_r = sqrt(sum x'^2 /
 *                                                sum (m x')^2), float32, 1 when
 *                                                either sum is 0; var = 0: gamma 1)
 *   X [rows x d] fp16, row-major, 16-byte aligned.  shift [rows] float32, nullable.
 *   norms [d] float32, 16-byte aligned, nullable.
 *   X_masked [rows x d] fp16 out, 16-byte aligned (required).
 *   mask_bits [rows x ceil(d/32)] uint32 out, nullable.  gamma_out [rows] float32 out, nullable.
 * 1 <= n <= m, m in {1, 2, 4, 8, 16, 32}, d % m == 0, d % 8 == 0.
 * Errors: SIG_ERR_ARG (n, m), SIG_ERR_SHAPE, SIG_ERR_NULL, SIG_ERR_ALIGN, SIG_ERR_CUDA.
 */
SIG_API int sparsify_nm_ex(const uint16_t* X, int64_t rows, int64_t d, int n, int m,
                           const float* shift, const float* norms, int var,
                           uint16_t* X_masked, uint32_t* mask_bits, float* gamma_out,
                           sig_stream_t stream);

/*
 * N:M activation GEMM with the variants of sparsify_nm_ex:
 *   Y = X_masked WT + shift col_sums^T       (the shift added back: col_sums[j] =
 *                                             sum_i WT[i, j], see sig_col_sums)
 * on the tensor cores as nm_act_gemm.  shift NULL: no added term (col_sums may
 * be NULL); otherwise col_sums [N] float32 is required.  Shapes, workspace
 * (sig_workspace_bytes(SIG_OP_NM_GEMM, K, N, rows)) and errors as nm_act_gemm.
 */
SIG_API int nm_act_gemm_ex(const uint16_t* X, int64_t rows, int64_t K, const uint16_t* WT,
                           int64_t N, int n, int m, const float* shift, const float* norms,
                           int var, const float* col_sums, uint16_t* Y, void* ws,
                           size_t ws_bytes, sig_stream_t stream);

/*
 * Column sums of a row-major fp16 matrix, accumulated in float64 and rounded
 * once to float32: for WT, r_j = sum_i W[j, i], the vector a per-token shift
 * mu brings back as mu * r (x W = (x - mu) W + mu r).
 *   WT [rows x cols] fp16, rows >= 1, 1 <= cols <= 2^30.  sums [cols] float32 out.
 * Errors: SIG_ERR_NULL, SIG_ERR_SHAPE, SIG_ERR_ALIGN.
 */
SIG_API int sig_col_sums(const uint16_t* WT, int64_t rows, int64_t cols, float* sums,
                         sig_stream_t stream);

/*
 * Gated MLP with TEAL's magnitude threshold on the input of every product
 * (TEAL README, Abstract: the hidden states that feed each matrix
 * multiplication):
 *   m_x = |x_i| >= t_x;  g = GateProj(m_x . x), u = UpProj(m_x . x)
 *                                        (one fused sparse GEMV for both,
 *                                         float32 accumulation)
 *   h = fp16(SiLU(g) * u)                (SiLU(z) = z / (1 + exp(-z)), float32)
 *   m_h = |h_i| >= t_h;  y = W_down (m_h . h)        (sparse GEMV as sparse_gemv)
 *   x [d_model] fp16.  WgT, WuT [d_model x d_ff] fp16.  WdT [d_ff x d_model] fp16.
 *   y [d_model] fp16 out.  h_out [d_ff] fp16 out, nullable.
 *   mask_out [ceil(d_ff/32)] uint32 out (m_h), nullable.
 *   ws sig_workspace_bytes(SIG_OP_GATED_MLP, d_model, d_ff, 0) bytes.
 * d_model % 8 == 0, d_ff % 8 == 0, d_model and d_ff <= SIG_MAX_D_IN.
 * Errors: as sparse_gemv.
 */
SIG_API int teal_mlp_sparse(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                            const uint16_t* WdT, int64_t d_model, int64_t d_ff, float t_x,
                            float t_h, uint16_t* y, uint16_t* h_out, uint32_t* mask_out,
                            void* ws, size_t ws_bytes, sig_stream_t stream);

/*
 * l2 norm of every row of a row-major fp16 matrix, accumulated in float64 and
 * rounded once to float32.  For WdT it yields the ||W^down_i|| of RaNA Eqn. 12.
 *   WT [rows x cols] fp16 (16-byte aligned, cols % 8 == 0).  norms [rows] float32 out.
 * Errors: SIG_ERR_NULL, SIG_ERR_SHAPE, SIG_ERR_ALIGN.
 */
SIG_API int sig_row_norms(const uint16_t* WT, int64_t rows, int64_t cols, float* norms,
                  sig_stream_t stream);

/*
 * Batched N:M activation GEMM (Block Q-Sparse, Q-Sparse rebuttal A2):
 *   Y = (M . X) WT, M the per-row n:m mask of X (as sparsify_nm), float32
 *   accumulation on the tensor cores, Y rounded once to fp16.  When n == m
 *   the GEMM runs on X directly.  For 2:4 and 1:4 with K % 128 == 0, X is
 *   packed (as sparsify_nm's packed output) and the product runs on the
 *   sparse tensor cores (as nm_act_gemm_packed); other patterns run the dense
 *   tensor cores on the masked X.
 *   X  [rows x K] fp16 row-major.   WT [K x N] fp16 row-major.   Y [rows x N] fp16 out.
 *   All three 16-byte aligned (WT and X are read by TMA).
 *   rows % 128 == 0, K % 64 == 0, N % 128 == 0, rows <= 2^24, K and N <= 2^20;
 *   m in {1,2,4,8,16,32}, 1 <= n <= m, K % m == 0.
 *   ws sig_workspace_bytes(SIG_OP_NM_GEMM, K, N, rows) bytes (the masked or
 *      packed X; not touched when n == m, so it may be NULL then).
 * Errors: SIG_ERR_NULL, SIG_ERR_SHAPE, SIG_ERR_ARG, SIG_ERR_ALIGN, SIG_ERR_WORKSPACE,
 *         SIG_ERR_CUDA.
 */
SIG_API int nm_act_gemm(const uint16_t* X, int64_t rows, int64_t K, const uint16_t* WT,
                int64_t N, int n, int m, uint16_t* Y, void* ws, size_t ws_bytes,
                sig_stream_t stream);

/*
 * The product of nm_act_gemm on an operand that sparsify_nm has already
 * packed (2:4, or 1:4 padded to 2:4): Y = A WT, A the rows x K activation
 * block the packed values and metadata describe, on the sparse tensor cores
 * (tcgen05.mma.sp, kind::f16: half the A bytes, each MMA covers 32 logical K).
 * Float32 accumulation, Y rounded once to fp16.
 *   packed  sig_nm_packed_bytes(rows, K) bytes, 16-byte aligned (the layout
 *           of sparsify_nm).   WT [K x N] fp16.   Y [rows x N] fp16 out.
 *   rows % 128 == 0, K % 128 == 0, N % 128 == 0, rows <= 2^24, K and N <= 2^20.
 * Errors: SIG_ERR_NULL, SIG_ERR_SHAPE, SIG_ERR_ALIGN, SIG_ERR_CUDA.
 */
SIG_API int nm_act_gemm_packed(const void* packed, int64_t rows, int64_t K, const uint16_t* WT,
                               int64_t N, uint16_t* Y, sig_stream_t stream);

/*
 * gated_mlp_sparse without a workspace argument, for callers that cannot
 * allocate device memory where they run this layer: a plugin inside a host
 * program whose own pool owns all device memory, a serving loop whose memory
 * budget is fixed at start-up, or plain C code with no allocator.  The pages
 * have no counterpart to this entry point; it computes exactly what
 * gated_mlp_sparse computes, with the same arguments minus ws / ws_bytes.
 * Its scratch (the split-K partial sums of the two products with their
 * epoch words, and the fp16 hidden vector h when h_out is NULL) lives in one
 * device array of SIG_NOALLOC_SCRATCH_BYTES (4 MiB) inside the library,
 * which every GPU that loads the library holds until the process exits.  It
 * allocates nothing and calls no allocating routine.
 *   - A call whose scratch (sig_workspace_bytes(SIG_OP_GATED_MLP, d_model,
 *     d_ff, 0)) would exceed SIG_NOALLOC_SCRATCH_BYTES returns SIG_ERR_SHAPE
 *     with nothing enqueued.  Every shape gated_mlp_sparse accepts
 *     (d_model, d_ff <= SIG_MAX_D_IN) needs at most 3703 KiB, so it fits;
 *     larger sizes are rejected with SIG_ERR_SHAPE like everywhere else.
 *   - Every call shares the array and finds the previous call's contents in
 *     it; the call clears what must start at zero (a memset of the partial-sum
 *     area, about 3.3 MB at Llama-2-7B MLP shapes).  Calls that overlap on the
 *     GPU (other streams, other host threads) race; serialise them.
 *   - The first call on each device, with that device current, looks up the
 *     array's device address (cudaGetSymbolAddress) and caches it; make that
 *     first call before any stream capture.  The cached address belongs to
 *     the device's primary context as it was then: cudaDeviceReset (or
 *     anything else that destroys that context) leaves it stale, so do not
 *     call this entry point on a device after resetting it in the same
 *     process.
 * Errors: as gated_mlp_sparse, except SIG_ERR_WORKSPACE (none is taken).
 */
#define SIG_NOALLOC_SCRATCH_BYTES (4u << 20)
SIG_API int gated_mlp_sparse_noalloc(const uint16_t* x, const uint16_t* WgT, const uint16_t* WuT,
                                     const uint16_t* WdT, const float* down_norms,
                                     int64_t d_model, int64_t d_ff, float t,
                                     uint16_t* y, uint16_t* h_out, uint32_t* mask_out,
                                     sig_stream_t stream);

/*
 * Read and clear the library's device error words (no counterpart on the
 * pages; they report the bounded waits: bit 0, a tensor-core GEMM pipeline
 * wait; bit 1, the split-K finish of an fp16 GEMV).  Synchronises `stream`.
 * *code receives 0 when no kernel gave up on a wait, else the bits set; the
 * call then returns SIG_ERR_TIMEOUT.
 * Errors: SIG_ERR_NULL (code), SIG_ERR_CUDA.
 */
SIG_API int sig_take_device_error(unsigned* code, sig_stream_t stream);

/*
 * Set the limit, in SM clock cycles, after which a pipeline wait of the
 * tensor-core GEMMs (nm_act_gemm, nm_act_gemm_ex, nm_act_gemm_packed) gives
 * up, on the current device; cycles <= 0 restores the default (4e9, about 2 s
 * at 1.9 GHz).  No counterpart on the pages: it lets a caller (or a test)
 * shorten the failure-detection window.  A kernel that gives up records a bit
 * in the device error word (sig_take_device_error), lets the copies it has
 * issued land (waiting up to the default limit for each), frees its tensor
 * memory and returns; its output is not valid.  Synchronous with respect to
 * the host (cudaMemcpyToSymbol); do not call it during stream capture.
 * Errors: SIG_ERR_CUDA.
 */
SIG_API int sig_set_wait_limit(long long cycles);

#ifdef __cplusplus
}
#endif

#endif /* SIG_H */
