// Split-K sparse-input GEMV y = W (m . x) with the mask step fused ahead of it,
// for fp16 weights and for 8-bit (int8 or fp8 e4m3) or int4 weights with one
// float32 scale per output column.  The pages leave quantised sparse kernels
// open (TEAL README, Limitations) and call weight quantisation orthogonal to
// activation sparsity (Q-Sparse rebuttal, A1 on batched inference): an 8-bit
// kept row moves d_out bytes instead of 2 d_out, an int4 row d_out / 2.
//
// The product reads only the weight rows of the kept inputs ("Adaptive Rank
// Allocation ... RaNA Adapters", Q5.1: the columns of A that meet a zero mask
// entry are skipped).  WT is stored transposed (d_in x d_out, row-major), so a
// kept input i costs one contiguous row of 2*d_out bytes.
//
// Launch shape: C x S CTAs of 256 threads, about four per SM on every SM.  A
// CTA owns a 256-output column tile (one warp spans it with 16-byte lanes) and
// one slice s of the kept rows.  Under a threshold the slices interleave by
// 8-input groups (slice s owns groups s, s+S, s+2S, ...), so a CTA needs only
// its own 1/S of the activation to know its rows; an index list is cut into S
// equal runs.  Up to four weights that read the same input (q, k, v; gate, up)
// share one launch and one mask: their column tiles are laid end to end.  One
// launch does everything:
//   1. the CTA loads its groups of the activation (from L2) and takes their
//      mask bits with fp16 SIMD compares against the threshold rounded up to
//      fp16 (exact for fp16 inputs).  A slice of at most 256 groups (every
//      Llama-2-7B and 70B launch) gives one group to each thread: one
//      block-wide exclusive scan of the popcounts gives each thread the rank
//      of its first kept row, and the thread places its rows itself.  Wider
//      slices keep mask words in shared memory, prefix-sum their popcounts,
//      and the warps place the rows one word per warp and one bit per lane
//      (rank = word prefix + popcount of the lower bits);
//   2. 8 warps stream the slice's rows of the tile, 8 rows in flight per warp:
//      16-byte non-allocating loads with an L2 evict-first policy, the
//      activation value riding along as a broadcast load, fp32 FMA (8-bit
//      weights: 12 rows in flight, 8-byte lanes of eight weights, each made an
//      exact float value in registers (int8: sign extension and an int-to-
//      float conversion; e4m3: the hardware conversion to fp16 pairs, then
//      packed float32 FMAs); int4 weights: 8 rows, 4-byte lanes of eight
//      nibbles, sign-extended by shifts; the column scale multiplies the
//      finished sum);
//   3. the warps' sums meet in shared memory (fixed order) and the CTA
//      stores one partial per column as a 64-bit word {value, tag} (tag = the
//      tile's epoch + 1, read from the workspace at the start) with a relaxed
//      store, and exits.  The tile's last two slices, the CTAs dispatched
//      last, instead finish one 128-column half each: two threads per column
//      poll the partial words of half the slices each, in batches, until
//      every tag is current, add them in slice order, and the two halves are
//      added in a fixed order and stored as fp16.  A finisher whose half holds
//      a column then advances the tile's epoch (it has seen every slice's
//      word, so every slice has read the epoch).  The value and its tag
//      travel in one single-copy-atomic 64-bit word, so no fence and no atomic
//      stand between the last partial store and the sum.  The wait is bounded
//      (~2 s of clock cycles; on expiry the kernel sets a bit in the device
//      error word and stores what it has).
// No floating-point atomics; y is bit-identical from run to run.
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace sig {

// Device error word of the split-K finish (bit 1: a tile's finishing slice gave up
// waiting for the other slices' partial sums); read with the GEMM's word.
__device__ unsigned g_gemv_error = 0u;

namespace {

constexpr int kThreads = kGemvThreads;        // 256
constexpr long long kFinishSpinCycles = 4000000000ll;   // ~2 s at 1.9 GHz
constexpr int kWarps = kThreads / 32;         // 8
constexpr int kTile = kGemvTile;              // 256 outputs per CTA
constexpr int kMaxS = kGemvMaxSplits;         // 64

struct KArgs {
  // weights that share the input and its mask: column tiles [tile0[p],
  // tile0[p+1]) belong to weight p, whose columns start at col0[p] in the
  // concatenated partial-sum space of d_out_total columns
  const uint16_t* WT[kGemvMaxMat];
  uint16_t* y[kGemvMaxMat];
  int d_out[kGemvMaxMat];
  int tile0[kGemvMaxMat + 1];
  int col0[kGemvMaxMat];
  int n_mat, d_out_total;
  const uint16_t* WT2;    // dual partner of WT[0] (gate/up)
  const uint16_t* x;
  const float* scale;
  const float* col_scale; // 8-bit weights: one float32 per output column
  const uint8_t* QT;      // 8-bit weights (d_in x d_out bytes), in place of WT[0]
  const int32_t* idx;
  const int32_t* nnz;
  float t;
  int d_in, S, chunk;
  uint32_t words_bytes;   // shared bytes of the mask words (and again of their prefixes)
  uint32_t union_bytes;   // shared bytes of words + prefixes / the warp-sum buffer
  uint32_t* mask_out;
  unsigned* epochs;       // [C]: calls completed on each tile
  unsigned long long* slots;   // [S][d_out_total] {value, tag} (then again for the second product)
};

// Mask bits of the 8-input groups this slice owns.  Group g covers inputs
// 8g .. 8g+7; slice s owns groups s, s + S, s + 2S, ... (K of them), four to
// a local word: bit 8q + b of local word lw is input 8 (s + (4 lw + q) S) + b.
template <int MODE>
__device__ __forceinline__ void build_local_words(const KArgs& a, int s, int K, int nlw,
                                                  uint32_t* words) {
  const int d_in = a.d_in, S = a.S;
  const float t = a.t;
  const __half2 th2 = thresh_half2(t);
  for (int lw = threadIdx.x; lw < nlw; lw += kThreads) {
    uint4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {     // the word's four groups in flight together
      const int k = lw * 4 + q;
      const int e0 = (s + k * S) * 8;
      v[q] = k < K && e0 + 8 <= d_in ? __ldg(reinterpret_cast<const uint4*>(a.x + e0))
                                     : make_uint4(0, 0, 0, 0);
    }
    uint32_t w = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int k = lw * 4 + q;
      if (k >= K) break;
      const int e0 = (s + k * S) * 8;
      uint32_t b = 0;
      if (MODE == MASK_THRESH && e0 + 8 <= d_in) {
        b = thresh_bits8(v[q], th2);
      } else {
        for (int j = 0; j < 8; ++j) {
          const int i = e0 + j;
          if (i >= d_in) break;
          const float m = fabsf(h2f(e0 + 8 <= d_in ? lane_half(v[q], j) : a.x[i]));
          const bool keep = MODE == MASK_THRESH_SCALED ? __fmul_rn(m, __ldg(a.scale + i)) >= t
                            : MODE == MASK_SQUARE      ? __fmul_rn(m, m) >= t
                                                       : m >= t;
          b |= (keep ? 1u : 0u) << j;
        }
      }
      w |= b << (8 * q);
    }
    words[lw] = w;
  }
}

// Mask bits of one 8-input group starting at input e0 (inputs past d_in are
// not kept).
template <int MODE>
__device__ __forceinline__ uint32_t group_bits(const KArgs& a, int e0, __half2 th2) {
  const int d_in = a.d_in;
  const float t = a.t;
  if (e0 + 8 <= d_in) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.x + e0));
    if (MODE == MASK_THRESH) return thresh_bits8(v, th2);
    uint32_t b = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float m = fabsf(h2f(lane_half(v, j)));
      const bool keep = MODE == MASK_THRESH_SCALED ? __fmul_rn(m, __ldg(a.scale + e0 + j)) >= t
                        : MODE == MASK_SQUARE      ? __fmul_rn(m, m) >= t
                                                   : m >= t;
      b |= (keep ? 1u : 0u) << j;
    }
    return b;
  }
  uint32_t b = 0;
  for (int j = 0; j < 8 && e0 + j < d_in; ++j) {
    const float m = fabsf(h2f(a.x[e0 + j]));
    const bool keep = MODE == MASK_THRESH_SCALED ? __fmul_rn(m, __ldg(a.scale + e0 + j)) >= t
                      : MODE == MASK_SQUARE      ? __fmul_rn(m, m) >= t
                                                 : m >= t;
    b |= (keep ? 1u : 0u) << j;
  }
  return b;
}

template <int MODE, bool DUAL, int EPI, bool MULTI>
__global__ void __launch_bounds__(kThreads, 4)
sgemv_kernel(const __grid_constant__ KArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int warp_tot[kWarps];
  __shared__ unsigned s_tag;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cg = blockIdx.x, s = blockIdx.y;   // global column tile, slice
  const int d_in = a.d_in, S = a.S;

  uint32_t* words = reinterpret_cast<uint32_t*>(smem);
  int* wpre = reinterpret_cast<int*>(smem + a.words_bytes);
  int* sidx = reinterpret_cast<int*>(smem + a.union_bytes);

  pdl_trigger();
  pdl_wait();
  // tag of this call's partial sums: the tile's epoch + 1 (the tile's finishing
  // slices advance the epoch only after every slice of the tile has read it
  // and stored its partials).  The word was written by an earlier grid that
  // has completed, so a plain load suffices; it is issued now and published
  // to shared memory only after the prologue, so that it does not delay
  // thread 0's own activation load.
  const unsigned epoch0 = (tid == 0 && S > 1) ? __ldcg(a.epochs + cg) : 0u;

  // ---- 1. this CTA's rows [lo, hi) of its kept-row list -----------------
  // threshold modes: the kept inputs of the slice's own 8-input groups, in
  // ascending order; index and dense modes: the s-th of S equal slices of the
  // index list / of all rows
  int lo = 0, hi = 0, nwords = 0, K = 0;
  bool placed = false;   // the kept-row list is already in sidx (one chunk)
  if (MODE == MASK_THRESH || MODE == MASK_THRESH_SCALED || MODE == MASK_SQUARE) {
    const int ngroups = (d_in + 7) >> 3;
    K = s < ngroups ? (ngroups - 1 - s) / S + 1 : 0;
    if (K <= kThreads) {
      // one group per thread: its 8 mask bits from one 16-byte load, one
      // block-wide exclusive scan of the popcounts (ascending group order is
      // ascending input order), then the thread places its own kept rows
      const int e0 = (s + tid * S) * 8;
      const uint32_t b = tid < K ? group_bits<MODE>(a, e0, thresh_half2(a.t)) : 0u;
      const int cnt = __popc(b);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += n;
      }
      if (lane == 31) warp_tot[warp] = incl;
      __syncthreads();
      int before = 0, total = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const int v = warp_tot[w];
        before += w < warp ? v : 0;
        total += v;
      }
      int r = before + incl - cnt;
      for (uint32_t m = b; m != 0u; m &= m - 1u) sidx[r++] = e0 + (__ffs(m) - 1);
      if (a.mask_out != nullptr && cg == 0) {
        uint8_t* mb = reinterpret_cast<uint8_t*>(a.mask_out);
        if (tid < K) mb[s + tid * S] = (uint8_t)b;
        if (s == 0 && tid < 4 * ((d_in + 31) >> 5) - ngroups) mb[ngroups + tid] = 0;
      }
      lo = 0;
      hi = total;
      placed = true;
      __syncthreads();
    } else {
      nwords = (K + 3) >> 2;
      build_local_words<MODE>(a, s, K, nwords, words);
      __syncthreads();
      // exclusive prefix of the words' popcounts, thread-contiguous word ranges
      const int per = (nwords + kThreads - 1) / kThreads;
      const int w0 = min(nwords, tid * per), w1 = min(nwords, w0 + per);
      int cnt = 0;
      for (int w = w0; w < w1; ++w) cnt += __popc(words[w]);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += n;
      }
      if (lane == 31) warp_tot[warp] = incl;
      __syncthreads();
      int before = 0, total = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const int v = warp_tot[w];
        before += w < warp ? v : 0;
        total += v;
      }
      int r = before + incl - cnt;
      for (int w = w0; w < w1; ++w) {            // first rank held by each word
        wpre[w] = r;
        r += __popc(words[w]);
      }
      lo = 0;
      hi = total;
      if (a.mask_out != nullptr && cg == 0) {
        // byte g of the mask words holds group g's bits; the slice writes its
        // own groups, slice 0 also the padding bytes of the last word
        uint8_t* mb = reinterpret_cast<uint8_t*>(a.mask_out);
        for (int k = tid; k < K; k += kThreads) mb[s + k * S] = (uint8_t)(words[k >> 2] >> (8 * (k & 3)));
        if (s == 0 && tid < 4 * ((d_in + 31) >> 5) - ngroups) mb[ngroups + tid] = 0;
      }
      __syncthreads();
    }
  } else if (MODE == MASK_IDX) {
    const int total = min(max(__ldg(a.nnz), 0), d_in);
    lo = (int)(((long long)s * total) / S);
    hi = (int)(((long long)(s + 1) * total) / S);
  } else {  // MASK_DENSE
    lo = (int)(((long long)s * d_in) / S);
    hi = (int)(((long long)(s + 1) * d_in) / S);
  }
  const int n_rows = hi - lo;
  if (tid == 0) s_tag = epoch0 + 1u;   // read after the barriers that follow

  // ---- 2. stream the slice's rows of this column tile ------------------
  // the weight this tile belongs to (static indices only: the arguments stay
  // in the parameter bank)
  const uint16_t* wsel = a.WT[0];
  int d_out = a.d_out[0], t_first = 0;
  if (MULTI) {
#pragma unroll
    for (int i = 1; i < kGemvMaxMat; ++i)
      if (i < a.n_mat && cg >= a.tile0[i]) { wsel = a.WT[i]; d_out = a.d_out[i]; t_first = a.tile0[i]; }
  }
  const int col = (cg - t_first) * kTile + lane * 8;
  const bool col_ok = col < d_out;
  constexpr bool Q8 = EPI == EPI_SCALE_I8 || EPI == EPI_SCALE_E4M3;   // 8-bit weights
  constexpr bool Q4 = EPI == EPI_SCALE_I4;                              // int4 weights
  const uint16_t* wp = wsel + col;
  const uint8_t* wq = Q8 ? a.QT + col : nullptr;     // 8 weights = 8 bytes per lane
  const uint8_t* wq4 = Q4 ? a.QT + col / 2 : nullptr;  // 8 weights = 4 bytes per lane
  const uint16_t* wp2 = DUAL ? a.WT2 + col : nullptr;
  const uint64_t pol = l2_evict_first_policy();
  float acc[8], acc2[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) { acc[k] = 0.f; acc2[k] = 0.f; }
  // rows in flight per warp: 4 KB for fp16 (8 rows x 512 B),
  // 8-bit weights 3 KB (12 rows x 256 B), int4 weights 1 KB (8 rows x 128 B;
  // measured on B200 against 16 rows: 4096 -> 11008 at 50 % in 11.8 against
  // 12.9 us); 2 x 4 rows for the dual product
  constexpr int U = DUAL ? 4 : (Q8 ? 12 : 8);

  for (int cb = 0; cb < n_rows; cb += a.chunk) {
    const int c_lo = lo + cb, c_hi = min(hi, c_lo + a.chunk), cn = c_hi - c_lo;
    if (MODE != MASK_DENSE && !placed) {
      if (cb > 0) __syncthreads();   // the previous chunk's rows are no longer read
      if (MODE == MASK_IDX) {
        for (int j = tid; j < cn; j += kThreads) {
          const int i = __ldg(a.idx + c_lo + j);
          sidx[j] = (unsigned)i < (unsigned)d_in ? i : -1;
        }
      } else {
        // one local word per warp, one bit per lane: rank = word's first
        // rank + popcount of the word's lower bits
        for (int w = warp; w < nwords; w += kWarps) {
          const int base = wpre[w];
          if (base >= c_hi) break;                     // uniform across the warp
          const uint32_t bits = words[w];
          const int rk = base + __popc(bits & ((1u << lane) - 1u));
          if (((bits >> lane) & 1u) && rk >= c_lo && rk < c_hi)
            sidx[rk - c_lo] = (s + (w * 4 + (lane >> 3)) * S) * 8 + (lane & 7);
        }
      }
      __syncthreads();
    }
    if (col_ok) {
      for (int j0 = warp; j0 < cn; j0 += kWarps * U) {
        if constexpr (Q4) {
          uint32_t q[U];
          uint16_t xh[U];
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int j = j0 + kWarps * u;
            const int r = j < cn ? sidx[j] : -1;
            if (r >= 0) {
              xh[u] = __ldg(a.x + r);
              q[u] = ld_stream_u32(wq4 + (size_t)r * (size_t)(d_out / 2), pol);
            } else {
              xh[u] = 0;
              q[u] = 0u;
            }
          }
#pragma unroll
          for (int u = 0; u < U; ++u) fma8_i4(acc, q[u], h2f(xh[u]));
        } else if constexpr (Q8) {
          uint2 q[U];
          uint16_t xh[U];
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int j = j0 + kWarps * u;
            const int r = j < cn ? (MODE == MASK_DENSE ? c_lo + j : sidx[j]) : -1;
            if (r >= 0) {
              xh[u] = __ldg(a.x + r);
              q[u] = ld_stream_v2(wq + (size_t)r * d_out, pol);
            } else {
              xh[u] = 0;
              q[u] = make_uint2(0, 0);
            }
          }
#pragma unroll
          for (int u = 0; u < U; ++u) {
            if (EPI == EPI_SCALE_I8) fma8_i8(acc, q[u], h2f(xh[u]));
            else fma8_e4m3(acc, q[u], h2f(xh[u]));
          }
        } else {
          uint4 v[U], v2[U];
          uint16_t xh[U];
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int j = j0 + kWarps * u;
            const int r = j < cn ? (MODE == MASK_DENSE ? c_lo + j : sidx[j]) : -1;
            if (r >= 0) {
              xh[u] = __ldg(a.x + r);
              v[u] = ld_stream_v4(wp + (size_t)r * d_out, pol);
              if (DUAL) v2[u] = ld_stream_v4(wp2 + (size_t)r * d_out, pol);
            } else {
              xh[u] = 0;
              v[u] = make_uint4(0, 0, 0, 0);
              if (DUAL) v2[u] = make_uint4(0, 0, 0, 0);
            }
          }
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const float xv = h2f(xh[u]);
            fma8(acc, v[u], xv);
            if (DUAL) fma8(acc2, v2[u], xv);
          }
        }
      }
    }
  }

  // ---- 3. CTA partial, then the last two slices finish the tile -------
  __syncthreads();   // the words / prefixes region becomes the warp-sum buffer
  float* red = reinterpret_cast<float*>(smem);
  {
    float4* r4 = reinterpret_cast<float4*>(red + warp * kTile + lane * 8);
    r4[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    r4[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    if (DUAL) {
      float4* q4 = reinterpret_cast<float4*>(red + kWarps * kTile + warp * kTile + lane * 8);
      q4[0] = make_float4(acc2[0], acc2[1], acc2[2], acc2[3]);
      q4[1] = make_float4(acc2[4], acc2[5], acc2[6], acc2[7]);
    }
  }
  __syncthreads();
  float p = 0.f, p2 = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    p += red[w * kTile + tid];
    if (DUAL) p2 += red[kWarps * kTile + w * kTile + tid];
  }
  // the tile's weight again (kept out of registers through the main loop)
  uint16_t* __restrict__ Y = a.y[0];
  int e_dout = a.d_out[0], e_first = 0, e_col0 = 0;
  if (MULTI) {
#pragma unroll
    for (int i = 1; i < kGemvMaxMat; ++i)
      if (i < a.n_mat && cg >= a.tile0[i]) {
        Y = a.y[i]; e_dout = a.d_out[i]; e_first = a.tile0[i]; e_col0 = a.col0[i];
      }
  }
  const int colr = (cg - e_first) * kTile + tid;
  const bool colr_ok = colr < e_dout;
  const int dtot = a.d_out_total;

  // the finished column: fp16(g), fp16(SiLU(g) u) or fp16(s_j g)
  auto store_col = [&](int cc, float g, float u) {
    if (EPI == EPI_SILU_MUL) {
      const float sg = g / (1.0f + expf(-g));
      Y[cc] = f2h_rn(sg * u);
    } else if (EPI == EPI_STORE) {
      Y[cc] = f2h_rn(g);
    } else {
      Y[cc] = f2h_rn(g * __ldg(a.col_scale + cc));
    }
  };
  auto finish = [&](float g, float u) { store_col(colr, g, u); };

  if (S == 1) {
    if (colr_ok) finish(p, p2);
    return;
  }
  // ---- split-K finish: slices S-1 and S-2 finish the tile's two 128-column
  // halves (slice S-1 the first, S-2 the second); every other partial sum is
  // stored as a tagged 64-bit word and the CTA exits
  const unsigned tag = s_tag;
  const int kdes = S - 1 - s;                 // 0 or 1 for the finishing slices
  const bool des = kdes == 0 || kdes == 1;
  const size_t pbase = (size_t)e_col0 + (size_t)(cg - e_first) * kTile;   // tile column 0
  unsigned long long* const slots = a.slots;
  unsigned long long* const slots2 = a.slots + (size_t)S * dtot;
  if (colr_ok && !(des && (tid >> 7) == kdes)) {
    st_relaxed_u64(slots + (size_t)s * dtot + pbase + tid,
                   ((unsigned long long)tag << 32) | __float_as_uint(p));
    if (DUAL)
      st_relaxed_u64(slots2 + (size_t)s * dtot + pbase + tid,
                     ((unsigned long long)tag << 32) | __float_as_uint(p2));
  }
  if (!des) return;
  // this CTA's own partials of every column, then two threads per column of
  // the half it finishes: thread h sums slices [0, mid) (h = 0) or
  // [mid, S) (h = 1) in order, polling each word until it carries the tag
  __syncthreads();                            // the warp sums have been read
  float* own = red;                           // [256] (and [256] for the second product)
  float* half_sum = red + 2 * kTile;          // [128] (and [128])
  own[tid] = p;
  if (DUAL) own[kTile + tid] = p2;
  __syncthreads();
  const int c = kdes * (kTile / 2) + (tid & (kTile / 2 - 1));   // tile column finished here
  const int h = tid >> 7;
  const int mid = S >> 1;
  const int q_lo = h ? mid : 0, q_hi = h ? S : mid;
  const int colc = (cg - e_first) * kTile + c;
  const bool colc_ok = colc < e_dout;
  bool gave_up = false;
  float g = 0.f, u = 0.f;
  if (colc_ok) {
    // words of the column in flight together: a half of up to 20 slices
    // (37 slices of a 16-tile launch) in one batch for the single product
    constexpr int B = DUAL ? 4 : (MULTI ? 16 : 20);
    unsigned long long* sl = slots + pbase + c;
    unsigned long long* sl2 = slots2 + pbase + c;
    const long long t0 = clock64();
    for (int q0 = q_lo; q0 < q_hi; q0 += B) {
      unsigned long long v[B], v2[B];
      uint32_t missing = 0u;
#pragma unroll
      for (int k = 0; k < B; ++k) {
        const int q = q0 + k;
        if (q < q_hi && q != s) {
          v[k] = ld_relaxed_u64(sl + (size_t)q * dtot);
          if (DUAL) v2[k] = ld_relaxed_u64(sl2 + (size_t)q * dtot);
        } else {   // past the range (adds +0), or this CTA's own slice (from shared memory)
          v[k] = ((unsigned long long)tag << 32) | (q < q_hi ? __float_as_uint(own[c]) : 0u);
          v2[k] = ((unsigned long long)tag << 32) |
                  (DUAL && q < q_hi ? __float_as_uint(own[kTile + c]) : 0u);
        }
      }
#pragma unroll
      for (int k = 0; k < B; ++k)
        missing |= ((unsigned)(v[k] >> 32) != tag || (DUAL && (unsigned)(v2[k] >> 32) != tag) ? 1u : 0u) << k;
      while (missing != 0u) {
        if (clock64() - t0 > kFinishSpinCycles) {
          gave_up = true;
          break;
        }
#pragma unroll
        for (int k = 0; k < B; ++k) {
          if ((missing >> k) & 1u) {
            v[k] = ld_relaxed_u64(sl + (size_t)(q0 + k) * dtot);
            if (DUAL) v2[k] = ld_relaxed_u64(sl2 + (size_t)(q0 + k) * dtot);
          }
        }
        missing = 0u;
#pragma unroll
        for (int k = 0; k < B; ++k)
          missing |= ((unsigned)(v[k] >> 32) != tag || (DUAL && (unsigned)(v2[k] >> 32) != tag) ? 1u : 0u) << k;
      }
#pragma unroll
      for (int k = 0; k < B; ++k) {
        g += __uint_as_float((unsigned)v[k]);
        if (DUAL) u += __uint_as_float((unsigned)v2[k]);
      }
    }
  }
  if (h == 1) {
    half_sum[tid & 127] = g;
    if (DUAL) half_sum[kTile / 2 + (tid & 127)] = u;
  }
  __syncthreads();
  if (h == 0 && colc_ok) {
    const float gs = g + half_sum[tid];                      // slices [0, mid) then [mid, S)
    const float us = DUAL ? u + half_sum[kTile / 2 + tid] : 0.f;
    store_col(colc, gs, us);
  }
  if (gave_up) atomicOr(&g_gemv_error, 2u);
  // the next call tags with tag + 1.  Only a finisher that has seen every
  // slice's word (its half holds a column) knows that every slice has read
  // the epoch; the finisher of a tile's empty second half (a tile of at most
  // 128 columns) must leave the epoch alone, or a slice that reads it late
  // would tag with the next call's tag
  const bool half_has_cols = (cg - e_first) * kTile + kdes * (kTile / 2) < e_dout;
  if (tid == 0 && half_has_cols) st_relaxed_u32(a.epochs + cg, tag);
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

template <int MODE, bool DUAL, int EPI, bool MULTI = false>
cudaError_t launch_t(const GemvPlan& p, const KArgs& k, cudaStream_t stream) {
  auto fn = sgemv_kernel<MODE, DUAL, EPI, MULTI>;
  cudaError_t e =
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(fn, dim3(p.C, p.S), dim3(kThreads), p.smem, stream, k);
}

}  // namespace

GemvPlan plan_gemv_multi(int64_t d_in, const int64_t* d_out, int n_mat, bool dual) {
  GemvPlan p{};
  int64_t total = 0;
  p.C = 0;
  for (int i = 0; i < n_mat; ++i) {
    p.C += (int)((d_out[i] + kTile - 1) / kTile);
    total += d_out[i];
  }
  // launches of up to 16 column tiles may cut the rows finer to fill every
  // CTA slot (16 tiles: 37 slices, 592 CTAs; measured on B200 for 4096 x 4096
  // at 50 %: 6.53 us against 7.12 us with 32 slices, whose 512 CTAs left some
  // SMs with two or three); wider ones stop at 32 slices
  const int cap = p.C > 16 ? 32 : kMaxS;
  p.S = std::max(1, std::min(cap, (kNumSMs * kGemvCtasPerSM) / std::max(1, p.C)));
  // rows per slice: at most ceil(d_in / S) for an index or dense slice, at
  // most 8 ceil(ceil(d_in / 8) / S) for a threshold slice's own groups
  const int64_t groups = (d_in + 7) / 8;
  p.chunk = (int)std::max<int64_t>(1, std::min<int64_t>((groups + p.S - 1) / p.S * 8, kIdxCap));
  const size_t words = round_up((size_t)((d_in + 31) / 32) * 4, 16);
  const size_t red = (size_t)kWarps * kTile * 4 * (dual ? 2 : 1);
  p.smem = std::max(2 * words, red) + round_up((size_t)p.chunk * 4, 16);
  // workspace: one epoch word per column tile, then the slices' 64-bit
  // {partial sum, tag} words
  p.counters = p.S > 1 ? round_up((size_t)p.C * 4, 256) : 0;
  p.partials = p.S > 1 ? round_up((size_t)p.S * total * 8 * (dual ? 2 : 1), 256) : 0;
  return p;
}

GemvPlan plan_gemv(int64_t d_in, int64_t d_out, bool dual) {
  return plan_gemv_multi(d_in, &d_out, 1, dual);
}

cudaError_t launch_gemv(int mode, int epi, const GemvPlan& p, const GemvLaunch& a,
                        cudaStream_t stream) {
  if (a.n_mat < 1 || a.n_mat > kGemvMaxMat) return cudaErrorInvalidValue;
  if (epi == EPI_SILU_MUL && a.n_mat != 1) return cudaErrorInvalidValue;
  KArgs k{};
  k.n_mat = a.n_mat;
  int tiles = 0, cols = 0;
  for (int i = 0; i < a.n_mat; ++i) {
    k.WT[i] = a.WT[i];
    k.y[i] = a.y[i];
    k.d_out[i] = a.d_out[i];
    k.tile0[i] = tiles;
    k.col0[i] = cols;
    tiles += (a.d_out[i] + kTile - 1) / kTile;
    cols += a.d_out[i];
  }
  k.tile0[a.n_mat] = tiles;
  k.d_out_total = cols;
  if (tiles != p.C) return cudaErrorInvalidValue;
  k.WT2 = a.WT2; k.x = a.x; k.scale = a.scale; k.idx = a.idx; k.nnz = a.nnz;
  k.col_scale = a.col_scale; k.QT = a.QT;
  k.t = a.t; k.d_in = a.d_in; k.S = p.S; k.chunk = p.chunk;
  const size_t words = round_up((size_t)((a.d_in + 31) / 32) * 4, 16);
  const size_t red = (size_t)kWarps * kTile * 4 * (epi == EPI_SILU_MUL ? 2 : 1);
  k.words_bytes = (uint32_t)words;
  k.union_bytes = (uint32_t)std::max(2 * words, red);
  k.mask_out = a.mask_out;
  k.epochs = reinterpret_cast<unsigned*>(a.ws);
  k.slots = a.ws != nullptr
                ? reinterpret_cast<unsigned long long*>(reinterpret_cast<char*>(a.ws) + p.counters)
                : nullptr;
  if (epi == EPI_SCALE_I8 || epi == EPI_SCALE_E4M3 || epi == EPI_SCALE_I4) {
    if (mode != MASK_THRESH || a.n_mat != 1 || a.QT == nullptr) return cudaErrorInvalidValue;
    if (epi == EPI_SCALE_I8) return launch_t<MASK_THRESH, false, EPI_SCALE_I8>(p, k, stream);
    if (epi == EPI_SCALE_I4) return launch_t<MASK_THRESH, false, EPI_SCALE_I4>(p, k, stream);
    return launch_t<MASK_THRESH, false, EPI_SCALE_E4M3>(p, k, stream);
  }
  if (epi == EPI_SILU_MUL) {
    if (mode == MASK_DENSE) return launch_t<MASK_DENSE, true, EPI_SILU_MUL>(p, k, stream);
    if (mode == MASK_THRESH) return launch_t<MASK_THRESH, true, EPI_SILU_MUL>(p, k, stream);
    return cudaErrorInvalidValue;
  }
  if (a.n_mat > 1) {
    if (mode == MASK_THRESH) return launch_t<MASK_THRESH, false, EPI_STORE, true>(p, k, stream);
    if (mode == MASK_IDX) return launch_t<MASK_IDX, false, EPI_STORE, true>(p, k, stream);
    return cudaErrorInvalidValue;
  }
  switch (mode) {
    case MASK_THRESH: return launch_t<MASK_THRESH, false, EPI_STORE>(p, k, stream);
    case MASK_THRESH_SCALED: return launch_t<MASK_THRESH_SCALED, false, EPI_STORE>(p, k, stream);
    case MASK_SQUARE: return launch_t<MASK_SQUARE, false, EPI_STORE>(p, k, stream);
    case MASK_IDX: return launch_t<MASK_IDX, false, EPI_STORE>(p, k, stream);
    case MASK_DENSE: return launch_t<MASK_DENSE, false, EPI_STORE>(p, k, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t read_gemv_error(unsigned* out, cudaStream_t stream) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_gemv_error, sizeof(unsigned), 0,
                                            cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  const unsigned zero = 0;
  return cudaMemcpyToSymbolAsync(g_gemv_error, &zero, sizeof(unsigned), 0, cudaMemcpyHostToDevice,
                                 stream);
}

}  // namespace sig
