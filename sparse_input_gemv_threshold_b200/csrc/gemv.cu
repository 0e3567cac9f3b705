// Split-K sparse-input GEMV y = W (m . x) with the mask step fused ahead of it.
//
// The product reads only the weight rows of the kept inputs ("Adaptive Rank
// Allocation ... RaNA Adapters", Q5.1: the columns of A that meet a zero mask
// entry are skipped).  WT is stored transposed (d_in x d_out, row-major), so a
// kept input i costs one contiguous row of 2*d_out bytes.
//
// One launch does everything:
//   1. every CTA ballots the whole activation (it sits in L2), packs the mask
//      into shared words and prefix-scans their popcounts, which gives nnz and
//      the CTA's equal share [lo, hi) of the ascending kept-row list; each
//      thread then places its ranks by a binary search over the word prefixes;
//   2. the CTA streams its share of kept rows for its 256-column tile with
//      16-byte non-allocating loads, 8 rows in flight per warp (each with its
//      activation value, a broadcast load), fp32 FMA;
//   3. the 8 warps' sums meet in shared memory, the CTA writes one fp32 partial
//      per column, and the CTA that arrives last for the tile (a counter in
//      the workspace) adds the partials in split order and stores fp16.
// The reduction order is fixed, so y is bit-identical from run to run; no
// floating-point atomics are used and no CTA ever waits for another.
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace sig {

namespace {

struct KArgs {
  const uint16_t* WT;
  const uint16_t* WT2;
  const uint16_t* x;
  const float* scale;
  const int32_t* idx;
  const int32_t* nnz;
  float t;
  int d_in, d_out, S, cap;
  uint32_t words_bytes;   // shared bytes of the mask words (and of their prefixes)
  uint32_t union_bytes;   // shared bytes of the words + prefixes / reduction union
  uint16_t* y;
  uint32_t* mask_out;
  unsigned* counters;
  float* partials;        // [S][d_out] (then [S][d_out] for the second product)
};

template <int MODE, bool DUAL, int EPI>
__global__ void __launch_bounds__(kGemvThreads, kGemvCtasPerSM)
sgemv_kernel(const KArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int scan_scratch[kGemvThreads / 32 + 1];
  __shared__ int s_last;

  constexpr int kWarps = kGemvThreads / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x, s = blockIdx.y;
  const int d_in = a.d_in, d_out = a.d_out, S = a.S;

  uint32_t* words = reinterpret_cast<uint32_t*>(smem);
  int* wpre = reinterpret_cast<int*>(smem + a.words_bytes);
  int* sidx = reinterpret_cast<int*>(smem + a.union_bytes);

  pdl_trigger();
  pdl_wait();

  // ---- 1. which rows does this CTA own? --------------------------------
  int n_rows = 0;
  if (MODE == MASK_THRESH || MODE == MASK_THRESH_SCALED) {
    const float t = a.t;
    const float* scale = a.scale;
    build_mask_words<kGemvThreads>(a.x, d_in, words, [&](uint16_t h, int i) {
      const float m = fabsf(h2f(h));
      if (MODE == MASK_THRESH_SCALED) return __fmul_rn(m, __ldg(scale + i)) >= t;
      return m >= t;
    });
    __syncthreads();
    const int nwords = (d_in + 31) >> 5;
    const int per = (nwords + kGemvThreads - 1) / kGemvThreads;
    const int w0 = min(nwords, tid * per), w1 = min(nwords, w0 + per);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(words[w]);
    int total;
    int r = block_exclusive_scan<kGemvThreads>(cnt, scan_scratch, &total);
    for (int w = w0; w < w1; ++w) {   // exclusive kept-count before each word
      wpre[w] = r;
      r += __popc(words[w]);
    }
    __syncthreads();
    const int lo = (int)(((long long)s * total) / S);
    const int hi = (int)(((long long)(s + 1) * total) / S);
    n_rows = hi - lo;
    // Every thread places its own ranks: the word holding rank lo + j is the
    // last one whose prefix is <= that rank; __fns finds the bit inside it.
    for (int j = tid; j < n_rows; j += kGemvThreads) {
      const int rank = lo + j;
      int a0 = 0, a1 = nwords - 1;
      while (a0 < a1) {
        const int mid = (a0 + a1 + 1) >> 1;
        if (wpre[mid] <= rank) a0 = mid; else a1 = mid - 1;
      }
      sidx[j] = a0 * 32 + (int)__fns(words[a0], 0, rank - wpre[a0] + 1);
    }
    if (a.mask_out != nullptr && c == 0 && s == 0)
      for (int w = tid; w < nwords; w += kGemvThreads) a.mask_out[w] = words[w];
  } else if (MODE == MASK_IDX) {
    const int total = min(max(__ldg(a.nnz), 0), d_in);
    const int lo = (int)(((long long)s * total) / S);
    const int hi = (int)(((long long)(s + 1) * total) / S);
    n_rows = hi - lo;
    for (int j = tid; j < n_rows; j += kGemvThreads) {
      const int i = __ldg(a.idx + lo + j);
      sidx[j] = (unsigned)i < (unsigned)d_in ? i : -1;
    }
  } else {  // MASK_DENSE
    const int lo = (int)(((long long)s * d_in) / S);
    const int hi = (int)(((long long)(s + 1) * d_in) / S);
    n_rows = hi - lo;
    for (int j = tid; j < n_rows; j += kGemvThreads) sidx[j] = lo + j;
  }
  __syncthreads();

  // ---- 2. stream the kept rows of this column tile ----------------------
  const int col = c * kGemvTile + lane * 8;
  const bool col_ok = col < d_out;
  float acc[8], acc2[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) { acc[k] = 0.f; acc2[k] = 0.f; }

  if (col_ok) {
    const uint16_t* wp = a.WT + col;
    const uint16_t* wp2 = DUAL ? a.WT2 + col : nullptr;
    const uint64_t pol = l2_evict_first_policy();
    // U rows per warp in flight; the last batch is predicated, so a warp with
    // only a few rows still issues all of its loads at once.
    constexpr int U = DUAL ? 4 : 8;
    for (int j0 = warp; j0 < n_rows; j0 += kWarps * U) {
      uint4 v[U], v2[U];
      uint16_t xh[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + kWarps * u;
        const int r = j < n_rows ? sidx[j] : -1;
        if (r >= 0) {
          // the activation rides along with its weight row: both in flight
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

  // ---- 3. CTA partial, then the last arriver finishes the tile ---------
  // The words region is free again (only the prologue read it).
  float* red = reinterpret_cast<float*>(smem);
  float4* red4 = reinterpret_cast<float4*>(red + warp * kGemvTile + lane * 8);
  red4[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  red4[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  if (DUAL) {
    float4* r2 = reinterpret_cast<float4*>(red + kWarps * kGemvTile + warp * kGemvTile + lane * 8);
    r2[0] = make_float4(acc2[0], acc2[1], acc2[2], acc2[3]);
    r2[1] = make_float4(acc2[4], acc2[5], acc2[6], acc2[7]);
  }
  __syncthreads();
  float p = 0.f, p2 = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    p += red[w * kGemvTile + tid];
    if (DUAL) p2 += red[kWarps * kGemvTile + w * kGemvTile + tid];
  }
  const int colr = c * kGemvTile + tid;
  const bool colr_ok = colr < d_out;

  auto finish = [&](float g, float u) {
    if (EPI == EPI_STORE) {
      a.y[colr] = f2h_rn(g);
    } else {
      const float sg = g / (1.0f + expf(-g));
      a.y[colr] = f2h_rn(sg * u);
    }
  };

  if (S == 1) {
    if (colr_ok) finish(p, p2);
    return;
  }

  if (colr_ok) {
    a.partials[(size_t)s * d_out + colr] = p;
    if (DUAL) a.partials[(size_t)S * d_out + (size_t)s * d_out + colr] = p2;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(a.counters + c, 1u) == (unsigned)(S - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (colr_ok) {
    // all loads of a batch in flight together, then added in split order
    constexpr int B = DUAL ? 16 : 32;
    float g = 0.f, u = 0.f;
    for (int q0 = 0; q0 < S; q0 += B) {
      float pg[B], pu[B];
#pragma unroll
      for (int k = 0; k < B; ++k) {
        const bool ok = q0 + k < S;
        pg[k] = ok ? __ldcg(a.partials + (size_t)(q0 + k) * d_out + colr) : 0.f;
        if (DUAL) pu[k] = ok ? __ldcg(a.partials + (size_t)S * d_out + (size_t)(q0 + k) * d_out + colr) : 0.f;
      }
#pragma unroll
      for (int k = 0; k < B; ++k) {
        g += pg[k];
        if (DUAL) u += pu[k];
      }
    }
    finish(g, u);
  }
  if (tid == 0) a.counters[c] = 0u;  // ready for the next call on this workspace
}

template <int MODE, bool DUAL, int EPI>
cudaError_t launch_t(const GemvPlan& p, const KArgs& k, cudaStream_t stream) {
  auto fn = sgemv_kernel<MODE, DUAL, EPI>;
  static bool attr_done = false;  // per instantiation; the attribute is per function
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         96 * 1024);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  return launch_pdl(fn, dim3(p.C, p.S), dim3(kGemvThreads), p.smem, stream, k);
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

GemvPlan plan_gemv(int64_t d_in, int64_t d_out, bool dual) {
  GemvPlan p{};
  p.C = (int)((d_out + kGemvTile - 1) / kGemvTile);
  int S = std::max(1, (kNumSMs * kGemvCtasPerSM) / p.C);
  S = (int)std::min<int64_t>(S, std::max<int64_t>(1, d_in));
  S = std::max<int>(S, (int)((d_in + kIdxCap - 1) / kIdxCap));
  p.S = S;
  p.cap = (int)((d_in + S - 1) / S);
  const size_t words = round_up((size_t)((d_in + 31) / 32) * 4, 16);
  const size_t red = (size_t)(kGemvThreads / 32) * kGemvTile * 4 * (dual ? 2 : 1);
  const size_t uni = std::max(2 * words, red);
  p.smem = uni + round_up((size_t)p.cap * 4, 16);
  p.counters = round_up((size_t)p.C * 4, 256);
  p.partials = S > 1 ? round_up((size_t)S * d_out * 4 * (dual ? 2 : 1), 256) : 0;
  return p;
}

cudaError_t launch_gemv(int mode, int epi, const GemvPlan& p, const GemvLaunch& a,
                        cudaStream_t stream) {
  KArgs k{};
  k.WT = a.WT; k.WT2 = a.WT2; k.x = a.x; k.scale = a.scale; k.idx = a.idx; k.nnz = a.nnz;
  k.t = a.t; k.d_in = a.d_in; k.d_out = a.d_out; k.S = p.S; k.cap = p.cap;
  const size_t words = round_up((size_t)((a.d_in + 31) / 32) * 4, 16);
  const size_t red = (size_t)(kGemvThreads / 32) * kGemvTile * 4 * (epi == EPI_SILU_MUL ? 2 : 1);
  k.words_bytes = (uint32_t)words;
  k.union_bytes = (uint32_t)std::max(2 * words, red);
  k.y = a.y; k.mask_out = a.mask_out;
  k.counters = reinterpret_cast<unsigned*>(a.ws);
  k.partials = reinterpret_cast<float*>(reinterpret_cast<char*>(a.ws) + p.counters);
  if (epi == EPI_SILU_MUL) {
    if (mode != MASK_DENSE) return cudaErrorInvalidValue;
    return launch_t<MASK_DENSE, true, EPI_SILU_MUL>(p, k, stream);
  }
  switch (mode) {
    case MASK_THRESH: return launch_t<MASK_THRESH, false, EPI_STORE>(p, k, stream);
    case MASK_THRESH_SCALED: return launch_t<MASK_THRESH_SCALED, false, EPI_STORE>(p, k, stream);
    case MASK_IDX: return launch_t<MASK_IDX, false, EPI_STORE>(p, k, stream);
    case MASK_DENSE: return launch_t<MASK_DENSE, false, EPI_STORE>(p, k, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace sig
