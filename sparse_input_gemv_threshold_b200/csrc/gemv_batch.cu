// A few tokens, each with its own threshold mask, through one weight:
// y_b = W (m_b . x_b), m_b,i = |x_b,i| >= t, for b < B <= 8.
//
// The pages define the single-token product ("Adaptive Rank Allocation ...
// RaNA Adapters", rebuttal Q5.1: the columns of A that meet a zero mask entry
// are skipped) and leave the batched case with inconsistent masks open (Q6).
// Here one launch reads every weight row that ANY token keeps (the union of
// the masks) once from HBM and applies each token's own mask to it in
// registers: a row that token b drops contributes x_b,i = 0 to y_b.
//
// Launch shape, as the single-token kernel: C x S CTAs of 256 threads, a CTA
// owns a 256-output column tile (one warp spans it with 16-byte lanes) and
// the union rows of its interleaved 8-input groups (slice s owns groups s,
// s+S, s+2S, ...), staged in shared memory with the tokens' masked values:
//   1. the CTA loads its groups of every token's x (from L2), ballots the
//      union of their fp16 threshold compares into shared words, prefix-sums
//      the words' popcounts and places the union rows in ascending order,
//      each with the NB masked token values (0 where that token drops it);
//   2. 8 warps stream the rows of the tile, 6 or 8 in flight per warp, FMA
//      into NB x 8 float32 accumulators per lane;
//   3. per token, the warps' sums meet in shared memory, the CTA writes one
//      partial per column, and the last CTA to arrive for the tile (one
//      acquire-release atomic per CTA) adds the S partials of every token in
//      slice order and stores fp16.
// Deterministic: no floating-point atomics, no spin-waits.
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace sig {

namespace {

constexpr int kThreads = kGemvThreads;   // 256
constexpr int kWarps = kThreads / 32;
constexpr int kTile = kGemvTile;         // 256

struct BArgs {
  const uint16_t* WT;     // d_in x d_out
  const uint16_t* X;      // B x d_in, row-major
  uint16_t* Y;            // B x d_out, row-major
  float t;
  int B, d_in, d_out, S, chunk;
  uint32_t words_bytes;   // shared bytes of the union words (and again of their prefixes)
  uint32_t union_bytes;   // shared bytes of words + prefixes / the warp-sum buffer
  unsigned* counters;     // [C]
  float* partials;        // [S][B][d_out]
};

// CTAs per SM each width is sized for (registers: NB x 8 accumulators).
template <int NB>
constexpr int ctas_per_sm() { return NB <= 2 ? 4 : NB <= 4 ? 3 : 2; }

template <int NB>
__global__ void __launch_bounds__(kThreads, ctas_per_sm<NB>())
batch_gemv_kernel(const __grid_constant__ BArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int warp_tot[kWarps];
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x, s = blockIdx.y;
  const int d_in = a.d_in, d_out = a.d_out, S = a.S, B = a.B;

  uint32_t* words = reinterpret_cast<uint32_t*>(smem);
  int* wpre = reinterpret_cast<int*>(smem + a.words_bytes);
  int* sidx = reinterpret_cast<int*>(smem + a.union_bytes);
  uint16_t* sxv = reinterpret_cast<uint16_t*>(smem + a.union_bytes + (size_t)a.chunk * 4);

  pdl_trigger();
  pdl_wait();

  // ---- 1. the union of the tokens' masks over this slice's groups -------
  const __half2 th2 = thresh_half2(a.t);
  const int ngroups = (d_in + 7) >> 3;    // d_in % 8 == 0: whole groups
  const int K = s < ngroups ? (ngroups - 1 - s) / S + 1 : 0;
  const int nwords = (K + 3) >> 2;
  for (int lw = tid; lw < nwords; lw += kThreads) {
    uint32_t w = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int k = lw * 4 + q;
      if (k < K) {
        const int e0 = (s + k * S) * 8;
        uint32_t u = 0;
        for (int b = 0; b < B; ++b)
          u |= thresh_bits8(__ldg(reinterpret_cast<const uint4*>(a.X + (size_t)b * d_in + e0)), th2);
        w |= u << (8 * q);
      }
    }
    words[lw] = w;
  }
  __syncthreads();
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
  int r0 = before + incl - cnt;
  for (int w = w0; w < w1; ++w) {
    wpre[w] = r0;
    r0 += __popc(words[w]);
  }
  __syncthreads();

  // ---- 2. stream the union rows of this column tile ---------------------
  const int col = c * kTile + lane * 8;
  const bool col_ok = col < d_out;
  const uint16_t* wp = a.WT + col;
  const uint64_t pol = l2_evict_first_policy();
  float acc[NB][8];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[b][k] = 0.f;
  constexpr int U = NB == 8 ? 8 : 6;   // rows in flight per warp (registers: NB x 8 accumulators)

  for (int cb = 0; cb < total; cb += a.chunk) {
    const int c_lo = cb, c_hi = min(total, cb + a.chunk), cn = c_hi - c_lo;
    if (cb > 0) __syncthreads();   // the previous chunk's rows are no longer read
    // one word per warp, one bit per lane; the row's masked token values beside it
    for (int w = warp; w < nwords; w += kWarps) {
      const int base = wpre[w];
      if (base >= c_hi) break;                       // uniform across the warp
      const uint32_t bits = words[w];
      const int rk = base + __popc(bits & ((1u << lane) - 1u));
      if (((bits >> lane) & 1u) && rk >= c_lo && rk < c_hi) {
        const int i = (s + (w * 4 + (lane >> 3)) * S) * 8 + (lane & 7);
        sidx[rk - c_lo] = i;
        uint16_t* dst = sxv + (size_t)(rk - c_lo) * NB;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          uint16_t h = 0;
          if (b < B) {
            h = a.X[(size_t)b * d_in + i];
            if (!(fabsf(h2f(h)) >= __half2float(__low2half(th2)))) h = 0;
          }
          dst[b] = h;
        }
      }
    }
    __syncthreads();
    if (col_ok) {
      for (int j0 = warp; j0 < cn; j0 += kWarps * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int j = j0 + kWarps * u;
          v[u] = j < cn ? ld_stream_v4(wp + (size_t)sidx[j] * d_out, pol) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int j = j0 + kWarps * u;
          if (j < cn) {
            const uint16_t* xs = sxv + (size_t)j * NB;
#pragma unroll
            for (int b = 0; b < NB; ++b) fma8(acc[b], v[u], h2f(xs[b]));
          }
        }
      }
    }
  }

  // ---- 3. per token: CTA partial; the last arriver finishes the tile ----
  float* red = reinterpret_cast<float*>(smem);
  const int colr = c * kTile + tid;
  const bool colr_ok = colr < d_out;
  float p[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    __syncthreads();   // the previous use of the buffer is over
    float4* r4 = reinterpret_cast<float4*>(red + warp * kTile + lane * 8);
    r4[0] = make_float4(acc[b][0], acc[b][1], acc[b][2], acc[b][3]);
    r4[1] = make_float4(acc[b][4], acc[b][5], acc[b][6], acc[b][7]);
    __syncthreads();
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) sum += red[w * kTile + tid];
    p[b] = sum;
  }
  if (S == 1) {
    if (colr_ok) {
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if (b < B) a.Y[(size_t)b * d_out + colr] = f2h_rn(p[b]);
    }
    return;
  }
  if (colr_ok) {
#pragma unroll
    for (int b = 0; b < NB; ++b)
      if (b < B) a.partials[((size_t)s * B + b) * d_out + colr] = p[b];
  }
  __syncthreads();
  if (tid == 0) s_last = atomic_add_acq_rel_gpu(a.counters + c, 1u) == (unsigned)(S - 1);
  __syncthreads();
  if (!s_last) return;
  if (colr_ok) {
    for (int b = 0; b < B; ++b) {
      const float* pp = a.partials + (size_t)b * d_out + colr;
      float g = 0.f;
      for (int q0 = 0; q0 < S; q0 += 32) {
        float pg[32];
#pragma unroll
        for (int k = 0; k < 32; ++k)
          pg[k] = q0 + k < S ? __ldcg(pp + (size_t)(q0 + k) * B * d_out) : 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) g += pg[k];
      }
      a.Y[(size_t)b * d_out + colr] = f2h_rn(g);
    }
  }
  if (tid == 0) a.counters[c] = 0u;  // ready for the next call on this workspace
}

size_t round_up(size_t v, size_t al) { return (v + al - 1) / al * al; }

int width_for(int B) { return B <= 2 ? 2 : B <= 4 ? 4 : 8; }

template <int NB>
cudaError_t launch_nb(const GemvPlan& p, const BArgs& k, cudaStream_t stream) {
  auto fn = batch_gemv_kernel<NB>;
  cudaError_t e =
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(fn, dim3(p.C, p.S), dim3(kThreads), p.smem, stream, k);
}

}  // namespace

GemvPlan plan_gemv_batch(int64_t d_in, int64_t d_out, int B) {
  GemvPlan p{};
  const int nb = width_for(B);
  const int cps = nb <= 2 ? 4 : nb <= 4 ? 3 : 2;
  p.C = (int)((d_out + kTile - 1) / kTile);
  p.S = std::max(1, std::min(32, (kNumSMs * cps) / std::max(1, p.C)));
  const int64_t groups = (d_in + 7) / 8;
  p.chunk = (int)std::max<int64_t>(1, std::min<int64_t>((groups + p.S - 1) / p.S * 8, 2048));
  const size_t words = round_up((size_t)((d_in + 31) / 32) * 4, 16);
  const size_t red = (size_t)kWarps * kTile * 4;
  p.smem = std::max(2 * words, red) + round_up((size_t)p.chunk * 4, 16) +
           round_up((size_t)p.chunk * nb * 2, 16);
  p.counters = p.S > 1 ? round_up((size_t)p.C * 4, 256) : 0;
  p.partials = p.S > 1 ? round_up((size_t)p.S * B * d_out * 4, 256) : 0;
  return p;
}

cudaError_t launch_gemv_batch(const GemvPlan& p, const uint16_t* WT, const uint16_t* X, uint16_t* Y,
                              int B, int d_in, int d_out, float t, void* ws, cudaStream_t stream) {
  BArgs k{};
  k.WT = WT; k.X = X; k.Y = Y; k.t = t; k.B = B; k.d_in = d_in; k.d_out = d_out;
  k.S = p.S; k.chunk = p.chunk;
  const size_t words = round_up((size_t)((d_in + 31) / 32) * 4, 16);
  k.words_bytes = (uint32_t)words;
  k.union_bytes = (uint32_t)std::max(2 * words, (size_t)kWarps * kTile * 4);
  k.counters = reinterpret_cast<unsigned*>(ws);
  k.partials = ws != nullptr ? reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + p.counters)
                             : nullptr;
  switch (width_for(B)) {
    case 2: return launch_nb<2>(p, k, stream);
    case 4: return launch_nb<4>(p, k, stream);
    default: return launch_nb<8>(p, k, stream);
  }
}

}  // namespace sig
