// Weight-quantised sparse GEMV: y_j = s_j * sum_i q_ij (m_i x_i), m_i = |x_i| >= t,
// q int8 or fp8 e4m3 (stored transposed, d_in x d_out), s float32 per output
// column.
//
// The pages leave quantised sparse kernels open (TEAL README, Limitations)
// and call weight quantisation orthogonal to activation sparsity: it shrinks
// the bytes moved per decoding step (Q-Sparse rebuttal, A1 on batched
// inference).  Here both act at once: a kept input costs one 8-bit row of
// d_out bytes, half the fp16 row.
//
// Same structure as the fp16 kernel, with a 512-column tile (a warp spans it
// with 16 weights = 16 bytes per lane):
//   1. the CTA masks its interleaved 8-input groups of x (slice s owns groups
//      s, s+S, ...) with fp16 SIMD compares: one group per thread and one
//      block-wide scan of the popcounts place its kept rows in ascending
//      order (slices of more than 256 groups take the chunked path of words,
//      prefixes and per-chunk placement);
//   2. 8 warps stream the rows, 6 in flight per warp; each weight becomes an
//      exact fp16 value (int8: byte permute into 1024 + u and one half2
//      subtract; e4m3: the hardware e4m3x2 -> f16x2 conversion), then two
//      columns at a time go through one packed float32 FMA (fma.rn.f32x2)
//      with the activation;
//   3. the warps meet in shared memory, the CTA writes one partial per
//      column, and the last CTA to arrive (one acquire-release atomic) adds
//      the S partials in slice order, multiplies by s_j and stores fp16.
#include "common.cuh"
#include "gemv_q8.h"

#include <cuda_fp8.h>

#include <algorithm>

namespace sig {

namespace {

constexpr int kThreads = kGemvThreads;    // 256
constexpr int kWarps = kThreads / 32;     // 8
constexpr int kTile = kQ8Tile;            // 512
constexpr int kCtasPerSM = 4;
constexpr int kMaxS = 64;                 // 32 unless fewer than 16 column tiles

struct QArgs {
  const uint8_t* QT;
  const float* scale;
  const uint16_t* x;
  uint16_t* y;
  float t;
  int d_in, d_out, S, chunk;
  uint32_t words_bytes, union_bytes;
  unsigned* counters;
  float* partials;   // [S][d_out]
};

// acc[k] += (w_2k, w_2k+1) * xv for the 16 int8 weights packed in v.
__device__ __forceinline__ void fma16_q8(float2 (&acc)[8], const uint4& v, float2 xv) {
  const uint32_t w[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u, v.z ^ 0x80808080u,
                         v.w ^ 0x80808080u};   // u = q + 128
  const __half2 bias = __half2half2(__ushort_as_half((uint16_t)0x6480));   // 1152 = 1024 + 128
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t lo = __byte_perm(w[k], 0x64646464u, 0x4140);   // halves 1024 + u0, 1024 + u1
    const uint32_t hi = __byte_perm(w[k], 0x64646464u, 0x4342);   // halves 1024 + u2, 1024 + u3
    const float2 a = __half22float2(__hsub2(*reinterpret_cast<const __half2*>(&lo), bias));
    const float2 b = __half22float2(__hsub2(*reinterpret_cast<const __half2*>(&hi), bias));
    acc[2 * k] = __ffma2_rn(a, xv, acc[2 * k]);
    acc[2 * k + 1] = __ffma2_rn(b, xv, acc[2 * k + 1]);
  }
}

// The same for 16 fp8 e4m3 weights: every e4m3 value is exact in fp16.
__device__ __forceinline__ void fma16_e4m3(float2 (&acc)[8], const uint4& v, float2 xv) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[k] & 0xffffu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[k] >> 16), __NV_E4M3);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    acc[2 * k] = __ffma2_rn(a, xv, acc[2 * k]);
    acc[2 * k + 1] = __ffma2_rn(b, xv, acc[2 * k + 1]);
  }
}

template <int FMT>
__global__ void __launch_bounds__(kThreads, kCtasPerSM)
q8_gemv_kernel(const __grid_constant__ QArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int warp_tot[kWarps];
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x, s = blockIdx.y;
  const int d_in = a.d_in, d_out = a.d_out, S = a.S;
  uint32_t* words = reinterpret_cast<uint32_t*>(smem);
  int* wpre = reinterpret_cast<int*>(smem + a.words_bytes);
  int* sidx = reinterpret_cast<int*>(smem + a.union_bytes);

  pdl_trigger();
  pdl_wait();

  // ---- 1. this slice's kept rows ----------------------------------------
  const __half2 th2 = thresh_half2(a.t);
  const int ngroups = (d_in + 7) >> 3;
  const int K = s < ngroups ? (ngroups - 1 - s) / S + 1 : 0;
  const int nwords = (K + 3) >> 2;
  int total = 0;
  bool placed = false;   // the kept-row list is already in sidx (one chunk)
  if (K <= kThreads) {
    // one group per thread, one block-wide scan, each thread places its rows
    const int e0 = (s + tid * S) * 8;
    uint32_t b = 0;
    if (tid < K) {
      if (e0 + 8 <= d_in) {
        b = thresh_bits8(__ldg(reinterpret_cast<const uint4*>(a.x + e0)), th2);
      } else {
        for (int j = 0; e0 + j < d_in; ++j)
          b |= (fabsf(h2f(a.x[e0 + j])) >= __half2float(__low2half(th2)) ? 1u : 0u) << j;
      }
    }
    const int cnt = __popc(b);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int v = warp_tot[w];
      before += w < warp ? v : 0;
      total += v;
    }
    int r = before + incl - cnt;
    for (uint32_t m = b; m != 0u; m &= m - 1u) sidx[r++] = e0 + (__ffs(m) - 1);
    placed = true;
    __syncthreads();
  } else {
    for (int lw = tid; lw < nwords; lw += kThreads) {
      uint4 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
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
        if (e0 + 8 <= d_in) {
          b = thresh_bits8(v[q], th2);
        } else {
          for (int j = 0; e0 + j < d_in; ++j)
            b |= (fabsf(h2f(a.x[e0 + j])) >= __half2float(__low2half(th2)) ? 1u : 0u) << j;
        }
        w |= b << (8 * q);
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
    int before = 0;
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
  }

  // ---- 2. stream the kept 8-bit rows of this column tile -----------------
  const int col = c * kTile + lane * 16;
  const bool col_ok = col < d_out;            // d_out % 16 == 0: whole 16-byte lanes
  const uint8_t* wp = a.QT + col;
  const uint64_t pol = l2_evict_first_policy();
  float2 acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = make_float2(0.f, 0.f);
  constexpr int U = 6;

  for (int cb = 0; cb < total; cb += a.chunk) {
    const int c_lo = cb, c_hi = min(total, cb + a.chunk), cn = c_hi - c_lo;
    if (cb > 0) __syncthreads();
    for (int w = warp; w < nwords && !placed; w += kWarps) {
      const int base = wpre[w];
      if (base >= c_hi) break;
      const uint32_t bits = words[w];
      const int rk = base + __popc(bits & ((1u << lane) - 1u));
      if (((bits >> lane) & 1u) && rk >= c_lo && rk < c_hi)
        sidx[rk - c_lo] = (s + (w * 4 + (lane >> 3)) * S) * 8 + (lane & 7);
    }
    if (!placed) __syncthreads();
    if (col_ok) {
      for (int j0 = warp; j0 < cn; j0 += kWarps * U) {
        uint4 v[U];
        uint16_t xh[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int j = j0 + kWarps * u;
          if (j < cn) {
            const int r = sidx[j];
            xh[u] = __ldg(a.x + r);
            v[u] = ld_stream_v4(wp + (size_t)r * d_out, pol);
          } else {
            xh[u] = 0;
            v[u] = make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const float xv = h2f(xh[u]);
          if (FMT == kFmtInt8) fma16_q8(acc, v[u], make_float2(xv, xv));
          else fma16_e4m3(acc, v[u], make_float2(xv, xv));
        }
      }
    }
  }

  // ---- 3. CTA partials, then the last arriver finishes the tile ---------
  __syncthreads();   // the words / prefixes region becomes the warp-sum buffer
  float* red = reinterpret_cast<float*>(smem);
  {
    float4* r4 = reinterpret_cast<float4*>(red + warp * kTile + lane * 16);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      r4[k] = make_float4(acc[2 * k].x, acc[2 * k].y, acc[2 * k + 1].x, acc[2 * k + 1].y);
  }
  __syncthreads();
  float p[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += red[w * kTile + h * kThreads + tid];
    p[h] = v;
  }
  if (S == 1) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cr = c * kTile + h * kThreads + tid;
      if (cr < d_out) a.y[cr] = f2h_rn(p[h] * __ldg(a.scale + cr));
    }
    return;
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int cr = c * kTile + h * kThreads + tid;
    if (cr < d_out) a.partials[(size_t)s * d_out + cr] = p[h];
  }
  __syncthreads();
  if (tid == 0) s_last = atomic_add_acq_rel_gpu(a.counters + c, 1u) == (unsigned)(S - 1);
  __syncthreads();
  if (!s_last) return;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int cr = c * kTile + h * kThreads + tid;
    if (cr < d_out) {
      const float* pp = a.partials + cr;
      float g = 0.f;
      for (int q0 = 0; q0 < S; q0 += 32) {   // 32 partials in flight, added in slice order
        float pg[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) pg[k] = q0 + k < S ? __ldcg(pp + (size_t)(q0 + k) * d_out) : 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) g += pg[k];
      }
      a.y[cr] = f2h_rn(g * __ldg(a.scale + cr));
    }
  }
  if (tid == 0) a.counters[c] = 0u;  // ready for the next call on this workspace
}

size_t round_up(size_t v, size_t al) { return (v + al - 1) / al * al; }

}  // namespace

GemvPlan plan_gemv_q8(int64_t d_in, int64_t d_out) {
  GemvPlan p{};
  p.C = (int)((d_out + kTile - 1) / kTile);
  const int cap = p.C >= 16 ? 32 : kMaxS;
  p.S = std::max(1, std::min(cap, (kNumSMs * kCtasPerSM) / std::max(1, p.C)));
  const int64_t groups = (d_in + 7) / 8;
  p.chunk = (int)std::max<int64_t>(1, std::min<int64_t>((groups + p.S - 1) / p.S * 8, kIdxCap));
  const size_t words = round_up((size_t)((d_in + 31) / 32) * 4, 16);
  const size_t red = (size_t)kWarps * kTile * 4;
  p.smem = std::max(2 * words, red) + round_up((size_t)p.chunk * 4, 16);
  p.counters = p.S > 1 ? round_up((size_t)p.C * 4, 256) : 0;
  p.partials = p.S > 1 ? round_up((size_t)p.S * d_out * 4, 256) : 0;
  return p;
}

cudaError_t launch_gemv_q8(const GemvPlan& p, int fmt, const uint8_t* QT, const float* scale,
                           const uint16_t* x, float t, uint16_t* y, int d_in, int d_out, void* ws,
                           cudaStream_t stream) {
  QArgs k{};
  k.QT = QT; k.scale = scale; k.x = x; k.y = y; k.t = t; k.d_in = d_in; k.d_out = d_out;
  k.S = p.S; k.chunk = p.chunk;
  const size_t words = round_up((size_t)((d_in + 31) / 32) * 4, 16);
  k.words_bytes = (uint32_t)words;
  k.union_bytes = (uint32_t)std::max(2 * words, (size_t)kWarps * kTile * 4);
  k.counters = reinterpret_cast<unsigned*>(ws);
  k.partials = ws != nullptr ? reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + p.counters)
                             : nullptr;
  auto fn = fmt == kFmtInt8 ? q8_gemv_kernel<kFmtInt8> : q8_gemv_kernel<kFmtE4M3>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(fn, dim3(p.C, p.S), dim3(kThreads), p.smem, stream, k);
}

}  // namespace sig
