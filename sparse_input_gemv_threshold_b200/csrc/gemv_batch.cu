// A few tokens, each with its own threshold mask, through one weight:
// y_b = W (m_b . x_b), m_b,i = |x_b,i| >= t, for b < B <= 16.
//
// The pages define the single-token product ("Adaptive Rank Allocation ...
// RaNA Adapters", rebuttal Q5.1: the columns of A that meet a zero mask entry
// are skipped) and leave the batched case with inconsistent masks open (Q6).
// Here one launch reads every weight row that ANY token keeps (the union of
// the masks) once from HBM and applies each token's own mask to it in
// registers: a row that token b drops contributes x_b,i = 0 to y_b.
//
// Launch shape: C x S CTAs of 256 threads (three per SM for up to 8 tokens,
// two for up to 16), a CTA owns a 256-output column tile and the union rows
// of its slice's 8-input groups (up to 8 tokens: slice s owns groups s, s+S,
// s+2S, ...; 16 tokens: a contiguous run of about 1/S of the groups):
//   1. one thread per group loads that group of every token's x (from L2,
//      all tokens' loads in flight together) and ORs their fp16 threshold
//      compares into a union byte; the popcounts are prefix-summed and the
//      union rows placed in ascending order, with the tokens' masked values
//      staged token-major (0 where a token drops the row);
//   2. for a column tile the work is a small dense contraction,
//      Y^T (256 outputs x 8 or 16 tokens) += W^T rows (256 x 16) . Xm per
//      step of 16 union rows, which the warp-level mma.m16n8k16 (fp16 in,
//      float32 accumulate) takes directly: the weight rows reach shared
//      memory through a multi-stage cp.async pipeline, each warp owns 32
//      output columns and runs every row of the slice, so warps never meet;
//   3. the CTA writes one partial per (token, column), and the last CTA to
//      arrive for the tile (one acquire-release atomic per CTA) adds the S
//      partials of every token in slice order and stores fp16.
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
  int B, d_in, d_out, S;
  uint32_t words_bytes;   // shared bytes of the union words (and again of their prefixes)
  uint32_t union_bytes;   // shared bytes of words + prefixes; the stages follow
  unsigned* counters;     // [C]
  float* partials;        // [S][B][d_out]
  uint32_t xg_stride;     // bytes per token of the slice's x groups kept in shared memory
                          // (0: not kept; the staging reads x from global memory)
};

// Shared-memory staging: weight rows padded to 528 bytes so that the
// transposing ldmatrix reads are free of bank conflicts; padding rows of a
// step and columns past d_out are written as zeros by plain shared stores.
// Tokens' masked values are staged token-major, padded rows apart likewise.

constexpr int kMmaStages = 5;
constexpr int kMmaRows = 16;                      // union rows per step
constexpr int kMmaRowBytes = kTile * 2 + 16;      // 528: padded shared row
constexpr int kMmaStageBytes = kMmaRows * kMmaRowBytes;
constexpr int kMmaChunk = 1024;                   // union rows staged per chunk
constexpr int kMmaXtStride = kMmaChunk * 2 + 16;  // bytes between token rows of staged values
// CTAs per SM for a token width (8 or 16 tokens per MMA column block):
// shared memory holds the tokens' staged values.
template <int TOK>
constexpr int mma_ctas_per_sm() { return TOK == 8 ? 3 : 2; }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
               "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

template <int TOK>
__global__ void __launch_bounds__(kThreads, mma_ctas_per_sm<TOK>())
batch_mma_kernel(const __grid_constant__ BArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int warp_tot[kWarps];
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x, s = blockIdx.y;
  const int d_in = a.d_in, d_out = a.d_out, S = a.S, B = a.B;
  constexpr int xt_stride = kMmaXtStride;

  uint32_t* words = reinterpret_cast<uint32_t*>(smem);
  int* wpre = reinterpret_cast<int*>(smem + a.words_bytes);
  unsigned char* stages = smem + a.union_bytes;
  int* sidx = reinterpret_cast<int*>(stages + kMmaStages * kMmaStageBytes);
  unsigned char* sxt = reinterpret_cast<unsigned char*>(sidx + kMmaChunk);   // TOK x kMmaXtStride bytes
  unsigned char* sxg = sxt + TOK * xt_stride;   // TOK x xg_stride bytes: the slice's x groups
  const uint32_t xg_stride = TOK == 16 ? a.xg_stride : 0u;   // kept for 16 tokens only

  pdl_trigger();
  pdl_wait();

  // ---- 1. union of the tokens' masks over this slice's groups ----------
  const __half2 th2 = thresh_half2(a.t);
  const float th = __half2float(__low2half(th2));
  const int ngroups = (d_in + 7) >> 3;
  // the slice's groups: for 16 tokens the contiguous run [g_lo, g_lo + K),
  // so that neighbouring threads load neighbouring 16-byte groups of each
  // token; for fewer tokens every S-th group from s, g = s + k * S.
  // Measured on B200 at 4096 -> 11008: 16 tokens 29.98 -> 27.99 us with the
  // contiguous run; 2 and 8 tokens 0.3 us slower with it (not taken)
  constexpr bool kContig = TOK == 16;
  const int g_lo = kContig ? (int)(((long long)s * ngroups) / S) : s;
  const int g_step = kContig ? 1 : S;
  const int K = kContig ? (int)(((long long)(s + 1) * ngroups) / S) - g_lo
                        : (s < ngroups ? (ngroups - 1 - s) / S + 1 : 0);
  const int nwords = (K + 3) >> 2;
  // one thread per group: every token's loads in flight together; for 16
  // tokens the groups are kept in shared memory for the staging
  uint8_t* wbytes = reinterpret_cast<uint8_t*>(words);
  for (int k = tid; k < nwords * 4; k += kThreads) {
    uint32_t u = 0;
    if (k < K) {
      const int e0 = (g_lo + k * g_step) * 8;
      uint4 v[TOK];
#pragma unroll
      for (int b = 0; b < TOK; ++b)
        v[b] = b < B ? __ldg(reinterpret_cast<const uint4*>(a.X + (size_t)b * d_in + e0))
                     : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int b = 0; b < TOK; ++b)
        if (b < B) {
          u |= thresh_bits8(v[b], th2);
          if (xg_stride != 0u) *reinterpret_cast<uint4*>(sxg + b * xg_stride + k * 16) = v[b];
        }
    }
    wbytes[k] = (uint8_t)u;
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

  // ---- 2. the contraction over the union rows ---------------------------
  const int tile0 = c * kTile;
  constexpr int NT = TOK / 8;               // n8 tiles of tokens
  float acc[2][NT][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[mt][nt][k] = 0.f;

  // this thread's two 16-byte pieces of every staged step (row, 16-byte column)
  int cp_row[2], cp_col[2];
  bool cp_in[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int q = tid + kThreads * e;
    cp_row[e] = q >> 5;
    cp_col[e] = q & 31;
    cp_in[e] = tile0 + cp_col[e] * 8 < d_out;
  }
  // rows past the chunk's end and columns past d_out are zeros in shared memory
  auto issue_step = [&](int step, int cn) {
    unsigned char* st = stages + (step % kMmaStages) * kMmaStageBytes;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = step * kMmaRows + cp_row[e];
      unsigned char* dst = st + cp_row[e] * kMmaRowBytes + cp_col[e] * 16;
      if (j < cn && cp_in[e])
        cp_async16(smem_u32(dst), a.WT + (size_t)sidx[j] * d_out + tile0 + cp_col[e] * 8);
      else
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
  };

  for (int cb = 0; cb < total; cb += kMmaChunk) {
    const int c_lo = cb, c_hi = min(total, cb + kMmaChunk), cn = c_hi - c_lo;
    const int nsteps = (cn + kMmaRows - 1) / kMmaRows;
    if (cb > 0) __syncthreads();   // every read of the previous chunk is over
    // union rows of this chunk, and the tokens' masked values token-major
    for (int w = warp; w < nwords; w += kWarps) {
      const int base = wpre[w];
      if (base >= c_hi) break;                       // uniform across the warp
      const uint32_t bits = words[w];
      const int rk = base + __popc(bits & ((1u << lane) - 1u));
      if (((bits >> lane) & 1u) && rk >= c_lo && rk < c_hi) {
        const int kg = w * 4 + (lane >> 3);              // the slice's group of this row
        const int i = (g_lo + kg * g_step) * 8 + (lane & 7);
        const int j = rk - c_lo;
        sidx[j] = i;
#pragma unroll
        for (int b = 0; b < TOK; ++b) {
          uint16_t h = 0;
          if (b < B) {
            h = xg_stride != 0u
                    ? *reinterpret_cast<const uint16_t*>(sxg + b * xg_stride + kg * 16 + (lane & 7) * 2)
                    : a.X[(size_t)b * d_in + i];
            if (!(fabsf(h2f(h)) >= th)) h = 0;
          }
          *reinterpret_cast<uint16_t*>(sxt + b * xt_stride + j * 2) = h;
        }
      }
    }
    // zero values for the padding rows of the last step
    for (int q = tid; q < TOK * kMmaRows; q += kThreads) {
      const int j = cn + (q % kMmaRows);
      if (j < nsteps * kMmaRows) *reinterpret_cast<uint16_t*>(sxt + (q / kMmaRows) * xt_stride + j * 2) = 0;
    }
    __syncthreads();

#pragma unroll
    for (int st = 0; st < kMmaStages - 1; ++st) {
      if (st < nsteps) issue_step(st, cn);
      cp_async_commit();
    }
    for (int ks = 0; ks < nsteps; ++ks) {
      cp_async_wait<kMmaStages - 2>();
      __syncthreads();                 // step ks has landed; step ks-1's stage is free
      if (ks + kMmaStages - 1 < nsteps) issue_step(ks + kMmaStages - 1, cn);
      cp_async_commit();
      __syncwarp();                    // the fragment loads and MMAs below are warp-wide
      const unsigned char* stg = stages + (ks % kMmaStages) * kMmaStageBytes;
      uint32_t bf[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int n = nt * 8 + (lane & 7), kh = (lane >> 3) & 1;
        ldsm_x2(bf[nt], smem_u32(sxt + n * xt_stride + (ks * kMmaRows + kh * 8) * 2));
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int q = lane >> 3, r = lane & 7;
        const int m = warp * 32 + mt * 16 + (q & 1) * 8;
        uint32_t af[4];
        ldsm_x4_trans(af, smem_u32(stg + ((q >> 1) * 8 + r) * kMmaRowBytes + m * 2));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816(acc[mt][nt], af, bf[nt]);
      }
    }
    cp_async_wait<0>();
  }

  // ---- 3. this CTA's partials; the last arriver finishes the tile -------
  const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int col = tile0 + warp * 32 + mt * 16 + g + h * 8;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int n = nt * 8 + t4 * 2 + e;
          if (col < d_out && n < B) {
            if (S == 1)
              a.Y[(size_t)n * d_out + col] = f2h_rn(acc[mt][nt][h * 2 + e]);
            else
              a.partials[((size_t)s * B + n) * d_out + col] = acc[mt][nt][h * 2 + e];
          }
        }
      }
  if (S == 1) return;
  __syncthreads();
  if (tid == 0) s_last = atomic_add_acq_rel_gpu(a.counters + c, 1u) == (unsigned)(S - 1);
  __syncthreads();
  if (!s_last) return;
  const int colr = tile0 + tid;
  if (colr < d_out) {
    // eight tokens' partials of a slice in flight together, two slices at a
    // time; each token's sum still runs in slice order
    const size_t slice_stride = (size_t)B * d_out;
    const float* pp = a.partials + colr;
#pragma unroll
    for (int b0 = 0; b0 < TOK; b0 += 8) {
      float sum[8];
#pragma unroll
      for (int b = 0; b < 8; ++b) sum[b] = 0.f;
#pragma unroll 2
      for (int q = 0; q < S; ++q) {
        float v[8];
#pragma unroll
        for (int b = 0; b < 8; ++b)
          v[b] = b0 + b < B ? __ldcg(pp + q * slice_stride + (size_t)(b0 + b) * d_out) : 0.f;
#pragma unroll
        for (int b = 0; b < 8; ++b) sum[b] += v[b];
      }
#pragma unroll
      for (int b = 0; b < 8; ++b)
        if (b0 + b < B) a.Y[(size_t)(b0 + b) * d_out + colr] = f2h_rn(sum[b]);
    }
  }
  if (tid == 0) a.counters[c] = 0u;  // ready for the next call on this workspace
}

size_t round_up(size_t v, size_t al) { return (v + al - 1) / al * al; }

// Bytes per token of a slice's x groups kept in shared memory from the union
// step for the staging of the masked values (16 per group): for 16-token
// launches whose groups take at most 48 KB; 0 otherwise (the staging then
// reads x from global memory).  Measured on B200 at 4096 -> 11008: 16 tokens
// 30.98 -> 29.91 us; 8 tokens 23.95 -> 24.71 us (not taken).
uint32_t xg_stride_bytes(int64_t d_in, int S, int tok) {
  const int64_t kmax = ((d_in + 7) / 8 + S - 1) / S;
  return tok == 16 && tok * kmax * 16 <= (48 << 10) ? (uint32_t)(kmax * 16) : 0u;
}

}  // namespace

GemvPlan plan_gemv_batch(int64_t d_in, int64_t d_out, int B) {
  GemvPlan p{};
  p.C = (int)((d_out + kTile - 1) / kTile);
  const int tok = B <= 8 ? 8 : 16;
  const int cps = tok == 8 ? mma_ctas_per_sm<8>() : mma_ctas_per_sm<16>();
  p.S = std::max(1, std::min(32, (kNumSMs * cps) / std::max(1, p.C)));
  p.chunk = kMmaChunk;
  const size_t words = round_up((size_t)((d_in + 31) / 32) * 4, 16);
  p.smem = 2 * words + (size_t)kMmaStages * kMmaStageBytes + (size_t)kMmaChunk * 4 +
           (size_t)tok * kMmaXtStride;
  p.smem += (size_t)tok * xg_stride_bytes(d_in, p.S, tok);
  p.counters = p.S > 1 ? round_up((size_t)p.C * 4, 256) : 0;
  p.partials = p.S > 1 ? round_up((size_t)p.S * B * d_out * 4, 256) : 0;
  return p;
}

cudaError_t launch_gemv_batch(const GemvPlan& p, const uint16_t* WT, const uint16_t* X, uint16_t* Y,
                              int B, int d_in, int d_out, float t, void* ws, cudaStream_t stream) {
  BArgs k{};
  k.WT = WT; k.X = X; k.Y = Y; k.t = t; k.B = B; k.d_in = d_in; k.d_out = d_out; k.S = p.S;
  k.xg_stride = xg_stride_bytes(d_in, p.S, B <= 8 ? 8 : 16);
  const size_t words = round_up((size_t)((d_in + 31) / 32) * 4, 16);
  k.words_bytes = (uint32_t)words;
  k.union_bytes = (uint32_t)(2 * words);
  k.counters = reinterpret_cast<unsigned*>(ws);
  k.partials = ws != nullptr ? reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + p.counters)
                             : nullptr;
  auto fn = B <= 8 ? batch_mma_kernel<8> : batch_mma_kernel<16>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(fn, dim3(p.C, p.S), dim3(kThreads), p.smem, stream, k);
}

}  // namespace sig
