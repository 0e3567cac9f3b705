// Mask kernels: threshold, top-k and N:M selection, and row norms.
//
//  - threshold (TEAL README, Abstract; ">= t" as in RaNA Eqn. 12);
//  - top-k by magnitude ("Q-Sparse ..." rebuttal, A1 on MoE): a radix select on
//    the 16-bit magnitude key finds the k-th largest key K* and the number q of
//    entries equal to K* that still fit, then the q lowest-index ties are kept;
//  - N:M ("Flexible (N:M) Activation Sparsity", Methodology; Block Q-Sparse in
//    the Q-Sparse rebuttal, A2): per block of m, the n entries of largest key;
//  - row norms (||W^down_i|| of RaNA Eqn. 12), float64 accumulation.
#include "common.cuh"
#include "internal.h"

namespace sig {

namespace {

constexpr int kMaskThreads = 1024;

// Write the ascending kept-index list and the count from shared mask words.
// Every thread of the block calls it.
template <int BLOCK>
__device__ void compact_words(const uint32_t* words, int nwords, int32_t* idx, int32_t* nnz,
                              int* scratch) {
  const int tid = threadIdx.x;
  const int per = (nwords + BLOCK - 1) / BLOCK;
  const int w0 = min(nwords, tid * per), w1 = min(nwords, w0 + per);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(words[w]);
  int total;
  int r = block_exclusive_scan<BLOCK>(cnt, scratch, &total);
  if (idx != nullptr) {
    for (int w = w0; w < w1; ++w) {
      uint32_t bits = words[w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        idx[r++] = w * 32 + b;
      }
    }
  }
  if (nnz != nullptr && tid == 0) *nnz = total;
}

__global__ void __launch_bounds__(kMaskThreads)
threshold_compact_kernel(const uint16_t* __restrict__ x, int d, float t, uint32_t* mask_bits,
                         int32_t* idx, int32_t* nnz) {
  extern __shared__ __align__(16) uint32_t words[];
  __shared__ int scratch[kMaskThreads / 32 + 1];
  build_mask_words<kMaskThreads>(x, d, words,
                                 [&](uint16_t h, int) { return fabsf(h2f(h)) >= t; });
  __syncthreads();
  const int nwords = (d + 31) >> 5;
  for (int w = threadIdx.x; w < nwords; w += kMaskThreads) mask_bits[w] = words[w];
  compact_words<kMaskThreads>(words, nwords, idx, nnz, scratch);
}

// Suffix search over a histogram held one bin per thread (bins <= BLOCK):
// finds the bin b with above(b) < need <= above(b) + hist[b], where above(b)
// counts entries in bins > b.  Writes b and above(b) to out[0], out[1].
template <int BLOCK>
__device__ void find_bin(const int* hist, int nbins, int need, int* scratch, int* out) {
  const int tid = threadIdx.x;
  // reverse order so that an exclusive prefix is the count above
  const int b = nbins - 1 - tid;
  const int v = (tid < nbins) ? hist[b] : 0;
  int total;
  const int above = block_exclusive_scan<BLOCK>(v, scratch, &total);
  if (tid < nbins && above < need && need <= above + v) {
    out[0] = b;
    out[1] = above;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kMaskThreads)
topk_kernel(const uint16_t* __restrict__ x, int d, int k, uint32_t* mask_bits, int32_t* idx,
            int32_t* nnz) {
  extern __shared__ __align__(16) uint32_t dyn[];
  constexpr int kWarps = kMaskThreads / 32;
  __shared__ int hist[kMaskThreads];           // merged histogram
  __shared__ int whist[kWarps][256];           // per-warp histograms
  __shared__ int scratch[kWarps + 1];
  __shared__ int sel[2];
  __shared__ int tie_cut;                      // index after the q-th tie (exclusive)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwords = (d + 31) >> 5;
  uint32_t* gt = dyn;                          // key > K*
  uint32_t* eq = dyn + nwords;                 // key == K*

  if (k <= 0) {
    for (int w = tid; w < nwords; w += kMaskThreads) { mask_bits[w] = 0u; gt[w] = 0u; }
    __syncthreads();
    compact_words<kMaskThreads>(gt, nwords, idx, nnz, scratch);
    return;
  }

  // Pass 1: histogram of key >> 8 (keys are <= 0x7c01, so 125 bins used).
  for (int i = tid; i < kWarps * 256; i += kMaskThreads) (&whist[0][0])[i] = 0;
  __syncthreads();
  for (int i = tid; i < d; i += kMaskThreads) atomicAdd(&whist[warp][mag_key(x[i]) >> 8], 1);
  __syncthreads();
  if (tid < 256) {
    int s = 0;
    for (int w = 0; w < kWarps; ++w) s += whist[w][tid];
    hist[tid] = s;
  }
  __syncthreads();
  find_bin<kMaskThreads>(hist, 256, k, scratch, sel);
  const int hi_bin = sel[0], above_hi = sel[1];

  // Pass 2: histogram of the low byte within the chosen high bin.
  for (int i = tid; i < kWarps * 256; i += kMaskThreads) (&whist[0][0])[i] = 0;
  __syncthreads();
  for (int i = tid; i < d; i += kMaskThreads) {
    const uint32_t key = mag_key(x[i]);
    if ((int)(key >> 8) == hi_bin) atomicAdd(&whist[warp][key & 0xff], 1);
  }
  __syncthreads();
  if (tid < 256) {
    int s = 0;
    for (int w = 0; w < kWarps; ++w) s += whist[w][tid];
    hist[tid] = s;
  }
  __syncthreads();
  find_bin<kMaskThreads>(hist, 256, k - above_hi, scratch, sel);
  const uint32_t kstar = ((uint32_t)hi_bin << 8) | (uint32_t)sel[0];
  const int q = k - above_hi - sel[1];          // ties at K* to keep, 1..count(K*)

  // Pass 3: bitmaps of key > K* and key == K*.
  build_mask_words<kMaskThreads>(x, d, gt, [&](uint16_t h, int) { return mag_key(h) > kstar; });
  build_mask_words<kMaskThreads>(x, d, eq, [&](uint16_t h, int) { return mag_key(h) == kstar; });
  __syncthreads();

  // Keep the q lowest-index ties: find the word holding the q-th tie.
  {
    const int per = (nwords + kMaskThreads - 1) / kMaskThreads;
    const int w0 = min(nwords, tid * per), w1 = min(nwords, w0 + per);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(eq[w]);
    int total;
    int r = block_exclusive_scan<kMaskThreads>(cnt, scratch, &total);
    for (int w = w0; w < w1; ++w) {
      uint32_t bits = eq[w];
      uint32_t kept = 0;
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (r < q) kept |= 1u << b;
        ++r;
      }
      gt[w] |= kept;
    }
  }
  (void)tie_cut;
  (void)lane;
  __syncthreads();
  for (int w = tid; w < nwords; w += kMaskThreads) mask_bits[w] = gt[w];
  compact_words<kMaskThreads>(gt, nwords, idx, nnz, scratch);
}

// One thread per 32-entry mask word of one row (m divides 32, so the blocks of
// m never straddle a word).  Selection inside a block: the entry's rank is the
// number of entries with a larger (key, lower index) composite; keep rank < n.
template <int M>
__global__ void __launch_bounds__(256)
nm_mask_kernel(const uint16_t* __restrict__ X, int64_t rows, int d, int n, uint16_t* X_masked,
               uint32_t* mask_bits) {
  const int wpr = (d + 31) >> 5;
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= rows * wpr) return;
  const int64_t row = g / wpr;
  const int w = (int)(g % wpr);
  const int e0 = w * 32;
  const int cnt = min(32, d - e0);   // a multiple of M
  const uint16_t* src = X + row * (int64_t)d + e0;
  uint16_t v[32];
  if (cnt == 32) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(src) + q);
#pragma unroll
      for (int k = 0; k < 8; ++k) v[q * 8 + k] = lane_half(u, k);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = k < cnt ? src[k] : (uint16_t)0;
  }
  uint32_t bits = 0;
#pragma unroll
  for (int b0 = 0; b0 < 32; b0 += M) {
    if (b0 < cnt) {
      uint32_t comp[M];
#pragma unroll
      for (int j = 0; j < M; ++j) comp[j] = (mag_key(v[b0 + j]) << 5) | (uint32_t)(31 - j);
#pragma unroll
      for (int j = 0; j < M; ++j) {
        int rank = 0;
#pragma unroll
        for (int l = 0; l < M; ++l) rank += comp[l] > comp[j] ? 1 : 0;
        if (rank < n) bits |= 1u << (b0 + j);
      }
    }
  }
  if (mask_bits != nullptr) mask_bits[row * wpr + w] = bits;
  if (X_masked != nullptr) {
    uint16_t* dst = X_masked + row * (int64_t)d + e0;
    if (cnt == 32) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t p[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int a = q * 8 + 2 * k;
          const uint32_t lo = ((bits >> a) & 1u) ? v[a] : 0u;
          const uint32_t hi = ((bits >> (a + 1)) & 1u) ? v[a + 1] : 0u;
          p[k] = lo | (hi << 16);
        }
        reinterpret_cast<uint4*>(dst)[q] = make_uint4(p[0], p[1], p[2], p[3]);
      }
    } else {
      for (int k = 0; k < cnt; ++k) dst[k] = ((bits >> k) & 1u) ? v[k] : (uint16_t)0;
    }
  }
}

// One warp per row: sum of squares in float64, sqrt, one rounding to float32.
__global__ void __launch_bounds__(256)
row_norms_kernel(const uint16_t* __restrict__ WT, int64_t rows, int cols, float* norms) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint16_t* p = WT + row * (int64_t)cols;
  double s = 0.0;
  for (int c = lane * 8; c < cols; c += 256) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p + c));
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const double f = (double)h2f(lane_half(u, k));
      s = fma(f, f, s);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
  if (lane == 0) norms[row] = __double2float_rn(sqrt(s));
}

}  // namespace

cudaError_t launch_threshold_compact(const uint16_t* x, int d, float t, uint32_t* mask_bits,
                                     int32_t* idx, int32_t* nnz, cudaStream_t stream) {
  const size_t smem = (size_t)((d + 31) / 32) * 4 + 16;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(threshold_compact_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  threshold_compact_kernel<<<1, kMaskThreads, smem, stream>>>(x, d, t, mask_bits, idx, nnz);
  return cudaPeekAtLastError();
}

cudaError_t launch_topk(const uint16_t* x, int d, int k, uint32_t* mask_bits, int32_t* idx,
                        int32_t* nnz, cudaStream_t stream) {
  const size_t smem = (size_t)((d + 31) / 32) * 4 * 2 + 16;
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  topk_kernel<<<1, kMaskThreads, smem, stream>>>(x, d, k, mask_bits, idx, nnz);
  return cudaPeekAtLastError();
}

cudaError_t launch_nm_mask(const uint16_t* X, int64_t rows, int d, int n, int m,
                           uint16_t* X_masked, uint32_t* mask_bits, cudaStream_t stream) {
  const int64_t threads = rows * ((d + 31) / 32);
  if (threads == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  switch (m) {
    case 1: nm_mask_kernel<1><<<blocks, 256, 0, stream>>>(X, rows, d, n, X_masked, mask_bits); break;
    case 2: nm_mask_kernel<2><<<blocks, 256, 0, stream>>>(X, rows, d, n, X_masked, mask_bits); break;
    case 4: nm_mask_kernel<4><<<blocks, 256, 0, stream>>>(X, rows, d, n, X_masked, mask_bits); break;
    case 8: nm_mask_kernel<8><<<blocks, 256, 0, stream>>>(X, rows, d, n, X_masked, mask_bits); break;
    case 16: nm_mask_kernel<16><<<blocks, 256, 0, stream>>>(X, rows, d, n, X_masked, mask_bits); break;
    case 32: nm_mask_kernel<32><<<blocks, 256, 0, stream>>>(X, rows, d, n, X_masked, mask_bits); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaPeekAtLastError();
}

cudaError_t launch_row_norms(const uint16_t* WT, int64_t rows, int cols, float* norms,
                             cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  row_norms_kernel<<<blocks, 256, 0, stream>>>(WT, rows, cols, norms);
  return cudaPeekAtLastError();
}

}  // namespace sig
