// Mask kernels: threshold, top-k and N:M selection, and row norms.
//
//  - threshold (TEAL README, Abstract; ">= t" as in RaNA Eqn. 12);
//  - top-k by magnitude ("Q-Sparse ..." rebuttal, A1 on MoE): a radix select on
//    the 16-bit magnitude key, spread over a thread-block cluster, finds the
//    k-th largest key K* and the number q of entries equal to K* that still
//    fit, then the q lowest-index ties are kept;
//  - N:M ("Flexible (N:M) Activation Sparsity", Methodology; Block Q-Sparse in
//    the Q-Sparse rebuttal, A2): per block of m, the n entries of largest key;
//  - row norms (||W^down_i|| of RaNA Eqn. 12), float64 accumulation.
#include "common.cuh"
#include "internal.h"
#include "nm_select.cuh"

#include <cooperative_groups.h>

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

  pdl_trigger();
  pdl_wait();
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

// Count key `bin` into a per-warp histogram; lanes with equal bins add once.
__device__ __forceinline__ void warp_hist_add(int* hist, uint32_t bin, bool active) {
  const unsigned grp = __match_any_sync(kFull, active ? bin : 0xffffffffu);
  const int lane = threadIdx.x & 31;
  if (active && lane == __ffs(grp) - 1) atomicAdd(&hist[bin], __popc(grp));
}

// Radix select on the 16-bit magnitude key, spread over a cluster of
// kTopkCluster CTAs.  CTA q owns the keys [q*chunk, (q+1)*chunk) (whole mask
// words) and stages them in its shared memory.
//   pass 1  local histogram of key >> 8; after a cluster barrier every CTA sums
//           all CTAs' histograms through distributed shared memory and finds
//           the high byte of K* (the k-th largest key) the same way;
//   pass 2  the same for the low byte among keys with that high byte, giving
//           K* and q = the number of entries equal to K* that still fit;
//   then    local bitmaps key > K* and key == K*; a CTA's first tie rank and
//           its first output slot are the counts published by lower-ranked
//           CTAs, so the q lowest-index ties are kept and the index list comes
//           out ascending.
constexpr int kTopkCluster = 8;

__global__ void __launch_bounds__(kMaskThreads)
topk_cluster_kernel(const uint16_t* __restrict__ x, int d, int k, int chunk, uint32_t* mask_bits,
                    int32_t* idx, int32_t* nnz) {
  namespace cg = cooperative_groups;
  extern __shared__ __align__(16) unsigned char dyn_raw[];
  constexpr int kWarps = kMaskThreads / 32;
  __shared__ int whist[kWarps][256];           // per-warp histograms
  __shared__ int hist1[256], hist2[256];       // this CTA's pass-1 / pass-2 histograms
  __shared__ int ghist[256];                   // cluster-wide histogram
  __shared__ int scratch[kWarps + 1];
  __shared__ int sel[2];
  __shared__ int pub[2];                       // [0] ties here, [1] kept here

  cg::cluster_group cluster = cg::this_cluster();
  const int cq = (int)cluster.block_rank();
  pdl_trigger();
  pdl_wait();

  const int tid = threadIdx.x, warp = tid >> 5;
  const int e_begin = cq * chunk;
  const int nloc = max(0, min(d, e_begin + chunk) - e_begin);
  const int nwl = (nloc + 31) >> 5;             // local words holding keys
  const int w_begin = e_begin >> 5;             // first global mask word of this CTA
  uint16_t* keys = reinterpret_cast<uint16_t*>(dyn_raw);
  uint32_t* gt = reinterpret_cast<uint32_t*>(dyn_raw + (size_t)chunk * 2);
  uint32_t* eq = gt + (chunk >> 5);

  if (k <= 0) {
    for (int w = tid; w < nwl; w += kMaskThreads) mask_bits[w_begin + w] = 0u;
    if (cq == 0 && tid == 0) *nnz = 0;
    return;
  }

  // Stage the keys of this CTA's range (zero padding is never counted).
  for (int e0 = tid * 8; e0 < nwl * 32; e0 += kMaskThreads * 8) {
    const int g0 = e_begin + e0;
    uint32_t p[4];
    if (g0 + 8 <= d) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + g0));
#pragma unroll
      for (int q = 0; q < 4; ++q)
        p[q] = mag_key(lane_half(v, 2 * q)) | (mag_key(lane_half(v, 2 * q + 1)) << 16);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t lo = g0 + 2 * q < d ? mag_key(x[g0 + 2 * q]) : 0u;
        const uint32_t hi = g0 + 2 * q + 1 < d ? mag_key(x[g0 + 2 * q + 1]) : 0u;
        p[q] = lo | (hi << 16);
      }
    }
    *reinterpret_cast<uint4*>(keys + e0) = make_uint4(p[0], p[1], p[2], p[3]);
  }
  for (int i = tid; i < kWarps * 256; i += kMaskThreads) (&whist[0][0])[i] = 0;
  __syncthreads();

  // ---- pass 1: high byte ----
  for (int i0 = 0; i0 < nloc; i0 += kMaskThreads) {
    const int i = i0 + tid;
    const bool ok = i < nloc;
    warp_hist_add(whist[warp], ok ? (uint32_t)keys[i] >> 8 : 0u, ok);
  }
  __syncthreads();
  if (tid < 256) {
    int v = 0;
    for (int w = 0; w < kWarps; ++w) { v += whist[w][tid]; whist[w][tid] = 0; }
    hist1[tid] = v;
  }
  cluster.sync();
  if (tid < 256) {
    int v = 0;
    for (int r = 0; r < kTopkCluster; ++r) v += cluster.map_shared_rank(hist1, r)[tid];
    ghist[tid] = v;
  }
  __syncthreads();
  find_bin<kMaskThreads>(ghist, 256, k, scratch, sel);
  const int hi_bin = sel[0], above_hi = sel[1];

  // ---- pass 2: low byte among keys with that high byte ----
  for (int i0 = 0; i0 < nloc; i0 += kMaskThreads) {
    const int i = i0 + tid;
    const uint32_t key = i < nloc ? keys[i] : 0u;
    const bool ok = i < nloc && (int)(key >> 8) == hi_bin;
    warp_hist_add(whist[warp], key & 0xffu, ok);
  }
  __syncthreads();
  if (tid < 256) {
    int v = 0;
    for (int w = 0; w < kWarps; ++w) v += whist[w][tid];
    hist2[tid] = v;
  }
  cluster.sync();
  if (tid < 256) {
    int v = 0;
    for (int r = 0; r < kTopkCluster; ++r) v += cluster.map_shared_rank(hist2, r)[tid];
    ghist[tid] = v;
  }
  __syncthreads();
  find_bin<kMaskThreads>(ghist, 256, k - above_hi, scratch, sel);
  const uint32_t kstar = ((uint32_t)hi_bin << 8) | (uint32_t)sel[0];
  const int q_ties = k - above_hi - sel[1];     // ties at K* to keep, cluster-wide

  // ---- bitmaps of key > K* and key == K* for this CTA's words ----
  for (int w = tid; w < nwl; w += kMaskThreads) {
    const uint4* kp = reinterpret_cast<const uint4*>(keys + w * 32);
    uint32_t g = 0, e = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = kp[c];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t key = lane_half(v, j);
        const bool in = w * 32 + c * 8 + j < nloc;
        g |= (in && key > kstar ? 1u : 0u) << (c * 8 + j);
        e |= (in && key == kstar ? 1u : 0u) << (c * 8 + j);
      }
    }
    gt[w] = g;
    eq[w] = e;
  }
  __syncthreads();

  // ---- ties: this CTA's first tie rank is the ties of lower-ranked CTAs ----
  const int per = (nwl + kMaskThreads - 1) / kMaskThreads;
  const int w0 = min(nwl, tid * per), w1 = min(nwl, w0 + per);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(eq[w]);
  int ties_here;
  int r = block_exclusive_scan<kMaskThreads>(cnt, scratch, &ties_here);
  if (tid == 0) pub[0] = ties_here;
  cluster.sync();
  int tie_base = 0;
  for (int rr = 0; rr < cq; ++rr) tie_base += cluster.map_shared_rank(pub, rr)[0];
  r += tie_base;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = eq[w], kept = 0;
    while (bits && r < q_ties) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      kept |= 1u << b;
      ++r;
    }
    gt[w] |= kept;
  }
  __syncthreads();

  // ---- output: mask words and the ascending index list ----
  cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(gt[w]);
  int kept_here;
  int o = block_exclusive_scan<kMaskThreads>(cnt, scratch, &kept_here);
  if (tid == 0) pub[1] = kept_here;
  cluster.sync();
  int out_base = 0;
  for (int rr = 0; rr < cq; ++rr) out_base += cluster.map_shared_rank(pub, rr)[1];
  o += out_base;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = gt[w];
    mask_bits[w_begin + w] = bits;
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      idx[o++] = e_begin + w * 32 + b;
    }
  }
  if (cq == 0 && tid == 0) *nnz = k;
  cluster.sync();   // no CTA leaves while another may still read its shared memory
}

// One thread per 32-entry mask word of one row (m divides 32, so blocks of m
// never straddle a word).  Inside a block the entries are ranked by the
// composite (magnitude key << 5 | (31 - position)): unique, larger magnitude
// first, lower index first among equal magnitudes.
template <int M>
__global__ void __launch_bounds__(256)
nm_mask_kernel(const uint16_t* __restrict__ X, int64_t rows, int d, int n, uint16_t* X_masked,
               uint32_t* mask_bits) {
  const int wpr = (d + 31) >> 5;
  pdl_trigger();
  pdl_wait();
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= rows * wpr) return;
  const int64_t row = g / wpr;
  const int w = (int)(g % wpr);
  const int e0 = w * 32;
  const int cnt = min(32, d - e0);   // a multiple of 8 and of M
  const uint16_t* src = X + row * (int64_t)d + e0;
  uint4 q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    q[i] = i * 8 < cnt ? __ldg(reinterpret_cast<const uint4*>(src) + i) : make_uint4(0, 0, 0, 0);
  const uint32_t bits = nm_word_bits<M>(q, n, cnt);
  if (mask_bits != nullptr) mask_bits[row * wpr + w] = bits;
  if (X_masked != nullptr) {
    uint16_t* dst = X_masked + row * (int64_t)d + e0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (i * 8 < cnt) reinterpret_cast<uint4*>(dst)[i] = nm_apply(q[i], bits, i);
  }
}

// One warp per row: sum of squares in float64, sqrt, one rounding to float32.
__global__ void __launch_bounds__(256)
row_norms_kernel(const uint16_t* __restrict__ WT, int64_t rows, int cols, float* norms) {
  pdl_trigger();
  pdl_wait();
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
  return launch_pdl(threshold_compact_kernel, dim3(1), dim3(kMaskThreads), smem, stream, x, d, t,
                    mask_bits, idx, nnz);
}

cudaError_t launch_topk(const uint16_t* x, int d, int k, uint32_t* mask_bits, int32_t* idx,
                        int32_t* nnz, cudaStream_t stream) {
  // whole words per CTA, and a multiple of 8 keys for the 16-byte staging loads
  const int chunk = ((d + kTopkCluster - 1) / kTopkCluster + 31) / 32 * 32;
  const size_t smem = (size_t)chunk * 2 + (size_t)(chunk / 32) * 8;
  cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kTopkCluster);
  cfg.blockDim = dim3(kMaskThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kTopkCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel, x, d, k, chunk, mask_bits, idx, nnz);
}

cudaError_t launch_nm_mask(const uint16_t* X, int64_t rows, int d, int n, int m,
                           uint16_t* X_masked, uint32_t* mask_bits, cudaStream_t stream) {
  const int64_t threads = rows * ((d + 31) / 32);
  if (threads == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  cudaError_t e = cudaSuccess;
  switch (m) {
    case 1: e = launch_pdl(nm_mask_kernel<1>, dim3(blocks), dim3(256), 0, stream, X, rows, d, n, X_masked, mask_bits); break;
    case 2: e = launch_pdl(nm_mask_kernel<2>, dim3(blocks), dim3(256), 0, stream, X, rows, d, n, X_masked, mask_bits); break;
    case 4: e = launch_pdl(nm_mask_kernel<4>, dim3(blocks), dim3(256), 0, stream, X, rows, d, n, X_masked, mask_bits); break;
    case 8: e = launch_pdl(nm_mask_kernel<8>, dim3(blocks), dim3(256), 0, stream, X, rows, d, n, X_masked, mask_bits); break;
    case 16: e = launch_pdl(nm_mask_kernel<16>, dim3(blocks), dim3(256), 0, stream, X, rows, d, n, X_masked, mask_bits); break;
    case 32: e = launch_pdl(nm_mask_kernel<32>, dim3(blocks), dim3(256), 0, stream, X, rows, d, n, X_masked, mask_bits); break;
    default: return cudaErrorInvalidValue;
  }
  return e;
}

cudaError_t launch_row_norms(const uint16_t* WT, int64_t rows, int cols, float* norms,
                             cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  return launch_pdl(row_norms_kernel, dim3(blocks), dim3(256), 0, stream, WT, rows, cols, norms);
}

}  // namespace sig
