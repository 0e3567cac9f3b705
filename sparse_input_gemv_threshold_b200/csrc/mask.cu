// Mask kernels: threshold, top-k and N:M selection, and row norms.
//
//  - threshold (TEAL README, Abstract; ">= t" as in RaNA Eqn. 12);
//  - top-k by magnitude ("Q-Sparse ..." rebuttal, A1 on MoE): a radix select on
//    the 16-bit magnitude key (in one CTA for short vectors, spread over a
//    thread-block cluster for long ones) finds the k-th largest key K* and the number
//    q of entries equal to K* that still fit, then the q lowest-index ties are
//    kept;
//  - N:M ("Flexible (N:M) Activation Sparsity", Methodology; Block Q-Sparse in
//    the Q-Sparse rebuttal, A2): per block of m, the n entries of largest key;
//  - row norms (||W^down_i|| of RaNA Eqn. 12), float64 accumulation.
#include "common.cuh"
#include "internal.h"
#include "nm_ex.h"
#include "nm_pack.cuh"
#include "nm_select.cuh"

#include <cooperative_groups.h>
#include <type_traits>

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

// Stage the magnitude keys of x[e_begin, e_begin + n) into keys[0, n_pad)
// (n_pad a multiple of 32, slots past n get key 0), four 16-byte loads in
// flight per thread; e_begin is a multiple of 32.
template <int BLOCK>
__device__ __forceinline__ void stage_keys(const uint16_t* __restrict__ x, int e_begin, int n,
                                           int n_pad, uint16_t* keys) {
  constexpr int kStage = 4;
  const int tid = threadIdx.x;
  for (int base = 0; base < n_pad; base += BLOCK * 8 * kStage) {
    uint4 v[kStage];
#pragma unroll
    for (int u = 0; u < kStage; ++u) {
      const int e0 = base + (u * BLOCK + tid) * 8;
      v[u] = e0 + 8 <= n ? __ldg(reinterpret_cast<const uint4*>(x + e_begin + e0))
                         : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kStage; ++u) {
      const int e0 = base + (u * BLOCK + tid) * 8;
      if (e0 >= n_pad) break;
      uint32_t p[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t lo, hi;
        if (e0 + 8 <= n) {
          lo = mag_key(lane_half(v[u], 2 * q));
          hi = mag_key(lane_half(v[u], 2 * q + 1));
        } else {
          lo = e0 + 2 * q < n ? mag_key(x[e_begin + e0 + 2 * q]) : 0u;
          hi = e0 + 2 * q + 1 < n ? mag_key(x[e_begin + e0 + 2 * q + 1]) : 0u;
        }
        p[q] = lo | (hi << 16);
      }
      *reinterpret_cast<uint4*>(keys + e0) = make_uint4(p[0], p[1], p[2], p[3]);
    }
  }
}

// Histogram of the high digit (key >> 5, 1024 bins) of keys[0, n), two keys
// per shared load.
template <int BLOCK>
__device__ __forceinline__ void hist_high_digit(const uint16_t* keys, int n, int* hist) {
  const uint32_t* key2 = reinterpret_cast<const uint32_t*>(keys);
  for (int i2 = threadIdx.x; 2 * i2 < n; i2 += BLOCK) {
    const uint32_t pr = key2[i2];
    atomicAdd(&hist[(pr & 0xffffu) >> 5], 1);
    if (2 * i2 + 1 < n) atomicAdd(&hist[pr >> 21], 1);
  }
}

// Histogram of the low digit (key & 31, 32 bins) of the keys whose high digit
// is hi_bin.
template <int BLOCK>
__device__ __forceinline__ void hist_low_digit(const uint16_t* keys, int n, int hi_bin, int* hist) {
  const uint32_t* key2 = reinterpret_cast<const uint32_t*>(keys);
  for (int i2 = threadIdx.x; 2 * i2 < n; i2 += BLOCK) {
    const uint32_t pr = key2[i2];
    const uint32_t lo = pr & 0xffffu, hi = pr >> 16;
    if ((int)(lo >> 5) == hi_bin) atomicAdd(&hist[lo & 31u], 1);
    if (2 * i2 + 1 < n && (int)(hi >> 5) == hi_bin) atomicAdd(&hist[hi & 31u], 1);
  }
}

// Bitmaps key > kstar and key == kstar of keys[0, n): one word per warp, one
// key per lane.
template <int BLOCK>
__device__ __forceinline__ void bitmaps_gt_eq(const uint16_t* keys, int n, uint32_t kstar,
                                              uint32_t* gt, uint32_t* eq) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (n + 31) >> 5;
  for (int w = warp; w < nw; w += BLOCK / 32) {
    const int i = w * 32 + lane;
    const uint32_t key = keys[i];
    const uint32_t g = __ballot_sync(kFull, i < n && key > kstar);
    const uint32_t e = __ballot_sync(kFull, i < n && key == kstar);
    if (lane == 0) {
      gt[w] = g;
      eq[w] = e;
    }
  }
}

// The index list entries of nw words, one word per warp: word w's kept bits
// go to idx[wpre[w] ...] in ascending order (index = e_begin + 32 w + bit).
template <int BLOCK>
__device__ __forceinline__ void write_index_list(const uint32_t* gt, const int* wpre, int nw,
                                                 int e_begin, int32_t* idx) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int w = warp; w < nw; w += BLOCK / 32) {
    const uint32_t bits = gt[w];
    if ((bits >> lane) & 1u)
      idx[wpre[w] + __popc(bits & ((1u << lane) - 1u))] = e_begin + w * 32 + lane;
  }
}

// Top-k in one CTA for d <= kTopkBlockMaxD: the keys sit in shared memory and
// a two-digit radix select finds K*, the k-th largest magnitude key.  Keys are
// below 2^15, so the high digit (key >> 5) has 1024 bins, one per thread, and
// the low digit 32.
//   pass 1  histogram of key >> 5 (shared atomics), suffix scan: the high
//           digit of K* and the count of keys above its bin;
//   pass 2  histogram of key & 31 among keys in that bin: K* and q = the
//           number of entries equal to K* that still fit;
//   then    bitmaps key > K* and key == K* (a ballot per word); the q
//           lowest-index ties join the first; a scan of the words' popcounts
//           gives each word's first slot, and the warps write the ascending
//           index list one word at a time (contiguous stores).
// The packed scan below holds two counts of at most d in 16-bit halves.
constexpr int kTopkBlockMaxD = 32767;
// Up to this d one CTA is faster than the cluster (measured on B200: 5.8 vs
// 7.2 us at d = 8192, 11.9 vs 8.1 us at d = 28672).
constexpr int kTopkBlockUpTo = 12288;

__global__ void __launch_bounds__(kMaskThreads)
topk_block_kernel(const uint16_t* __restrict__ x, int d, int k, uint32_t* mask_bits, int32_t* idx,
                  int32_t* nnz) {
  extern __shared__ __align__(16) unsigned char dyn_raw[];
  __shared__ int hist[1024];
  __shared__ int scratch[kMaskThreads / 32 + 1];
  __shared__ int sel[2];
  const int tid = threadIdx.x;
  const int nw = (d + 31) >> 5;
  uint16_t* keys = reinterpret_cast<uint16_t*>(dyn_raw);            // nw * 32 keys
  uint32_t* gt = reinterpret_cast<uint32_t*>(dyn_raw + (size_t)nw * 64);
  int* wpre = reinterpret_cast<int*>(gt + nw);                       // ties bits, then prefixes
  uint32_t* eq = reinterpret_cast<uint32_t*>(wpre);

  pdl_trigger();
  pdl_wait();
  if (k <= 0) {
    for (int w = tid; w < nw; w += kMaskThreads) mask_bits[w] = 0u;
    if (tid == 0) *nnz = 0;
    return;
  }
  hist[tid] = 0;
  stage_keys<kMaskThreads>(x, 0, d, nw * 32, keys);
  __syncthreads();

  // ---- pass 1: high digit ----
  hist_high_digit<kMaskThreads>(keys, d, hist);
  __syncthreads();
  find_bin<kMaskThreads>(hist, 1024, k, scratch, sel);
  const int hi_bin = sel[0], above_hi = sel[1];
  hist[tid] = 0;
  __syncthreads();

  // ---- pass 2: low digit among keys in that bin ----
  hist_low_digit<kMaskThreads>(keys, d, hi_bin, hist);
  __syncthreads();
  find_bin<kMaskThreads>(hist, 32, k - above_hi, scratch, sel);
  const uint32_t kstar = ((uint32_t)hi_bin << 5) | (uint32_t)sel[0];
  const int q_ties = k - above_hi - sel[1];

  bitmaps_gt_eq<kMaskThreads>(keys, d, kstar, gt, eq);
  __syncthreads();

  // ---- thread-contiguous words: one packed scan of (ties, keys above) ----
  const int per = (nw + kMaskThreads - 1) / kMaskThreads;
  const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
  int gcnt = 0, ecnt = 0;
  for (int w = w0; w < w1; ++w) {
    gcnt += __popc(gt[w]);
    ecnt += __popc(eq[w]);
  }
  int packed_total;
  const int packed = block_exclusive_scan<kMaskThreads>((ecnt << 16) | gcnt, scratch, &packed_total);
  const int g_excl = packed & 0xffff, e_excl = packed >> 16;
  // the q lowest-index ties join the kept set; this thread's first slot
  int r_tie = e_excl;
  int o = g_excl + min(max(q_ties, 0), e_excl);
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = eq[w], kept = 0;
    while (bits && r_tie < q_ties) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      kept |= 1u << b;
      ++r_tie;
    }
    const uint32_t gw = gt[w] | kept;
    gt[w] = gw;
    wpre[w] = o;
    o += __popc(gw);
  }
  __syncthreads();

  for (int w = tid; w < nw; w += kMaskThreads) mask_bits[w] = gt[w];
  write_index_list<kMaskThreads>(gt, wpre, nw, 0, idx);
  if (tid == 0) *nnz = k;
}

// Radix select on the 16-bit magnitude key, spread over a cluster of
// kTopkCluster CTAs.  CTA c owns the keys [c*chunk, (c+1)*chunk) (whole mask
// words) and stages them in its shared memory.
//   pass 1  local histogram of the high digit; after a cluster barrier every
//           CTA sums all CTAs' histograms through distributed shared memory
//           and finds the high digit of K* (the k-th largest key);
//   pass 2  the same for the low digit among keys with that high digit,
//           giving K* and q = the number of entries equal to K* that still fit;
//   then    local bitmaps key > K* and key == K*; each CTA publishes its
//           counts of both, and from the counts of lower-ranked CTAs finds
//           its first tie rank and its first output slot, so the q
//           lowest-index ties are kept and the index list comes out
//           ascending.  The last cluster barrier is split: a CTA arrives once
//           it has read the others' shared memory and waits before it exits.
constexpr int kTopkCluster = 8;

__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(kMaskThreads)
topk_cluster_kernel(const uint16_t* __restrict__ x, int d, int k, int chunk, uint32_t* mask_bits,
                    int32_t* idx, int32_t* nnz) {
  namespace cg = cooperative_groups;
  extern __shared__ __align__(16) unsigned char dyn_raw[];
  __shared__ int hist1[1024], ghist[1024];
  __shared__ int hist2[32];
  __shared__ int scratch[kMaskThreads / 32 + 1];
  __shared__ int sel[2];
  __shared__ int pub[2];                       // [0] ties at K* here, [1] keys above K* here

  cg::cluster_group cluster = cg::this_cluster();
  const int cq = (int)cluster.block_rank();
  pdl_trigger();
  pdl_wait();

  const int tid = threadIdx.x;
  const int e_begin = cq * chunk;
  const int nloc = max(0, min(d, e_begin + chunk) - e_begin);
  const int nwl = (nloc + 31) >> 5;             // local words holding keys
  const int w_begin = e_begin >> 5;             // first global mask word of this CTA
  uint16_t* keys = reinterpret_cast<uint16_t*>(dyn_raw);
  uint32_t* gt = reinterpret_cast<uint32_t*>(dyn_raw + (size_t)chunk * 2);
  int* wpre = reinterpret_cast<int*>(gt + (chunk >> 5));
  uint32_t* eq = reinterpret_cast<uint32_t*>(wpre);

  if (k <= 0) {
    for (int w = tid; w < nwl; w += kMaskThreads) mask_bits[w_begin + w] = 0u;
    if (cq == 0 && tid == 0) *nnz = 0;
    return;
  }
  hist1[tid] = 0;
  if (tid < 32) hist2[tid] = 0;
  stage_keys<kMaskThreads>(x, e_begin, nloc, nwl * 32, keys);
  __syncthreads();

  // ---- pass 1: high digit ----
  hist_high_digit<kMaskThreads>(keys, nloc, hist1);
  cluster.sync();
  {
    int v = 0;
#pragma unroll
    for (int r = 0; r < kTopkCluster; ++r) v += cluster.map_shared_rank(hist1, r)[tid];
    ghist[tid] = v;
  }
  __syncthreads();
  find_bin<kMaskThreads>(ghist, 1024, k, scratch, sel);
  const int hi_bin = sel[0], above_hi = sel[1];

  // ---- pass 2: low digit among keys with that high digit ----
  hist_low_digit<kMaskThreads>(keys, nloc, hi_bin, hist2);
  cluster.sync();
  if (tid < 32) {
    int v = 0;
#pragma unroll
    for (int r = 0; r < kTopkCluster; ++r) v += cluster.map_shared_rank(hist2, r)[tid];
    ghist[tid] = v;
  }
  __syncthreads();
  find_bin<kMaskThreads>(ghist, 32, k - above_hi, scratch, sel);
  const uint32_t kstar = ((uint32_t)hi_bin << 5) | (uint32_t)sel[0];
  const int q_ties = k - above_hi - sel[1];     // ties at K* to keep, cluster-wide

  bitmaps_gt_eq<kMaskThreads>(keys, nloc, kstar, gt, eq);
  __syncthreads();

  // ---- thread-contiguous words: one packed scan of (ties, keys above) ----
  const int per = (nwl + kMaskThreads - 1) / kMaskThreads;
  const int w0 = min(nwl, tid * per), w1 = min(nwl, w0 + per);
  int gcnt = 0, ecnt = 0;
  for (int w = w0; w < w1; ++w) {
    gcnt += __popc(gt[w]);
    ecnt += __popc(eq[w]);
  }
  int packed_total;
  const int packed = block_exclusive_scan<kMaskThreads>((ecnt << 16) | gcnt, scratch, &packed_total);
  const int g_excl = packed & 0xffff, e_excl = packed >> 16;
  if (tid == 0) {
    pub[0] = packed_total >> 16;
    pub[1] = packed_total & 0xffff;
  }
  cluster.sync();
  int tie_base = 0, out_base = 0;
  for (int r = 0; r < cq; ++r) {
    const int* rp = cluster.map_shared_rank(pub, r);
    const int ties_r = rp[0], gt_r = rp[1];
    out_base += gt_r + min(max(q_ties - tie_base, 0), ties_r);
    tie_base += ties_r;
  }
  cluster_arrive_release();   // no more reads of other CTAs' shared memory

  // the q lowest-index ties join the kept set; this thread's first slot
  int r_tie = tie_base + e_excl;
  int o = out_base + g_excl + min(max(q_ties - tie_base, 0), e_excl);
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = eq[w], kept = 0;
    while (bits && r_tie < q_ties) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      kept |= 1u << b;
      ++r_tie;
    }
    const uint32_t gw = gt[w] | kept;
    gt[w] = gw;
    wpre[w] = o;
    o += __popc(gw);
  }
  __syncthreads();

  for (int w = tid; w < nwl; w += kMaskThreads) mask_bits[w_begin + w] = gt[w];
  write_index_list<kMaskThreads>(gt, wpre, nwl, e_begin, idx);
  if (cq == 0 && tid == 0) *nnz = k;
  cluster_wait_acquire();     // no CTA leaves while another may still read its shared memory
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

// M <= 8: one thread per 16-byte vector (8 entries, whole blocks), so a
// warp's loads and stores are 512 contiguous bytes.  Rows hold d/8 vectors;
// the mask byte of vector vi of row r is byte vi of the row's mask words (bit
// i%32 of word i/32, little-endian), and the row's last vector also clears
// the padding bytes of its last word.  Each thread takes kVecPerThread
// vectors a grid-stride apart, all loads issued first.
constexpr int kVecPerThread = 1;

template <int M>
__global__ void __launch_bounds__(256)
nm_vec_kernel(const uint16_t* __restrict__ X, int64_t rows, int d, int n, uint16_t* X_masked,
              uint32_t* mask_bits) {
  const int vpr = d >> 3;
  const int wpr = (d + 31) >> 5;
  const int64_t nvec = rows * vpr;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t v0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  pdl_trigger();
  pdl_wait();
  uint4 q[kVecPerThread];
#pragma unroll
  for (int i = 0; i < kVecPerThread; ++i) {
    const int64_t v = v0 + i * stride;
    q[i] = v < nvec ? __ldg(reinterpret_cast<const uint4*>(X) + v) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < kVecPerThread; ++i) {
    const int64_t v = v0 + i * stride;
    if (v >= nvec) break;
    const uint32_t bits = nm_vec_bits<M>(q[i], n);
    if (X_masked != nullptr) reinterpret_cast<uint4*>(X_masked)[v] = nm_apply(q[i], bits, 0);
    if (mask_bits != nullptr) {
      const int64_t r = v / vpr;
      const int vi = (int)(v - r * vpr);
      uint8_t* mb = reinterpret_cast<uint8_t*>(mask_bits + r * wpr);
      mb[vi] = (uint8_t)bits;
      if (vi == vpr - 1)
        for (int j = vpr; j < 4 * wpr; ++j) mb[j] = 0;
    }
  }
}

// N:M variants, one warp per row ("Motivating Next-Gen Accelerators with
// Flexible (N:M) Activation Sparsity ...", Methodology: selection criteria
// ACT and WT, error mitigation PTS and VAR).  For every 32-entry word of the
// row the lane shifts the entries (x' = fp16(float32(x) - mu); without a
// shift x' is x, bit for bit), ranks each block of M by |x'| (ACT) or by float32(|x'|) * norm_i
// (WT) with lower indices first among equals and NaN last, and keeps n.
// With VAR the warp sums x'^2 and kept x'^2 over the row (float32, fixed
// order), gamma = sqrt(full / kept) (1 when either is 0), and a second pass
// writes fp16(gamma * x') for the kept entries.
template <int M, bool WT>
__device__ __forceinline__ uint32_t nm_ex_word(const uint16_t* src, int cnt, bool shifted, float mu,
                                               const float* norms, int e0, int n,
                                               uint32_t (&xs)[16]) {
  uint4 q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    q[i] = i * 8 < cnt ? __ldg(reinterpret_cast<const uint4*>(src) + i) : make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (shifted) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
        const __half2 h = __floats2half2_rn(__fsub_rn(f.x, mu), __fsub_rn(f.y, mu));
        xs[i * 4 + k] = *reinterpret_cast<const uint32_t*>(&h);
      } else {
        xs[i * 4 + k] = w[k];   // no shift: the input bits as they are
      }
    }
  }
  float nv[WT ? 32 : 1];
  if constexpr (WT) {   // the word's 32 norms as eight 16-byte loads
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 f = i * 4 < cnt ? __ldg(reinterpret_cast<const float4*>(norms + e0) + i)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
      nv[4 * i] = f.x; nv[4 * i + 1] = f.y; nv[4 * i + 2] = f.z; nv[4 * i + 3] = f.w;
    }
  }
  uint32_t bits = 0;
#pragma unroll
  for (int b0 = 0; b0 < 32; b0 += M) {
    if (b0 < cnt) {
      using T = typename std::conditional<WT, uint64_t, uint32_t>::type;
      T comp[M];
#pragma unroll
      for (int j = 0; j < M; ++j) {
        const int e = b0 + j;
        const uint16_t h = (uint16_t)(xs[e >> 1] >> (16 * (e & 1)));
        T key;
        if constexpr (WT) {
          const float sc = __fmul_rn(fabsf(h2f(h)), nv[e]);
          key = isnan(sc) ? T(0) : (T)__float_as_uint(sc) + T(1);
        } else {
          key = (T)mag_key(h);
        }
        comp[j] = (key << 5) | (T)(31 - j);
      }
      bits |= select_top_n<M>(comp, n) << b0;
    }
  }
  return bits;
}

// The fp16 words of gamma * (m . x') for one 32-entry word.
__device__ __forceinline__ void nm_ex_store(uint16_t* dst, int cnt, const uint32_t (&xs)[16],
                                            uint32_t bits, bool scale, float gamma) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (i * 8 < cnt) {
      uint32_t p[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int e = i * 8 + 2 * k;
        if (!scale) {
          const uint32_t lo = ((bits >> e) & 1u) ? (xs[i * 4 + k] & 0xffffu) : 0u;
          const uint32_t hi = ((bits >> (e + 1)) & 1u) ? (xs[i * 4 + k] & 0xffff0000u) : 0u;
          p[k] = lo | hi;
        } else {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&xs[i * 4 + k]));
          const float a = ((bits >> e) & 1u) ? __fmul_rn(gamma, f.x) : 0.f;
          const float b = ((bits >> (e + 1)) & 1u) ? __fmul_rn(gamma, f.y) : 0.f;
          const __half2 h = __floats2half2_rn(a, b);
          p[k] = *reinterpret_cast<const uint32_t*>(&h);
        }
      }
      reinterpret_cast<uint4*>(dst)[i] = make_uint4(p[0], p[1], p[2], p[3]);
    }
}

// Up to kExKeep words per lane (rows up to 32 * 32 * kExKeep entries) stay in
// registers between the VAR reduction and the scaled store; longer rows run
// the word a second time.
constexpr int kExKeep = 2;

template <int M, bool WT, bool VAR>
__global__ void __launch_bounds__(256)
nm_ex_kernel(const uint16_t* __restrict__ X, int64_t rows, int d, int n, const float* shift,
             const float* norms, uint16_t* X_masked, uint32_t* mask_bits, float* gamma_out) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  pdl_trigger();
  pdl_wait();
  if (row >= rows) return;                      // uniform across the warp
  const int wpr = (d + 31) >> 5;
  const bool shifted = shift != nullptr;
  const float mu = shifted ? __ldg(shift + row) : 0.f;
  const uint16_t* xrow = X + row * (int64_t)d;
  uint16_t* orow = X_masked + row * (int64_t)d;
  const bool keep = wpr <= 32 * kExKeep;
  uint32_t kx[VAR ? kExKeep : 1][16], kb[VAR ? kExKeep : 1];
  float full = 0.f, kept = 0.f;
  for (int w = lane, t = 0; w < wpr; w += 32, ++t) {
    const int e0 = w * 32, cnt = min(32, d - e0);
    uint32_t xs[16];
    const uint32_t bits = nm_ex_word<M, WT>(xrow + e0, cnt, shifted, mu, norms, e0, n, xs);
    if (mask_bits != nullptr) mask_bits[row * wpr + w] = bits;
    if constexpr (!VAR) {
      nm_ex_store(orow + e0, cnt, xs, bits, false, 1.f);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float v = h2f((uint16_t)(xs[e >> 1] >> (16 * (e & 1))));
        const float v2 = e < cnt ? v * v : 0.f;
        full += v2;
        kept += ((bits >> e) & 1u) ? v2 : 0.f;
      }
      if (keep) {
#pragma unroll
        for (int u = 0; u < kExKeep; ++u)
          if (u == t) {
#pragma unroll
            for (int k = 0; k < 16; ++k) kx[u][k] = xs[k];
            kb[u] = bits;
          }
      }
    }
  }
  if constexpr (!VAR) {
    if (gamma_out != nullptr && lane == 0) gamma_out[row] = 1.f;
  } else {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      full += __shfl_xor_sync(kFull, full, o);
      kept += __shfl_xor_sync(kFull, kept, o);
    }
    const float gamma = (full > 0.f && kept > 0.f) ? __fsqrt_rn(__fdiv_rn(full, kept)) : 1.f;
    if (gamma_out != nullptr && lane == 0) gamma_out[row] = gamma;
    if (keep) {
#pragma unroll
      for (int u = 0; u < kExKeep; ++u) {
        const int w = lane + 32 * u;
        if (w < wpr) nm_ex_store(orow + w * 32, min(32, d - w * 32), kx[u], kb[u], true, gamma);
      }
    } else {
      for (int w = lane; w < wpr; w += 32) {
        const int e0 = w * 32, cnt = min(32, d - e0);
        uint32_t xs[16];
        const uint32_t bits = nm_ex_word<M, WT>(xrow + e0, cnt, shifted, mu, norms, e0, n, xs);
        nm_ex_store(orow + e0, cnt, xs, bits, true, gamma);
      }
    }
  }
}

// One thread per column: sum over the rows in float64, one rounding to float32.
__global__ void __launch_bounds__(256)
col_sums_kernel(const uint16_t* __restrict__ WT, int64_t rows, int cols, float* sums) {
  pdl_trigger();
  pdl_wait();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= cols) return;
  double s = 0.0;
  for (int64_t i = 0; i < rows; ++i) s += (double)h2f(WT[i * cols + j]);
  sums[j] = __double2float_rn(s);
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
  if (d <= kTopkBlockUpTo && d <= kTopkBlockMaxD) {
    const int nw = (d + 31) / 32;
    const size_t smem = (size_t)nw * 64 + (size_t)nw * 8;
    cudaError_t e = cudaFuncSetAttribute(topk_block_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_block_kernel, dim3(1), dim3(kMaskThreads), smem, stream, x, d, k,
                      mask_bits, idx, nnz);
  }
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

// Packed 2:4 operand of the sparse tensor-core GEMM (the selection and the
// metadata layout are in nm_pack.cuh).  One CTA per 32 rows x 128 entries;
// thread t takes row t / 8 of them and entries 16 (t % 8) .. + 15: four
// blocks, i.e. exactly one 16-bit metadata field.  The quarter is assembled in
// shared memory and stored as 512 contiguous bytes.
template <int N>
__global__ void __launch_bounds__(256)
nm_pack_kernel(const uint16_t* __restrict__ X, int d, int kblocks, uint16_t* __restrict__ vals,
               uint8_t* __restrict__ meta) {
  __shared__ __align__(16) uint8_t quarter[512];
  const int rq = blockIdx.x / kblocks, kb = blockIdx.x - rq * kblocks;   // 32-row group, 128-entry block
  const int t = threadIdx.x, r32 = t >> 3, part = t & 7;
  const int64_t row = (int64_t)rq * 32 + r32;
  const uint16_t* src = X + row * d + kb * 128 + part * 16;
  pdl_trigger();
  pdl_wait();
  const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(src));
  const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(src) + 1);
  uint4 packed;
  const uint32_t nib = pack_piece<N>(v0, v1, packed);
  *reinterpret_cast<uint4*>(vals + row * (d / 2) + kb * 64 + part * 8) = packed;
  *reinterpret_cast<uint16_t*>(quarter + meta_quarter_offset(rq * 32 + r32, part)) = (uint16_t)nib;
  __syncthreads();
  if (t < 32) {
    const size_t tile = (size_t)(rq >> 2) * kblocks + kb;
    reinterpret_cast<uint4*>(meta + tile * 2048 + (size_t)(rq & 3) * 512)[t] =
        reinterpret_cast<const uint4*>(quarter)[t];
  }
}

cudaError_t launch_nm_pack(const uint16_t* X, int64_t rows, int d, int n, uint16_t* vals,
                           uint8_t* meta, cudaStream_t stream) {
  if (rows % 128 != 0 || d % 128 != 0 || (n != 1 && n != 2)) return cudaErrorInvalidValue;
  if (rows == 0) return cudaSuccess;
  const int kblocks = d / 128;
  const int64_t ctas = rows / 32 * kblocks;       // 32 rows x 128 entries each
  if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
  if (n == 2)
    return launch_pdl(nm_pack_kernel<2>, dim3((unsigned)ctas), dim3(256), 0, stream, X, d, kblocks,
                      vals, meta);
  return launch_pdl(nm_pack_kernel<1>, dim3((unsigned)ctas), dim3(256), 0, stream, X, d, kblocks,
                    vals, meta);
}

cudaError_t launch_nm_mask(const uint16_t* X, int64_t rows, int d, int n, int m,
                           uint16_t* X_masked, uint32_t* mask_bits, cudaStream_t stream) {
  const int64_t threads = rows * ((d + 31) / 32);
  if (threads == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  const int64_t nvec = rows * (d / 8);
  const unsigned vblocks = (unsigned)((nvec + 256 * kVecPerThread - 1) / (256 * kVecPerThread));
  cudaError_t e = cudaSuccess;
  switch (m) {
    case 1: e = launch_pdl(nm_vec_kernel<1>, dim3(vblocks), dim3(256), 0, stream, X, rows, d, n, X_masked, mask_bits); break;
    case 2: e = launch_pdl(nm_vec_kernel<2>, dim3(vblocks), dim3(256), 0, stream, X, rows, d, n, X_masked, mask_bits); break;
    case 4: e = launch_pdl(nm_vec_kernel<4>, dim3(vblocks), dim3(256), 0, stream, X, rows, d, n, X_masked, mask_bits); break;
    case 8: e = launch_pdl(nm_vec_kernel<8>, dim3(vblocks), dim3(256), 0, stream, X, rows, d, n, X_masked, mask_bits); break;
    case 16: e = launch_pdl(nm_mask_kernel<16>, dim3(blocks), dim3(256), 0, stream, X, rows, d, n, X_masked, mask_bits); break;
    case 32: e = launch_pdl(nm_mask_kernel<32>, dim3(blocks), dim3(256), 0, stream, X, rows, d, n, X_masked, mask_bits); break;
    default: return cudaErrorInvalidValue;
  }
  return e;
}

cudaError_t launch_nm_ex(const uint16_t* X, int64_t rows, int d, int n, int m, const float* shift,
                         const float* norms, bool var, uint16_t* X_masked, uint32_t* mask_bits,
                         float* gamma_out, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const dim3 grid((unsigned)((rows + 7) / 8)), block(256);
#define SIG_NM_EX_V(MM, W, V)                                                                  \
  launch_pdl(nm_ex_kernel<MM, W, V>, grid, block, 0, stream, X, rows, d, n, shift, norms,      \
             X_masked, mask_bits, gamma_out)
#define SIG_NM_EX(MM)                                                                           \
  if (m == MM) {                                                                                \
    if (norms != nullptr) return var ? SIG_NM_EX_V(MM, true, true) : SIG_NM_EX_V(MM, true, false); \
    return var ? SIG_NM_EX_V(MM, false, true) : SIG_NM_EX_V(MM, false, false);                 \
  }
  SIG_NM_EX(1) SIG_NM_EX(2) SIG_NM_EX(4) SIG_NM_EX(8) SIG_NM_EX(16) SIG_NM_EX(32)
#undef SIG_NM_EX
#undef SIG_NM_EX_V
  return cudaErrorInvalidValue;
}

cudaError_t launch_col_sums(const uint16_t* WT, int64_t rows, int cols, float* sums,
                            cudaStream_t stream) {
  if (cols == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((cols + 255) / 256);
  return launch_pdl(col_sums_kernel, dim3(blocks), dim3(256), 0, stream, WT, rows, cols, sums);
}

cudaError_t launch_row_norms(const uint16_t* WT, int64_t rows, int cols, float* norms,
                             cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  return launch_pdl(row_norms_kernel, dim3(blocks), dim3(256), 0, stream, WT, rows, cols, norms);
}

}  // namespace sig
