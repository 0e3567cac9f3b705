// Device helpers shared by the libsig kernels (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace sig {

constexpr unsigned kFull = 0xffffffffu;

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the previous kernel on the stream drains; it
// must wait for that grid (and its memory) before touching global memory.
// Triggering at once lets the next kernel's CTAs take SM slots as ours exit.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Atomic add with acquire-release semantics at GPU scope: publishes the
// writes that the CTA made before a preceding __syncthreads, and makes the
// writes published by earlier arrivers visible to the CTA after the next one.
__device__ __forceinline__ unsigned atomic_add_acq_rel_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Relaxed (morally strong) global accesses at GPU scope.  An aligned 64-bit
// access is single-copy atomic, so a value and its tag stored together are
// seen together.
__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u32(unsigned* p, unsigned v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// L2 policy for data read exactly once (weight rows): evict first, so that
// the stream does not push the small reused buffers (x, index lists, split-K
// partials, counters) out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 16-byte streaming load of weights: not kept in L1, evict-first in L2.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p, uint64_t pol) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p), "l"(pol));
  return r;
}

__device__ __forceinline__ float h2f(uint16_t bits) {
  return __half2float(__ushort_as_half(bits));
}

__device__ __forceinline__ uint16_t f2h_rn(float v) {
  return __half_as_ushort(__float2half_rn(v));
}

// acc[k] += w[k] * xv for the eight fp16 weights packed in `v`, float32 FMA.
__device__ __forceinline__ void fma8(float (&acc)[8], const uint4& v, float xv) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
    acc[2 * k] = fmaf(f.x, xv, acc[2 * k]);
    acc[2 * k + 1] = fmaf(f.y, xv, acc[2 * k + 1]);
  }
}

// 8-byte streaming load of 8-bit weights (not kept in L1, evict-first in L2).
__device__ __forceinline__ uint2 ld_stream_v2(const void* p, uint64_t pol) {
  uint2 r;
  asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.u32 {%0,%1}, [%2], %3;"
      : "=r"(r.x), "=r"(r.y)
      : "l"(p), "l"(pol));
  return r;
}

// 4-byte streaming load of eight int4 weights (not kept in L1, evict-first in L2).
__device__ __forceinline__ uint32_t ld_stream_u32(const void* p, uint64_t pol) {
  uint32_t r;
  asm("ld.global.nc.L1::no_allocate.L2::cache_hint.u32 %0, [%1], %2;" : "=r"(r) : "l"(p), "l"(pol));
  return r;
}

// acc[k] += q_k * xv for the eight int4 weights of w (weight k in bits
// 4k .. 4k+3, two's complement): each nibble is sign-extended by two shifts
// and converted to float32 (exact), then one float32 FMA.
__device__ __forceinline__ void fma8_i4(float (&acc)[8], uint32_t w, float xv) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int q = (int)(w << (28 - 4 * k)) >> 28;           // nibble k, sign-extended
    acc[k] = fmaf(__int2float_rn(q), xv, acc[k]);
  }
}

// acc[k] += q_k * xv for the eight int8 weights packed in v: each byte is
// sign-extended by two shifts and converted to float32 (exact), then one
// float32 FMA.  Measured on B200 against a byte-permute into fp16 1024 + u
// with a half2 subtract (with scalar or packed FMAs): the conversion path is
// 1.6-2x faster at every Llama shape (4096 -> 11008 at 50 %: 10.9 against
// 17.4-17.9 us).
__device__ __forceinline__ void fma8_i8(float (&acc)[8], const uint2& v, float xv) {
  const uint32_t w[2] = {v.x, v.y};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int q = (int)(w[k] << (24 - 8 * b)) >> 24;      // byte b, sign-extended
      acc[4 * k + b] = fmaf(__int2float_rn(q), xv, acc[4 * k + b]);
    }
  }
}

// The same for eight fp8 e4m3 weights: the hardware converts two codes to an
// fp16 pair in one instruction (every e4m3 value is exact in fp16).
__device__ __forceinline__ void fma8_e4m3(float (&acc)[8], const uint2& v, float xv) {
  const uint32_t w[2] = {v.x, v.y};
  const float2 x2 = make_float2(xv, xv);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[k] & 0xffffu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[k] >> 16), __NV_E4M3);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    const float2 r0 = __ffma2_rn(a, x2, make_float2(acc[4 * k], acc[4 * k + 1]));
    const float2 r1 = __ffma2_rn(b, x2, make_float2(acc[4 * k + 2], acc[4 * k + 3]));
    acc[4 * k] = r0.x; acc[4 * k + 1] = r0.y; acc[4 * k + 2] = r1.x; acc[4 * k + 3] = r1.y;
  }
}

// 8 mask bits for the 8 fp16 values in v: |x| >= th (th = t rounded up to
// fp16, exact for fp16 inputs; NaN never passes an ordered compare).
__device__ __forceinline__ uint32_t thresh_bits8(const uint4& v, __half2 th2) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t b = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t m = __hge2_mask(__habs2(*reinterpret_cast<const __half2*>(&w[q])), th2);
    b |= ((m & 1u) | ((m >> 15) & 2u)) << (2 * q);
  }
  return b;
}

// The threshold as the fp16 pair thresh_bits8 compares against: t rounded up
// to fp16, or 0 for t <= 0 (every number passes).
__device__ __forceinline__ __half2 thresh_half2(float t) {
  return __half2half2(t <= 0.f ? __float2half(0.f) : __float2half_ru(t));
}

// fp16 element k (0..7) of a 16-byte vector.
__device__ __forceinline__ uint16_t lane_half(const uint4& v, int k) {
  const uint32_t w = (k < 2) ? v.x : (k < 4) ? v.y : (k < 6) ? v.z : v.w;
  return static_cast<uint16_t>((k & 1) ? (w >> 16) : (w & 0xffffu));
}

// Magnitude rank key of an fp16 value: 0 for NaN, 1 + (|x| bits) otherwise,
// so that a larger key means a larger magnitude and NaN ranks lowest.
__device__ __forceinline__ uint32_t mag_key(uint16_t bits) {
  const uint32_t a = bits & 0x7fffu;
  return a > 0x7c00u ? 0u : a + 1u;
}

// Exclusive prefix sum over a block of BLOCK threads.  `scratch` holds
// BLOCK/32 ints.  Returns the exclusive prefix; *total receives the sum.
template <int BLOCK>
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
  constexpr int kWarps = BLOCK / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kWarps ? scratch[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(kFull, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < kWarps) scratch[lane] = wi - w;  // exclusive warp offsets
    if (lane == kWarps - 1) scratch[kWarps] = wi;
  }
  __syncthreads();
  const int out = scratch[warp] + incl - v;
  *total = scratch[kWarps];
  __syncthreads();
  return out;
}

// Build the bit-packed mask of `d` entries into shared `words`
// (bit i%32 of word i/32) from a per-element predicate, reading the fp16
// vector x 16 bytes per thread.  Every thread of the block must call it.
template <int BLOCK, typename Pred>
__device__ __forceinline__ void build_mask_words(const uint16_t* __restrict__ x, int d,
                                                 uint32_t* words, Pred pred) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int nwords = (d + 31) >> 5;
  constexpr int kChunk = BLOCK * 8;   // elements per pass of the block
  constexpr int kUnroll = 8;          // passes whose loads are in flight together
  for (int base0 = 0; base0 < d; base0 += kChunk * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int e0 = base0 + u * kChunk + tid * 8;
      v[u] = e0 + 8 <= d ? __ldg(reinterpret_cast<const uint4*>(x + e0)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int base = base0 + u * kChunk;
      if (base >= d) break;               // uniform across the block
      const int e0 = base + tid * 8;
      uint32_t b = 0;
      if (e0 + 8 <= d) {
#pragma unroll
        for (int k = 0; k < 8; ++k) b |= (pred(lane_half(v[u], k), e0 + k) ? 1u : 0u) << k;
      } else {
        for (int k = 0; k < 8; ++k)
          if (e0 + k < d) b |= (pred(x[e0 + k], e0 + k) ? 1u : 0u) << k;
      }
      uint32_t w = b << (8 * (lane & 3));
      w |= __shfl_xor_sync(kFull, w, 1);
      w |= __shfl_xor_sync(kFull, w, 2);
      const int wi = (base >> 5) + (tid >> 2);
      if ((lane & 3) == 0 && wi < nwords) words[wi] = w;
    }
  }
}

}  // namespace sig
