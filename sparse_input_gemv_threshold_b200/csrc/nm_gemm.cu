// Tensor-core GEMM Y = A * B for the batched N:M activation product
// (Block Q-Sparse, "Q-Sparse ..." rebuttal, A2).  A is the masked activation
// block (tokens x K, K contiguous), B is the transposed weight WT (K x N,
// N contiguous), Y is tokens x N in fp16 with float32 accumulation.
//
// sm_100a design: one CTA per 128 x BN output tile, 256 threads.
//   - thread 0 streams 64-wide K slices of A and B into a 4-stage shared
//     ring with TMA (cp.async.bulk.tensor, 128-byte swizzle, no multicast),
//     signalling an mbarrier with the transaction byte count;
//   - thread 32 issues tcgen05.mma (kind::f16, M = 128, N = BN, K = 16) from
//     shared-memory descriptors into a float32 accumulator in tensor memory
//     and frees each stage with tcgen05.commit;
//   - all eight warps then read the accumulator with tcgen05.ld (each its
//     lane quarter and column half), round to fp16 and store through shared
//     memory with TMA.
// Launched with programmatic stream serialization: the launch, the mbarrier
// setup and the tensor-memory allocation overlap the end of the kernel before
// it; every thread then waits for that kernel (griddepcontrol.wait) before it
// reads global memory or starts a timed wait.
// Every mbarrier wait gives up after ~2 s of clock cycles (a device variable,
// settable through sig_set_wait_limit): the kernel then records
// SIG_ERR_TIMEOUT in a device error word, lets the copies it issued land
// (waiting at most the default ~2 s for each), frees its tensor memory and
// returns.
#include "common.cuh"
#include "internal.h"
#include "nm_ex.h"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace sig {

__device__ unsigned g_device_error = 0u;

// Cycles after which a pipeline wait gives up (sig_set_wait_limit); the waits
// that let already issued copies land after a give-up keep the full default.
constexpr long long kTimeoutCycles = 4000000000ll;  // ~2 s at 1.9 GHz
__device__ long long g_wait_limit = kTimeoutCycles;

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;          // one 128-byte swizzle row of fp16
constexpr int kStages = 4;
constexpr int kThreads = 256;   // warp 0 loads, warp 1 issues MMAs, all eight store
// Register cap of the GEMM kernels (64 per thread, the bound that four CTAs of
// 256 threads per SM would impose; shared memory allows one).  A GEMM CTA
// launched early behind the mask kernel before it (programmatic dependent
// launch) sits on an SM while that kernel still runs; 16 K registers leave
// the mask kernel six of its eight CTAs per SM, where the uncapped 90-128
// registers halved them (measured on B200: 2:4 and 8:16 mask + GEMM at
// 16384 x 4096 x 4096 slower by 85 us).
constexpr int kMinBlocksForRegs = 4;
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: false after the time limit or once another role aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  const long long t0 = clock64();
  const long long limit = *(volatile long long*)&g_wait_limit;
  while (!mbar_try(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      *abort_flag = 1;
      atomicOr(&g_device_error, 1u);
      return false;
    }
  }
  return true;
}

// Wait that is not cut short by a give-up: used to let issued copies and
// MMAs finish before the CTA frees its tensor memory and exits.  Bounded by
// the default limit; false if that ran out.
__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try(bar, parity))
    if (clock64() - t0 > kTimeoutCycles) return false;
  return true;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// Shared-memory matrix descriptor (tcgen05): start, leading and stride byte
// offsets in 16-byte units, version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fffu);
  d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3fffu) << 32;
  d |= (uint64_t)1 << 46;        // descriptor version for sm_100
  d |= (uint64_t)2 << 61;        // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: fp16 A and B, float32 D, A K-major,
// B MN-major, shape M x N.
__host__ __device__ constexpr uint32_t instr_desc_f16(int M, int N) {
  return (1u << 4)                       // D format: f32
         | (0u << 7) | (0u << 10)        // A, B format: f16
         | (0u << 15)                    // A K-major
         | (1u << 16)                    // B MN-major
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1)
               : "memory");
}

// Epilogue of one 128 x BN accumulator tile by the CTA's eight warps.  Warp w
// reads tensor-memory lanes 32 (w % 4) .. 32 (w % 4) + 31 (one output row per
// lane) and the columns of half w / 4 of the tile, 32 at a time (tcgen05.ld,
// wait), adds mu * colsum[c] when colsum is given, rounds to fp16 and writes
// the row's 64 bytes into the warp's staging area in shared memory
// (`stage_base` + w x 32 x BN fp16) in the 128-byte swizzled order of the
// output tensor map (box 64 columns x 32 rows), so that a quarter-warp of
// 16-byte stores covers all banks.  After every 64 columns one lane stores
// the block with TMA while the warp goes on to the next, and at the end waits
// only until the bulk stores have read shared memory.
template <int BN>
__device__ __forceinline__ void store_tile_tma(uint32_t tmem, int warp, int lane, uint32_t stage_base,
                                               const CUtensorMap* mapY, int m0, int n0, float mu,
                                               const float* colsum) {
  constexpr int kCols = BN / 2;                       // columns per warp
  const int q = warp & 3, c0 = (warp >> 2) * kCols;
  const uint32_t stage = stage_base + (uint32_t)warp * (32u * kCols * 2u);
  const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
  for (int cc = 0; cc < kCols; cc += 32) {
    const int c = c0 + cc;
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(lane_addr + (uint32_t)c));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    uint32_t p[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float v0 = __uint_as_float(r[2 * k]), v1 = __uint_as_float(r[2 * k + 1]);
      if (colsum != nullptr) {
        v0 = fmaf(mu, __ldg(colsum + n0 + c + 2 * k), v0);
        v1 = fmaf(mu, __ldg(colsum + n0 + c + 2 * k + 1), v1);
      }
      const __half2 h = __floats2half2_rn(v0, v1);
      p[k] = *reinterpret_cast<const uint32_t*>(&h);
    }
    // row `lane` of block cc / 64; 16-byte chunk j of the row at (j ^ (row % 8)) * 16
    const uint32_t row_base = stage + (uint32_t)(cc / 64) * 4096u + (uint32_t)lane * 128u;
    const int j0 = (cc % 64) / 8;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t addr = row_base + (uint32_t)(((j0 + j) ^ (lane & 7)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(p[4 * j]),
                   "r"(p[4 * j + 1]), "r"(p[4 * j + 2]), "r"(p[4 * j + 3])
                   : "memory");
    }
    if (cc % 64 == 32) {
      // the generic-proxy writes become visible to the bulk copy engine
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(mapY, stage + (uint32_t)(cc / 64) * 4096u, n0 + c - 32, m0 + q * 32);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    }
  }
  // shared memory may be reused or released once the stores have read it
  if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
  __syncwarp();
}

template <int BN>
struct __align__(1024) GemmSmem {
  uint16_t A[kStages][kBM * kBK];   // 16 KB per stage, K-major, swizzled rows of 128 B
  uint16_t B[kStages][kBK * BN];    // BN/64 blocks of 64 k-rows x 128 B
  unsigned long long full[kStages];
  unsigned long long empty[kStages];
  unsigned long long accum;
  uint32_t tmem_base;
  int abort_flag;
  int consumed;
};

template <int BN>
__global__ void __launch_bounds__(kThreads, kMinBlocksForRegs)
gemm_f16_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                const __grid_constant__ CUtensorMap mapY, int M, int N, int K, const float* __restrict__ shift,
                const float* __restrict__ colsum) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the dynamic window starts 1024-aligned only by request; align by hand
  GemmSmem<BN>& sm = *reinterpret_cast<GemmSmem<BN>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * kBM;
  const int kblocks = K / kBK;
  volatile int* abort_flag = &sm.abort_flag;
  pdl_trigger();

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.accum), 1);
    sm.abort_flag = 0;
    sm.consumed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(BN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = sm.tmem_base;
  // Nothing is read from global memory before the kernel before this one in
  // the stream has finished, and every timed wait starts after it.
  pdl_wait();

  constexpr uint32_t kStageBytes = (kBM * kBK + kBK * BN) * 2;
  int issued = 0;   // stages whose copies thread 0 has issued

  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer ----
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
        if (!mbar_wait(smem_u32(&sm.empty[s]), ph ^ 1u, abort_flag)) break;
        const uint32_t fb = smem_u32(&sm.full[s]);
        mbar_expect_tx(fb, kStageBytes);
        tma_load_2d(smem_u32(sm.A[s]), &mapA, kb * kBK, m0, fb);
#pragma unroll
        for (int j = 0; j < BN / 64; ++j)
          tma_load_2d(smem_u32(sm.B[s]) + j * (kBK * 128), &mapB, n0 + j * 64, kb * kBK, fb);
        ++issued;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer ----
      constexpr uint32_t idesc = instr_desc_f16(kBM, BN);
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
        if (!mbar_wait(smem_u32(&sm.full[s]), ph, abort_flag)) break;
        *(volatile int*)&sm.consumed = kb + 1;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t a0 = smem_u32(sm.A[s]), b0 = smem_u32(sm.B[s]);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          // A: K-major, advance 32 B inside the swizzled 128-B row.
          const uint64_t da = smem_desc(a0 + k * 32, 16, 1024);
          // B: MN-major, 16 k-rows = two 8-row groups (1024 B each) per step;
          // 64-wide N blocks sit kBK*128 bytes apart.
          const uint64_t db = smem_desc(b0 + k * 2048, kBK * 128, 1024);
          const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
          asm volatile(
              "{\n\t.reg .pred p;\n\t"
              "setp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
              "l"(da), "l"(db), "r"(idesc), "r"(acc)
              : "memory");
        }
        asm volatile(
            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                smem_u32(&sm.empty[s]))
            : "memory");
      }
      asm volatile(
          "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
              smem_u32(&sm.accum))
          : "memory");
    }
    __syncwarp();
  }

  // ---- epilogue: TMEM -> registers -> fp16 -> global ----
  // The MMA thread commits the accumulator barrier also after a give-up, so
  // it completes once every issued MMA has finished; this wait is not cut
  // short by the abort flag.
  const bool acc_done = drain_wait(smem_u32(&sm.accum), 0u);
  __syncwarp();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (acc_done && !*abort_flag) {
    const int row = m0 + (warp & 3) * 32 + lane;
    // the B stages are free once the accumulator is complete: 32 x BN fp16 per warp
    store_tile_tma<BN>(tmem, warp, lane, smem_u32(sm.B[0]), &mapY,
                       m0, n0, shift != nullptr ? __ldg(shift + row) : 0.f,   // the shift added back
                       shift != nullptr ? colsum : nullptr);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    // after a give-up: let the copies issued but never consumed land before
    // the CTA's shared memory goes away
    for (int kb = *(volatile int*)&sm.consumed; kb < issued; ++kb)
      drain_wait(smem_u32(&sm.full[kb % kStages]), (uint32_t)(kb / kStages) & 1u);
  }
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(BN)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// 2:4 sparse-operand GEMM (tcgen05.mma.sp, kind::f16).
//
// A is the packed activation: per row, the two kept values of every block of
// four entries (K/2 fp16, K contiguous), and their positions as 2-bit
// metadata.  For M = 128 and K = 32 logical entries one sparse MMA reads 32
// bits of metadata per tensor-memory lane; a 128 x 128 block of the logical
// A carries 2048 bytes of metadata = 128 lanes x 16 bytes, which one
// tcgen05.cp (128x128b) moves from shared to tensor memory.  The packed
// buffer keeps the metadata in exactly that lane order (see sparsify_nm in
// the header), so a stage brings it in with one 2048-byte bulk copy.
//
// Stage = 128 logical K: A 128 rows x 64 packed fp16 (16 KB, one 128-byte
// swizzled row each), B 128 k-rows x BN (BN/64 blocks of 16 KB), metadata
// 2 KB.  The issuer copies the stage's metadata into tensor memory, then
// issues four sparse MMAs (K = 32 each: A advances 32 bytes in its row, B
// 32 k-rows = 4096 bytes, the metadata one tensor-memory column; an odd
// column is addressed as the even one below it with selector id2 = 1).
// ---------------------------------------------------------------------------
constexpr int kSpBK = 128;        // logical K per stage
constexpr int kSpStages = 2;
constexpr uint32_t kSpMetaBytes = 2048;

template <int BN>
struct __align__(1024) SpSmem {
  uint16_t A[kSpStages][kBM * 64];      // 16 KB per stage
  uint16_t B[kSpStages][kSpBK * BN];    // BN/64 blocks of 128 k-rows x 128 B
  uint8_t E[kSpStages][kSpMetaBytes];   // metadata, lane-major (lane L at 16 L)
  unsigned long long full[kSpStages];
  unsigned long long empty[kSpStages];
  unsigned long long accum;
  uint32_t tmem_base;
  int abort_flag;
  int consumed;
};

// Instruction descriptor of the sparse MMA: the dense one with the sparse
// flag (bit 2) and the metadata selector id2 (bits 0-1).
__host__ __device__ constexpr uint32_t instr_desc_f16_sp(int M, int N, uint32_t id2) {
  return instr_desc_f16(M, N) | (1u << 2) | (id2 & 3u);
}

// Shared-memory descriptor of the metadata tile for tcgen05.cp 128x128b: no
// swizzle, K-major, 8-row core matrices of 16-byte rows stored contiguously
// (128 bytes apart); one 16-byte column, so the leading offset is unused.
__device__ __forceinline__ uint64_t smem_desc_meta(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fffu);
  d |= (uint64_t)((kSpMetaBytes >> 4) & 0x3fffu) << 16;   // leading offset (unused)
  d |= (uint64_t)((128u >> 4) & 0x3fffu) << 32;           // 8-row groups 128 B apart
  d |= (uint64_t)1 << 46;                                  // descriptor version for sm_100
  return d;                                                // layout type 0: no swizzle
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

template <int BN>
__global__ void __launch_bounds__(kThreads, kMinBlocksForRegs)
gemm_sp_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
               const uint8_t* __restrict__ meta, const __grid_constant__ CUtensorMap mapY, int M,
               int N, int K) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  SpSmem<BN>& sm = *reinterpret_cast<SpSmem<BN>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * kBM;
  const int kblocks = K / kSpBK;
  volatile int* abort_flag = &sm.abort_flag;
  constexpr uint32_t kTmemCols = BN == 256 ? 512u : 256u;   // BN accumulator + 4 metadata columns
  pdl_trigger();

  if (tid == 0) {
    for (int s = 0; s < kSpStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.accum), 1);
    sm.abort_flag = 0;
    sm.consumed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tmem_e = tmem + (uint32_t)BN;   // metadata columns, 4-aligned
  pdl_wait();

  constexpr uint32_t kStageBytes = kBM * 64 * 2 + kSpBK * BN * 2 + kSpMetaBytes;
  const uint8_t* meta_rb = meta + (size_t)blockIdx.y * (size_t)kblocks * kSpMetaBytes;
  int issued = 0;   // stages whose copies thread 0 has issued

  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer ----
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % kSpStages;
        const uint32_t ph = (uint32_t)(kb / kSpStages) & 1u;
        if (!mbar_wait(smem_u32(&sm.empty[s]), ph ^ 1u, abort_flag)) break;
        const uint32_t fb = smem_u32(&sm.full[s]);
        mbar_expect_tx(fb, kStageBytes);
        tma_load_2d(smem_u32(sm.A[s]), &mapA, kb * 64, m0, fb);
#pragma unroll
        for (int j = 0; j < BN / 64; ++j)
          tma_load_2d(smem_u32(sm.B[s]) + j * (kSpBK * 128), &mapB, n0 + j * 64, kb * kSpBK, fb);
        bulk_load(smem_u32(sm.E[s]), meta_rb + (size_t)kb * kSpMetaBytes, kSpMetaBytes, fb);
        ++issued;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer ----
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % kSpStages;
        const uint32_t ph = (uint32_t)(kb / kSpStages) & 1u;
        if (!mbar_wait(smem_u32(&sm.full[s]), ph, abort_flag)) break;
        *(volatile int*)&sm.consumed = kb + 1;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t a0 = smem_u32(sm.A[s]), b0 = smem_u32(sm.B[s]);
        asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(tmem_e),
                     "l"(smem_desc_meta(smem_u32(sm.E[s])))
                     : "memory");
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t da = smem_desc(a0 + j * 32, 16, 1024);
          const uint64_t db = smem_desc(b0 + j * 4096, kSpBK * 128, 1024);
          const uint32_t e_col = tmem_e + (uint32_t)j;
          const uint32_t idesc = instr_desc_f16_sp(kBM, BN, e_col & 1u);
          const uint32_t acc = (kb > 0 || j > 0) ? 1u : 0u;
          asm volatile(
              "{\n\t.reg .pred p;\n\t"
              "setp.ne.b32 p, %5, 0;\n\t"
              "tcgen05.mma.sp.cta_group::1.kind::f16 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(tmem),
              "l"(da), "l"(db), "r"(e_col & ~1u), "r"(idesc), "r"(acc)
              : "memory");
        }
        asm volatile(
            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                smem_u32(&sm.empty[s]))
            : "memory");
      }
      asm volatile(
          "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
              smem_u32(&sm.accum))
          : "memory");
    }
    __syncwarp();
  }

  // the accumulator barrier completes once every issued MMA has finished,
  // also after a give-up (see gemm_f16_kernel)
  const bool acc_done = drain_wait(smem_u32(&sm.accum), 0u);
  __syncwarp();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (acc_done && !*abort_flag)
    store_tile_tma<BN>(tmem, warp, lane, smem_u32(sm.B[0]), &mapY, m0, n0, 0.f, nullptr);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    for (int kb = *(volatile int*)&sm.consumed; kb < issued; ++kb)
      drain_wait(smem_u32(&sm.full[kb % kSpStages]), (uint32_t)(kb / kSpStages) & 1u);
  }
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// CTA-pair GEMMs (tcgen05 cta_group::2), dense kind::f16 and 2:4 sparse.
//
// A cluster of two CTAs computes a 256 x BN output tile: CTA r of the pair
// owns rows 128 r .. 128 r + 127 of the tile.  Each CTA loads its own 128 rows
// of A and HALF of the tile's B columns (BN/2, from column n0 + r BN/2) into
// the same shared-memory offsets; the leader (rank 0) issues one M = 256
// MMA that reads A and B from both CTAs' shared memory and accumulates each
// CTA's 128 rows in that CTA's tensor memory.  B (the weight) is therefore
// read from L2 half as often per SM as in the one-CTA kernels, and a stage is
// small enough for a four- (sparse) or six-stage (dense) ring.
//
// Both CTAs' copies for a stage complete on the LEADER's full barrier (the
// 2-SM form of the TMA load lets the peer signal it); the leader's thread
// posts the stage's bytes of both CTAs.  The leader's MMA thread frees a stage
// in both CTAs with one multicast commit, and commits the accumulator barrier
// of both CTAs the same way.  No TMA load multicasts: each CTA fetches its own
// tiles from this GPU's memory.
//
// Bounded waits as in the one-CTA kernels.  A give-up sets the CTA's abort
// flag; the epilogue of either CTA stores nothing if either flag is set
// (read across the pair through distributed shared memory), the leader lets
// the stages it posted land, and both CTAs then wait ~20 us before the final
// cluster barrier so that a peer copy whose stage the leader never posted has
// landed too.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// TMA load whose completion is signalled on the pair leader's barrier
// (`bar` is a shared::cluster address, possibly in the peer CTA).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                                 uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_load_1d_pair(uint32_t dst, const CUtensorMap* map, int c0,
                                                 uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.1d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2}], [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}

// WIDE (dense only): the pair computes a 256 x 512 tile as two M = 256,
// N = 256 MMAs per K step into tensor-memory columns [0, 256) and [256, 512);
// each CTA loads its 128 columns of each, so a stage brings 48 KB per CTA for
// twice the work of a 32 KB stage of the 256 x 256 tile.
template <bool SPARSE, bool WIDE = false>
struct PairCfg {
  static constexpr int kBN = WIDE ? 512 : 256;           // output columns of the pair's tile
  static constexpr int kBK = SPARSE ? 128 : 64;          // logical K per stage
  static constexpr int kStages = SPARSE ? 4 : (WIDE ? 4 : 6);
  static constexpr uint32_t kABytes = kBM * 64 * 2;      // 128 rows x 128 B
  static constexpr uint32_t kBBytes = kBK * (kBN / 2) * 2;
  static constexpr uint32_t kEBytes = SPARSE ? kSpMetaBytes : 0;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes + kEBytes;   // per CTA
  static constexpr uint32_t kTmemCols = (SPARSE || WIDE) ? 512u : 256u;
};

template <bool SPARSE, bool WIDE = false>
struct __align__(1024) PairSmem {
  using C = PairCfg<SPARSE, WIDE>;
  uint16_t A[C::kStages][kBM * 64];
  uint16_t B[C::kStages][C::kBK * (C::kBN / 2)];          // kBN / 128 blocks of 64 columns
  uint8_t E[SPARSE ? C::kStages : 1][SPARSE ? kSpMetaBytes : 16];
  unsigned long long full[C::kStages];                    // used in the leader
  unsigned long long empty[C::kStages];
  unsigned long long accum;
  uint32_t tmem_base;
  int abort_flag;
  int consumed;
};

template <bool SPARSE, bool WIDE = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, kMinBlocksForRegs)
gemm_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                 const __grid_constant__ CUtensorMap mapE, const __grid_constant__ CUtensorMap mapY,
                 int M, int N,
                 int K, const float* __restrict__ shift, const float* __restrict__ colsum) {
  using C = PairCfg<SPARSE, WIDE>;
  constexpr int BN = C::kBN, BK = C::kBK, S = C::kStages;
  constexpr int kMmas = BN / 256;                  // M = 256, N = 256 MMAs per K step
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  PairSmem<SPARSE, WIDE>& sm = *reinterpret_cast<PairSmem<SPARSE, WIDE>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int m0 = blockIdx.x * kBM;                 // this CTA's rows
  const int n0 = blockIdx.y * BN;                  // the pair's columns
  // this CTA's half of each MMA's 256 columns: columns n0 + 256 h + 128 rank
  const int nb = n0 + (int)rank * 128;
  const int kblocks = K / BK;
  volatile int* abort_flag = &sm.abort_flag;
  pdl_trigger();

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.accum), 1);
    sm.abort_flag = 0;
    sm.consumed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  // both CTAs' barriers exist before any copy or commit of the pair targets them
  cluster_sync();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer (both CTAs) ----
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (uint32_t)(kb / S) & 1u;
        if (!mbar_wait(smem_u32(&sm.empty[s]), ph ^ 1u, abort_flag)) break;
        const uint32_t fb = map_to_rank(smem_u32(&sm.full[s]), 0);
        if (leader) mbar_expect_tx(smem_u32(&sm.full[s]), 2 * C::kStageBytes);
        tma_load_2d_pair(smem_u32(sm.A[s]), &mapA, kb * 64, m0, fb);
#pragma unroll
        for (int j = 0; j < BN / 128; ++j)   // block j: MMA j / 2, columns (j % 2) * 64 of its half
          tma_load_2d_pair(smem_u32(sm.B[s]) + j * (BK * 128), &mapB,
                           nb + (j >> 1) * 256 + (j & 1) * 64, kb * BK, fb);
        if constexpr (SPARSE)
          tma_load_1d_pair(smem_u32(sm.E[s]), &mapE,
                           (int)(((size_t)blockIdx.x * kblocks + kb) * (kSpMetaBytes / 8)), fb);
        ++issued;
      }
    }
    __syncwarp();
  } else if (warp == 1 && leader) {
    if (lane == 0) {  // ---- MMA issuer (leader only) ----
      const uint32_t tmem_e = tmem + 256u;
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (uint32_t)(kb / S) & 1u;
        if (!mbar_wait(smem_u32(&sm.full[s]), ph, abort_flag)) break;
        *(volatile int*)&sm.consumed = kb + 1;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t a0 = smem_u32(sm.A[s]), b0 = smem_u32(sm.B[s]);
        if constexpr (SPARSE) {
          asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(tmem_e),
                       "l"(smem_desc_meta(smem_u32(sm.E[s])))
                       : "memory");
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t da = smem_desc(a0 + j * 32, 16, 1024);
            const uint64_t db = smem_desc(b0 + j * 4096, BK * 128, 1024);
            const uint32_t e_col = tmem_e + (uint32_t)j;
            const uint32_t idesc = instr_desc_f16_sp(2 * kBM, BN, e_col & 1u);
            const uint32_t acc = (kb > 0 || j > 0) ? 1u : 0u;
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.ne.b32 p, %5, 0;\n\t"
                "tcgen05.mma.sp.cta_group::2.kind::f16 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(tmem),
                "l"(da), "l"(db), "r"(e_col & ~1u), "r"(idesc), "r"(acc)
                : "memory");
          }
        } else {
          constexpr uint32_t idesc = instr_desc_f16(2 * kBM, 256);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t da = smem_desc(a0 + k * 32, 16, 1024);
            const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
#pragma unroll
            for (int h = 0; h < kMmas; ++h) {   // MMA h: its two 64-column blocks of B
              const uint64_t db = smem_desc(b0 + h * 2 * (BK * 128) + k * 2048, BK * 128, 1024);
              asm volatile(
                  "{\n\t.reg .pred p;\n\t"
                  "setp.ne.b32 p, %4, 0;\n\t"
                  "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(
                      tmem + (uint32_t)(h * 256)),
                  "l"(da), "l"(db), "r"(idesc), "r"(acc)
                  : "memory");
            }
          }
        }
        commit_pair(smem_u32(&sm.empty[s]));      // frees stage s in both CTAs
      }
      commit_pair(smem_u32(&sm.accum));
    }
    __syncwarp();
  }

  // ---- epilogue: each CTA its own 128 rows ----
  const bool acc_done = drain_wait(smem_u32(&sm.accum), 0u);
  __syncwarp();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const bool pair_ok =
      !*abort_flag && ld_cluster_u32(map_to_rank(smem_u32(&sm.abort_flag), rank ^ 1u)) == 0u;
  if (acc_done && pair_ok) {
    const int row = m0 + (warp & 3) * 32 + lane;
    store_tile_tma<BN>(tmem, warp, lane, smem_u32(sm.B[0]), &mapY,
                       m0, n0, shift != nullptr ? __ldg(shift + row) : 0.f,
                       shift != nullptr ? colsum : nullptr);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    if (leader)   // the stages this CTA posted: both CTAs' bytes land on these barriers
      for (int kb = *(volatile int*)&sm.consumed; kb < issued; ++kb)
        drain_wait(smem_u32(&sm.full[kb % S]), (uint32_t)(kb / S) & 1u);
    const long long t0 = clock64();
    while (clock64() - t0 < 40000) {
    }
  }
  __syncthreads();
  // the peer's tensor memory and shared memory stay until both CTAs are done
  cluster_sync();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::kTmemCols)
                 : "memory");
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D fp16 tensor map: inner extent `inner` (contiguous), outer extent
// `outer`, row pitch `pitch_elems`, box 64 x box_outer, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
              uint64_t pitch_elems, uint32_t box_outer) {
  auto enc = get_encode();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_elems * 2};
  cuuint32_t box[2] = {64, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 1-D tensor map over `bytes` of metadata as uint64 elements, box of one
// 2048-byte tile (256 elements), no swizzle.
bool make_map_meta(CUtensorMap* map, const void* base, uint64_t bytes) {
  auto enc = get_encode();
  if (enc == nullptr) return false;
  cuuint64_t dims[1] = {bytes / 8};
  cuuint64_t strides[1] = {0};
  cuuint32_t box[1] = {kSpMetaBytes / 8};
  cuuint32_t estr[1] = {1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 1, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// CTA pairs pay off once the weight tile is wide and deep enough that halving
// its L2 reads matters (measured on B200: 4096 x 4096 x 4096 2:4 GEMM 97 us
// with pairs against 115 us without; at 4096 x 1024 x 1024 10.9 against
// 10.2 us).
bool use_pair(int M, int N, int K) {
  return M % 256 == 0 && N % 256 == 0 && N >= 2048 && K >= 2048;
}

template <bool SPARSE, bool WIDE = false>
cudaError_t launch_pair(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& me,
                        const CUtensorMap& my, int M, int N, int K, const float* shift,
                        const float* colsum, cudaStream_t stream) {
  const size_t smem = sizeof(PairSmem<SPARSE, WIDE>) + 1024;
  auto fn = gemm_pair_kernel<SPARSE, WIDE>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(M / kBM, N / PairCfg<SPARSE, WIDE>::kBN);
  e = launch_pdl(fn, grid, dim3(kThreads), smem, stream, ma, mb, me, my, M, N, K, shift, colsum);
  if (e != cudaSuccess) return e;
  return cudaPeekAtLastError();
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& my, int M,
                      int N, int K, const float* shift, const float* colsum, cudaStream_t stream) {
  const size_t smem = sizeof(GemmSmem<BN>) + 1024;
  auto fn = gemm_f16_kernel<BN>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(N / BN, M / kBM);
  e = launch_pdl(fn, grid, dim3(kThreads), smem, stream, ma, mb, my, M, N, K, shift, colsum);
  if (e != cudaSuccess) return e;
  return cudaPeekAtLastError();
}

template <int BN>
cudaError_t launch_sp_bn(const CUtensorMap& ma, const CUtensorMap& mb, const uint8_t* meta,
                         const CUtensorMap& my, int M, int N, int K, cudaStream_t stream) {
  const size_t smem = sizeof(SpSmem<BN>) + 1024;
  auto fn = gemm_sp_kernel<BN>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(N / BN, M / kBM);
  e = launch_pdl(fn, grid, dim3(kThreads), smem, stream, ma, mb, meta, my, M, N, K);
  if (e != cudaSuccess) return e;
  return cudaPeekAtLastError();
}

}  // namespace

cudaError_t launch_gemm_f16_shift(const uint16_t* A, const uint16_t* WT, uint16_t* Y, int M, int N,
                                  int K, const float* shift, const float* colsum,
                                  cudaStream_t stream) {
  if (M % kBM != 0 || K % kBK != 0 || N % 128 != 0) return cudaErrorInvalidValue;
  if (shift != nullptr && colsum == nullptr) return cudaErrorInvalidValue;
  CUtensorMap ma, mb, my;
  if (!make_map(&ma, A, (uint64_t)K, (uint64_t)M, (uint64_t)K, kBM)) return cudaErrorInvalidValue;
  if (!make_map(&mb, WT, (uint64_t)N, (uint64_t)K, (uint64_t)N, kBK)) return cudaErrorInvalidValue;
  if (!make_map(&my, Y, (uint64_t)N, (uint64_t)M, (uint64_t)N, 32)) return cudaErrorInvalidValue;
  // 256 x 512 pair tiles also for K >= 1024 when there are enough of them to
  // fill the GPU's CTA pairs (A/B on B200, 16384 x 1024 x 1024: 35.0 against
  // 50.0 us on 128 x 256 one-CTA tiles)
  if (M % 256 == 0 && N % 512 == 0 && K >= 1024 && (M / 256) * (N / 512) >= kNumSMs / 2)
    return launch_pair<false, true>(ma, mb, ma, my, M, N, K, shift, colsum, stream);
  if (use_pair(M, N, K)) {   // CTA pairs: 256 x 512 (or 256 x 256) tiles, half of B per CTA
    if (N % 512 == 0)
      return launch_pair<false, true>(ma, mb, ma, my, M, N, K, shift, colsum, stream);
    return launch_pair<false>(ma, mb, ma, my, M, N, K, shift, colsum, stream);
  }
  if (N % 256 == 0) return launch_bn<256>(ma, mb, my, M, N, K, shift, colsum, stream);
  return launch_bn<128>(ma, mb, my, M, N, K, shift, colsum, stream);
}

cudaError_t launch_gemm_f16(const uint16_t* A, const uint16_t* WT, uint16_t* Y, int M, int N,
                            int K, cudaStream_t stream) {
  return launch_gemm_f16_shift(A, WT, Y, M, N, K, nullptr, nullptr, stream);
}

cudaError_t launch_gemm_sp(const uint16_t* vals, const uint8_t* meta, const uint16_t* WT,
                           uint16_t* Y, int M, int N, int K, cudaStream_t stream) {
  if (M % kBM != 0 || K % kSpBK != 0 || N % 128 != 0) return cudaErrorInvalidValue;
  CUtensorMap ma, mb;
  if (!make_map(&ma, vals, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2, kBM))
    return cudaErrorInvalidValue;
  if (!make_map(&mb, WT, (uint64_t)N, (uint64_t)K, (uint64_t)N, kSpBK)) return cudaErrorInvalidValue;
  CUtensorMap my;
  if (!make_map(&my, Y, (uint64_t)N, (uint64_t)M, (uint64_t)N, 32)) return cudaErrorInvalidValue;
  if (use_pair(M, N, K)) {   // CTA pairs: 256 x 256 tiles, half of B per CTA
    CUtensorMap me;
    if (!make_map_meta(&me, meta, (uint64_t)M * (uint64_t)K / 8)) return cudaErrorInvalidValue;
    return launch_pair<true>(ma, mb, me, my, M, N, K, nullptr, nullptr, stream);
  }
  // 128-column tiles (two CTAs per SM) once 128 x 256 tiles would take two
  // waves or more (A/B on B200, 16384 x 1024 x 1024: 34.8 against 38.1 us;
  // at 4096 x 1024 x 1024 the wide tiles win, 9.2 against 9.8 us)
  if (N % 256 == 0 && (M / kBM) * (N / 256) < 2 * kNumSMs)
    return launch_sp_bn<256>(ma, mb, meta, my, M, N, K, stream);
  return launch_sp_bn<128>(ma, mb, meta, my, M, N, K, stream);
}

cudaError_t set_wait_limit(long long cycles) {
  const long long v = cycles > 0 ? cycles : kTimeoutCycles;
  return cudaMemcpyToSymbol(g_wait_limit, &v, sizeof(v));
}

cudaError_t read_device_error(unsigned* out, cudaStream_t stream) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_device_error, sizeof(unsigned), 0,
                                            cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  const unsigned zero = 0;
  return cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(unsigned), 0,
                                 cudaMemcpyHostToDevice, stream);
}

}  // namespace sig
