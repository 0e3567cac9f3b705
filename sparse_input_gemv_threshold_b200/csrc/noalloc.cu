// gated_mlp_sparse_noalloc: the RaNA gated MLP without a caller-provided
// workspace, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run this layer: a plugin inside a host program that owns all device
// memory through its own pool, a serving loop with a fixed memory budget
// decided at start-up, or C code with no allocator of its own.  This entry
// point takes only the inputs and outputs.  Its scratch (split-K partial sums
// with their epoch words for the two products, and the fp16 hidden vector h when
// h_out is NULL) lives in one file-scope device array of
// SIG_NOALLOC_SCRATCH_BYTES (4 MiB) that every GPU which loads the library
// holds until the process exits.
//
// The array is shared by every call on a device and keeps the last call's
// contents, so each call first clears what must start at zero: the epoch and
// tagged partial-sum words of the two products.
// Calls that overlap on the GPU (other streams, other host threads) race on
// the array; serialise them.  A call whose scratch would exceed the array is
// rejected with SIG_ERR_SHAPE before anything is enqueued.
//
// In host code the array's name is a host-side stand-in, not a device
// address.  The first call on each device (with that device current) asks the
// runtime for the array's device address and caches it; make that first call
// before any stream capture.  The cache is keyed by device ordinal only: after
// cudaDeviceReset the primary context (and the array's address in it) is new,
// and the cached address is stale, so the header tells callers not to use
// this entry point on a device after resetting it.
#include "../../include/sig.h"
#include "internal.h"

#include <cuda_runtime.h>

#include <mutex>

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SIG_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" int gated_mlp_sparse_noalloc(const uint16_t* x, const uint16_t* WgT,
                                        const uint16_t* WuT, const uint16_t* WdT,
                                        const float* down_norms, int64_t d_model, int64_t d_ff,
                                        float t, uint16_t* y, uint16_t* h_out,
                                        uint32_t* mask_out, sig_stream_t stream) {
  using namespace sig;
  if (x == nullptr || WgT == nullptr || WuT == nullptr || WdT == nullptr ||
      down_norms == nullptr || y == nullptr)
    return SIG_ERR_NULL;
  if (d_model < 8 || d_model % 8 != 0 || d_model > kMaxDIn || d_ff < 8 || d_ff % 8 != 0 ||
      d_ff > kMaxDIn)
    return SIG_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(WgT) || !aligned16(WuT) || !aligned16(WdT) || !aligned16(y) ||
      (h_out != nullptr && !aligned16(h_out)) || !aligned4(down_norms) || !aligned4(mask_out))
    return SIG_ERR_ALIGN;
  const GatedPlan g = plan_gated(d_model, d_ff);
  if (g.total > (size_t)SIG_NOALLOC_SCRATCH_BYTES) return SIG_ERR_SHAPE;

  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return SIG_ERR_CUDA;
  char* base = static_cast<char*>(scratch);
  cudaStream_t st = (cudaStream_t)stream;

  // The split-K finish tags each partial sum with the tile's epoch; the array
  // keeps the previous call's words, which may come from another shape, so
  // every call starts from zeroed epochs and words (everything below h).
  if (g.off_h > 0 && cudaMemsetAsync(base, 0, g.off_h, st) != cudaSuccess) return SIG_ERR_CUDA;

  uint16_t* h = h_out != nullptr ? h_out : reinterpret_cast<uint16_t*>(base + g.off_h);
  GemvLaunch up{};
  up.WT[0] = WgT; up.WT2 = WuT; up.y[0] = h; up.d_out[0] = (int)d_ff;
  up.x = x; up.d_in = (int)d_model; up.ws = base;
  if (launch_gemv(MASK_DENSE, EPI_SILU_MUL, g.up, up, st) != cudaSuccess) return SIG_ERR_CUDA;
  GemvLaunch dn{};
  dn.WT[0] = WdT; dn.y[0] = y; dn.d_out[0] = (int)d_model;
  dn.x = h; dn.scale = down_norms; dn.t = t; dn.d_in = (int)d_ff; dn.mask_out = mask_out;
  dn.ws = base + g.off_down;
  if (launch_gemv(MASK_THRESH_SCALED, EPI_STORE, g.down, dn, st) != cudaSuccess)
    return SIG_ERR_CUDA;
  return SIG_OK;
}
