// moe_dispatch_static_scratch: the dispatch of moe_dispatch with its scratch
// in a fixed array inside libmoe instead of a caller-supplied workspace.
//
// Who this is for: callers that cannot hand the library device memory on
// each call. An allocation may synchronise the device, and it can fail
// once a caching pool has already reserved the GPU's memory. Examples are a
// latency-bound serving loop, or a host library with no allocator of its own.
// This entry point allocates nothing. Its scratch is one file-scope device
// array of fixed size. Every call in the process, on every stream, uses that
// same array.
//
// The kernels are the ones moe_dispatch launches; only where the per-chunk
// counts and bases live differs.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// Per-chunk expert counts followed by per-chunk bases (int32 each).
// Nothing here has to start at zero: the count pass writes every entry of
// the first array before the scan reads it, and the scan writes every entry
// of the second before the scatter reads it.
static __device__ __align__(256) unsigned char g_dispatch_scratch[MOE_DISPATCH_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];
std::mutex g_setup_mu;

inline size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline bool misaligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// One-time set-up on the current device: check that it is an sm_100 part and
// look up the device address of the scratch array.
int scratch_of_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p) {
    *out = p;
    return MOE_OK;
  }
  std::lock_guard<std::mutex> lock(g_setup_mu);
  p = g_scratch_addr[dev].load(std::memory_order_relaxed);
  if (!p) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED;
    if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || !p) {
      // the failed lookup must not surface as a later launch's error; this also
      // consumes any earlier unread error of the thread (stated in moe.h)
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" {

int moe_dispatch_static_scratch(const moe_shape_t* shape, const int32_t* idx, int32_t* counts,
                                int32_t* offsets, int32_t* perm, int32_t* inv,
                                moe_stream_t stream) {
  using namespace moe;
  size_t ws_unused = 0;
  if (int rc = moe_workspace_size(shape, &ws_unused)) return rc;  // shape validation only
  if (!counts || !offsets) return MOE_ERR_NULLPTR;
  if (shape->T > 0 && (!idx || !perm || !inv)) return MOE_ERR_NULLPTR;
  if (misaligned16(counts) || misaligned16(offsets) ||
      (shape->T > 0 && (misaligned16(idx) || misaligned16(perm) || misaligned16(inv))))
    return MOE_ERR_ALIGN;
  const size_t per_array =
      round256(static_cast<size_t>(dispatch_num_chunks(shape->T)) * shape->n_routed * 4);
  if (2 * per_array > MOE_DISPATCH_STATIC_SCRATCH_BYTES) return MOE_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if (int rc = scratch_of_current_device(&scratch)) return rc;
  int32_t* chunk_counts = static_cast<int32_t*>(scratch);
  int32_t* chunk_base = reinterpret_cast<int32_t*>(static_cast<unsigned char*>(scratch) + per_array);
  StageScope sg(MOE_KERNEL_DISPATCH, static_cast<cudaStream_t>(stream));
  return launch_dispatch(idx, shape->T, shape->top_k, shape->n_routed, chunk_counts, chunk_base,
                         counts, offsets, perm, inv, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
