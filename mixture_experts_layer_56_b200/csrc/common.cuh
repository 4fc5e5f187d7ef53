// Shared device helpers of libmoe: status word, bf16 conversion, launch
// bookkeeping.  Everything here is plain CUDA C++ for sm_100a.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>

#include "../../include/moe.h"

namespace moe {

// Element type tags for the two supported dtypes.
using bf16 = __nv_bfloat16;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

// 16-byte vector of elements: 8 bf16 or 4 float.
template <typename T> struct Vec16;
template <> struct Vec16<bf16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const bf16* p, float* out) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      out[2 * i] = f.x;
      out[2 * i + 1] = f.y;
    }
  }
  __device__ __forceinline__ static void store(bf16* p, const float* in) {
    uint4 v;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = v;
  }
};
template <> struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float* out) {
    float4 v = *reinterpret_cast<const float4*>(p);
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  }
  __device__ __forceinline__ static void store(float* p, const float* in) {
    *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
  }
};

// SiLU(g) * u = g * u / (1 + e^-g).  e^-g is computed as 2^(-g log2 e) and
// the reciprocal directly, both on the special-function unit (ex2.approx,
// rcp.approx: a few ulp each, far below the bf16 rounding that follows).
// g is clamped at -80 so that 1 + e^-g stays finite (the product is then 0
// to within 1e-33).
__device__ __forceinline__ float silu_mul(float g, float u) {
  const float gc = fmaxf(g, -80.0f);
  float e, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(gc * -1.4426950408889634f));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + e));
  return g * r * u;
}

// The workspace begins with a 256-byte header whose first int32 is the
// status word that kernels set when a bounded wait gives up.
__device__ __forceinline__ void record_status(int32_t* status, int32_t code) {
  if (status) *reinterpret_cast<volatile int32_t*>(status) = code;
}

// Programmatic dependent launch.  A kernel started by launch_k() may begin
// while the kernel before it in the stream is still running.  pdl_wait()
// blocks until that kernel has completed and its writes are visible, so it
// must precede the first read or write of global memory that earlier
// stream work may touch; only set-up (barriers, TMEM, descriptor prefetch)
// goes before it.  pdl_trigger() lets the next kernel start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// host-side bookkeeping shared by the launch wrappers
// ---------------------------------------------------------------------------
void count_launch(int n = 1);
int check_launch();  // MOE_OK or MOE_ERR_CUDA after a <<<>>> launch

// Tracer bracket of one stage (moe_profile_enable): records a start event on
// `st` when built and an end event when destroyed, if tracing of `kind` is on.
class StageScope {
 public:
  StageScope(int32_t kind, cudaStream_t st);
  ~StageScope();
  StageScope(const StageScope&) = delete;
  StageScope& operator=(const StageScope&) = delete;

 private:
  cudaStream_t st_;
  long idx_ = -1;
};

// A kernel's opt-in dynamic shared-memory size, set on the current device
// the first time it launches there (the attribute belongs to the device's
// copy of the kernel; `done` holds one bit per device).
inline int ensure_smem_optin(const void* kern, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  const uint64_t bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return MOE_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  done.fetch_or(bit, std::memory_order_release);
  return MOE_OK;
}

// Launch with programmatic stream serialisation (the kernel must call
// pdl_wait() before touching global memory) and, if cluster > 1, thread
// block clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
int launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
             unsigned cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cluster > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cluster;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  count_launch();
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return check_launch();
}

}  // namespace moe
