// Launch wrappers of the non-GEMM kernels of libmoe (host interface).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kDispatchChunk = 128;  // tokens per dispatch block

inline int64_t dispatch_num_chunks(int64_t T) { return (T + kDispatchChunk - 1) / kDispatchChunk; }
int router_num_ctas(int64_t T);

// chunk_counts (nullable): the tensor-core router also writes, per
// kDispatchChunk tokens, how many chose each expert ([chunks, n]); it returns
// false in *counted when it did not (the CUDA-core router, or no buffer).
int launch_router(int dtype, const void* u, const void* E, const float* bias, int64_t T, int d,
                  int n, int K, int flags, int32_t* idx, float* w, float* pstat,
                  int32_t* status, cudaStream_t st, int32_t* chunk_counts = nullptr,
                  bool* counted = nullptr);

// bf16 router on the tensor cores (router_tc.cu); pstat as launch_router's
int launch_router_tc(const void* u, const void* E, const float* bias, int64_t T, int d, int n,
                     int K, int flags, int32_t* idx, float* w, float* pstat, int32_t* status,
                     int32_t* chunk_counts, cudaStream_t st);

// Optional gather folded into the dispatch: xperm[p] = u[perm[p] / K].
struct DispatchGather {
  int dtype;       // MOE_DTYPE_*
  const void* u;   // [T, d]
  int d;
  void* xperm;     // [T*K, d]
};

// counts_ready: chunk_counts already hold the per-chunk counts of idx.
// dg (nullable): batches of more than one dispatch chunk also gather the
// rows into dg->xperm in the same launch; *gathered (nullable) tells
// whether that happened (single-chunk batches leave it to launch_gather).
int launch_dispatch(const int32_t* idx, int64_t T, int K, int n, int32_t* chunk_counts,
                    int32_t* chunk_base, int32_t* counts, int32_t* offsets, int32_t* perm,
                    int32_t* inv, cudaStream_t st, bool counts_ready = false,
                    const DispatchGather* dg = nullptr, bool* gathered = nullptr);

int launch_gather(int dtype, const void* u, const int32_t* perm, int64_t rows, int d, int K,
                  void* xperm, cudaStream_t st);

// Zeroes the n words at p (the grid-wide counters a decode kernel after it
// counts on) with a one-warp kernel: it waits for the kernel before it in the
// stream, which may still use the words, and then lets the next kernel begin
// its set-up while it writes (programmatic dependent launch).
int launch_zero_words(int32_t* p, int n, cudaStream_t st);

int launch_combine(int dtype, const void* u, const float* ysh, const void* y, const float* w,
                   const int32_t* inv, int64_t T, int d, int K, void* h, cudaStream_t st);

int launch_pack_w13(int dtype, const void* W1, const void* W3, void* W13, int n_experts, int I,
                    int d, cudaStream_t st);

// fp32 expert FFN on CUDA cores (the MOE_DTYPE_F32 path)
int launch_ffn_f32(const float* xperm, const float* u, const int32_t* offsets, int n_routed,
                   int64_t T, int n_shared, int d, int I, const float* W13, const float* W2,
                   const float* W13_s, const float* W2_s, float* act, float* act_s, float* y,
                   float* ysh, int max_routed_mtiles, cudaStream_t st);

int launch_balance_reduce(const float* pstat, int nblocks, const int32_t* counts, int64_t T,
                          int n, int K, float* f, float* P, cudaStream_t st);

int launch_zero(void* p, size_t bytes, cudaStream_t st);

}  // namespace moe
