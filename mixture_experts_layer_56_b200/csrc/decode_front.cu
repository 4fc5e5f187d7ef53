// Router, dispatch and gather of a small batch (T <= kDispatchChunk tokens)
// in one launch, for the staged layer forward of decode-sized batches that
// the one-kernel decode layer does not take.
//
// At a hundred tokens the three stages are latency chains, not bandwidth:
// the logits are 2 T d N_r FLOPs, the dispatch a few hundred slots.  Here
// they run on one CTA per token with a single grid-wide step:
//  A/B. CTA c routes token c (and c + G, ...): the token's row in registers,
//     warp w forms u_t . e_i for experts w, w + 8, ... (four rows in flight)
//     as one fp32 FMA chain per lane plus a fixed shuffle tree, into shared
//     memory; then thread i takes expert i: softmax over the block
//     (fixed-order max and sum) and its rank among the keys (larger first,
//     lower expert index first on ties) is its slot if below K; gates are
//     not renormalised;
//  C. after every token is routed, each CTA sorts the T*K slots by expert,
//     stably (a counting sort: warp w ranks the slots of its contiguous
//     range within their experts, 32 at a time by warp match / popc; a block
//     scan gives the experts' offsets and each range's start within them),
//     CTA 0 writes counts / offsets / perm / inv, and CTA c copies its
//     tokens' rows of u to their K positions of X_perm.
// The grid is at most one CTA per SM, so all of it is resident; the grid-wide
// step is a counter in the workspace (zeroed before the launch) with a
// bounded wait.  Results equal moe_route + moe_dispatch + the gather up to
// the fp32 summation order of the logits.
#include <cuda.h>
#include <math_constants.h>

#include "common.cuh"
#include "decode_fused.h"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace moe {

namespace {

using namespace sm100;

constexpr int kFrWarps = 8;
constexpr int kFrThreads = kFrWarps * 32;
constexpr unsigned kFull = 0xffffffffu;

struct FrontSync {
  int select_done;  // CTAs done with their tokens' routing
};

__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// every CTA arrives once; bounded wait until all `n` have (acquire)
__device__ __forceinline__ bool grid_step(int* counter, int n, int32_t* status) {
  __shared__ int ok;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    atomicAdd(counter, 1);
    const uint64_t t0 = sm100::global_timer_ns();
    int v = 0;
    ok = 1;
    while (true) {
      asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
      if (v >= n) break;
      if (sm100::global_timer_ns() - t0 > sm100::kWaitTimeoutNs) {
        record_status(status, MOE_ERR_DEVICE_CHECK);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
  }
  __syncthreads();
  __threadfence();
  return ok != 0;
}

template <int NV>
__global__ void __launch_bounds__(kFrThreads, 1)
decode_front_kernel(const bf16* __restrict__ u, const bf16* __restrict__ E,
                    const float* __restrict__ bias, int T, int n, int K, int flags,
                    int32_t* __restrict__ idx, float* __restrict__ w, float* __restrict__ logits,
                    int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                    int32_t* __restrict__ perm, int32_t* __restrict__ inv, bf16* __restrict__ xperm,
                    FrontSync* sync, int32_t* status) {
  constexpr int D = NV * 256;
  __shared__ int s_slot_e[kDispatchChunk * 32];  // expert of slot t*K + k
  __shared__ int s_pos[kDispatchChunk * 32];     // rank within (range, expert), then position
  __shared__ int s_wcnt[kFrWarps][256];          // per warp range and expert: slots, then start
  __shared__ int s_wsum[kFrWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = static_cast<int>(gridDim.x);
  pdl_wait();
  pdl_trigger();

  // ---- A. logits and B. softmax / top-K, one CTA per token ------------------
  __shared__ float s_logit[256], s_key[256];
  __shared__ float s_red[2][kFrWarps];
  const bool select_only = (flags & MOE_FLAG_BIAS_SELECT_ONLY) != 0;
  for (int t = blockIdx.x; t < T; t += G) {
    // the token's row stays in registers; warp w takes experts w, w + 8, ...,
    // two expert rows in flight at a time
    const uint4* ur = reinterpret_cast<const uint4*>(u + static_cast<int64_t>(t) * D);
    uint4 uv[NV];
#pragma unroll
    for (int v = 0; v < NV; ++v) uv[v] = ur[v * 32 + lane];
    for (int e0 = warp; e0 < n; e0 += 4 * kFrWarps) {
      uint4 x[4][NV];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = e0 + j * kFrWarps;
        const uint4* er = reinterpret_cast<const uint4*>(E + static_cast<int64_t>(e < n ? e : e0) * D);
#pragma unroll
        for (int v = 0; v < NV; ++v) x[j][v] = er[v * 32 + lane];
      }
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const float u0 = bf_lo(uv[v].x), u1 = bf_hi(uv[v].x), u2 = bf_lo(uv[v].y),
                    u3 = bf_hi(uv[v].y), u4 = bf_lo(uv[v].z), u5 = bf_hi(uv[v].z),
                    u6 = bf_lo(uv[v].w), u7 = bf_hi(uv[v].w);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 y = x[j][v];
          float a = acc[j];
          a = fmaf(u0, bf_lo(y.x), a); a = fmaf(u1, bf_hi(y.x), a);
          a = fmaf(u2, bf_lo(y.y), a); a = fmaf(u3, bf_hi(y.y), a);
          a = fmaf(u4, bf_lo(y.z), a); a = fmaf(u5, bf_hi(y.z), a);
          a = fmaf(u6, bf_lo(y.w), a); a = fmaf(u7, bf_hi(y.w), a);
          acc[j] = a;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] += __shfl_xor_sync(kFull, acc[j], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (e0 + j * kFrWarps < n) s_logit[e0 + j * kFrWarps] = acc[j];
      }
    }
    __syncthreads();
    // thread e takes expert e (n <= kFrThreads)
    {
      const int e = tid;
      float l = -CUDART_INF_F, key = -CUDART_INF_F;
      if (e < n) {
        const float raw = s_logit[e];
        key = raw + (bias ? bias[e] : 0.0f);
        l = select_only ? raw : key;
        s_key[e] = key;
      }
      float m = l;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
      if (lane == 0) s_red[0][warp] = m;
      __syncthreads();
      m = s_red[0][0];
#pragma unroll
      for (int w8 = 1; w8 < kFrWarps; ++w8) m = fmaxf(m, s_red[0][w8]);
      const float ex = e < n ? expf(l - m) : 0.0f;
      float z = ex;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
      if (lane == 0) s_red[1][warp] = z;
      __syncthreads();
      z = s_red[1][0];
#pragma unroll
      for (int w8 = 1; w8 < kFrWarps; ++w8) z += s_red[1][w8];
      if (e < n) {
        // rank: keys above this one, or equal to it at a lower index
        int rank = 0;
#pragma unroll 4
        for (int j = 0; j < n; ++j) {
          const float kj = s_key[j];
          rank += static_cast<int>(kj > key) | (static_cast<int>(kj == key) & static_cast<int>(j < e));
        }
        if (rank < K) {
          idx[t * K + rank] = e;
          w[t * K + rank] = ex * (1.0f / z);
        }
      }
    }
    __syncthreads();  // s_logit is free for the next token
  }
  if (!grid_step(&sync->select_done, G, status)) return;

  // ---- C. dispatch and gather -------------------------------------------------
  const int TK = T * K;
  for (int i = tid; i < kFrWarps * 256; i += kFrThreads) (&s_wcnt[0][0])[i] = 0;
  for (int i = tid; i < TK; i += kFrThreads) s_slot_e[i] = __ldcg(idx + i);
  __syncthreads();
  // 1. warp w ranks the slots of its range [w per, (w + 1) per) within their
  //    experts, in slot order: 32 at a time, equal experts ranked by lane
  const int per = (TK + kFrWarps - 1) / kFrWarps;
  const int i_lo = min(warp * per, TK), i_hi = min(i_lo + per, TK);
  for (int i0 = i_lo; i0 < i_hi; i0 += 32) {
    const int i = i0 + lane;
    const bool act = i < i_hi;
    const int e = act ? s_slot_e[i] : -1 - lane;
    const unsigned peers = __match_any_sync(kFull, e);
    const int before = __popc(peers & ((1u << lane) - 1u));
    const int base = act ? s_wcnt[warp][e] : 0;
    __syncwarp();
    if (act) {
      s_pos[i] = base + before;
      if (before == 0) s_wcnt[warp][e] = base + __popc(peers);
    }
    __syncwarp();
  }
  __syncthreads();
  // 2. thread e: the expert's count, its offset (block exclusive scan in
  //    expert order) and each warp range's start within the expert
  {
    const int e = tid;  // kFrThreads == 256 >= n
    int c = 0;
    if (e < n)
      for (int w8 = 0; w8 < kFrWarps; ++w8) c += s_wcnt[w8][e];
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w8 = 0; w8 < warp; ++w8) before += s_wsum[w8];
    const int off = before + incl - c;
    if (blockIdx.x == 0 && e < n) {
      counts[e] = c;
      offsets[e] = off;
      if (e == n - 1) offsets[n] = off + c;
    }
    if (e < n) {
      int run = off;
      for (int w8 = 0; w8 < kFrWarps; ++w8) {
        const int cw = s_wcnt[w8][e];
        s_wcnt[w8][e] = run;
        run += cw;
      }
    }
  }
  __syncthreads();
  // 3. each slot's position: its range's start within the expert + its rank
  for (int i = tid; i < TK; i += kFrThreads) {
    const int pos = s_wcnt[i / per][s_slot_e[i]] + s_pos[i];
    s_pos[i] = pos;
    if (blockIdx.x == 0) {
      perm[pos] = i;
      inv[i] = pos;
    }
  }
  __syncthreads();
  // gather: CTA c copies the rows of its tokens c, c + G, ...; warp w writes
  // the copies k = w, w + 8, ...
  for (int tt = blockIdx.x; tt < T; tt += G) {
    const uint4* src = reinterpret_cast<const uint4*>(u + static_cast<int64_t>(tt) * D);
    uint4 v[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) v[j] = src[j * 32 + lane];
    for (int kk = warp; kk < K; kk += kFrWarps) {
      uint4* dst = reinterpret_cast<uint4*>(xperm + static_cast<int64_t>(s_pos[tt * K + kk]) * D);
#pragma unroll
      for (int j = 0; j < NV; ++j) dst[j * 32 + lane] = v[j];
    }
  }
}

template <int NV>
int launch_front_nv(const moe_shape_t& s, const void* u, const void* E, const float* bias,
                    int32_t* idx, float* w, float* logits, int32_t* counts, int32_t* offsets,
                    int32_t* perm, int32_t* inv, void* xperm, FrontSync* sync, int32_t* status,
                    int grid, cudaStream_t st) {
  return launch_k(decode_front_kernel<NV>, grid, kFrThreads, 0, st, 1,
                  static_cast<const bf16*>(u), static_cast<const bf16*>(E), bias,
                  static_cast<int>(s.T), s.n_routed, s.top_k, s.flags, idx, w, logits, counts,
                  offsets, perm, inv, static_cast<bf16*>(xperm), sync, status);
}

}  // namespace

bool decode_front_eligible(const moe_shape_t& s) {
  const bool d_ok = s.d == 256 || s.d == 512 || s.d == 1024 || s.d == 2048;
  return s.dtype == MOE_DTYPE_BF16 && s.T >= 1 && s.T <= kDispatchChunk && d_ok &&
         s.top_k <= 32 && s.n_routed <= 256 && !(s.flags & MOE_FLAG_ROUTER_SIMT);
}

size_t decode_front_sync_bytes() { return sizeof(FrontSync); }

int launch_decode_front(const moe_shape_t& s, const void* u, const void* E, const float* bias,
                        int32_t* idx, float* w, float* logits, int32_t* counts, int32_t* offsets,
                        int32_t* perm, int32_t* inv, void* xperm, void* sync, int32_t* status,
                        int sms, cudaStream_t st) {
  const int grid = s.T < sms ? static_cast<int>(s.T) : sms;
  if (int rc = launch_zero_words(static_cast<int32_t*>(sync),
                                 static_cast<int>(sizeof(FrontSync) / sizeof(int32_t)), st))
    return rc;
  FrontSync* fs = static_cast<FrontSync*>(sync);
  switch (s.d) {
    case 256: return launch_front_nv<1>(s, u, E, bias, idx, w, logits, counts, offsets, perm, inv, xperm, fs, status, grid, st);
    case 512: return launch_front_nv<2>(s, u, E, bias, idx, w, logits, counts, offsets, perm, inv, xperm, fs, status, grid, st);
    case 1024: return launch_front_nv<4>(s, u, E, bias, idx, w, logits, counts, offsets, perm, inv, xperm, fs, status, grid, st);
    case 2048: return launch_front_nv<8>(s, u, E, bias, idx, w, logits, counts, offsets, perm, inv, xperm, fs, status, grid, st);
    default: return MOE_ERR_SHAPE;
  }
}

}  // namespace moe
