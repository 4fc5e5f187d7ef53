// Router, dispatch and gather of a small batch (T <= kDispatchChunk tokens)
// in one launch, for the staged layer forward of decode-sized batches that
// the one-kernel decode layer does not take.
//
// At a hundred tokens the three stages are latency chains, not bandwidth:
// the logits are 2 T d N_r FLOPs, the dispatch a few hundred slots.  Here
// they run on one CTA per token with a single grid-wide step:
//  A/B. CTA c routes token c (and c + G, ...): the token's row in registers,
//     warp w forms u_t . e_i for experts w, w + 8, ... as one fp32 FMA chain
//     per lane plus a fixed shuffle tree, into shared memory; warp 0 then
//     runs softmax and top-K (lower expert index first on ties, gates not
//     renormalised) and writes idx / w;
//  C. after every token is routed: each CTA builds the stable counting sort
//     of the T*K slots (warp ballots per 32 tokens, as the one-block
//     dispatch does), CTA 0 writes counts / offsets / perm / inv, and CTA c
//     copies its tokens' rows of u to their K positions of X_perm.
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

template <int NV, int NW>
__global__ void __launch_bounds__(kFrThreads, 1)
decode_front_kernel(const bf16* __restrict__ u, const bf16* __restrict__ E,
                    const float* __restrict__ bias, int T, int n, int K, int flags,
                    int32_t* __restrict__ idx, float* __restrict__ w, float* __restrict__ logits,
                    int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                    int32_t* __restrict__ perm, int32_t* __restrict__ inv, bf16* __restrict__ xperm,
                    FrontSync* sync, int32_t* status) {
  constexpr int D = NV * 256;
  __shared__ int wc[4][256];
  __shared__ int tot[256];
  __shared__ int spos[kDispatchChunk][32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = static_cast<int>(gridDim.x);
  pdl_wait();
  pdl_trigger();

  // ---- A. logits and B. softmax / top-K, one CTA per token ------------------
  __shared__ float s_logit[256];
  const bool select_only = (flags & MOE_FLAG_BIAS_SELECT_ONLY) != 0;
  for (int t = blockIdx.x; t < T; t += G) {
    // the token's row stays in registers; warp w takes experts w, w + 8, ...,
    // two expert rows in flight at a time
    const uint4* ur = reinterpret_cast<const uint4*>(u + static_cast<int64_t>(t) * D);
    uint4 uv[NV];
#pragma unroll
    for (int v = 0; v < NV; ++v) uv[v] = ur[v * 32 + lane];
    for (int e0 = warp; e0 < n; e0 += 2 * kFrWarps) {
      const int e1 = e0 + kFrWarps;
      const uint4* er0 = reinterpret_cast<const uint4*>(E + static_cast<int64_t>(e0) * D);
      const uint4* er1 = reinterpret_cast<const uint4*>(E + static_cast<int64_t>(e1 < n ? e1 : e0) * D);
      uint4 x0[NV], x1[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        x0[v] = er0[v * 32 + lane];
        x1[v] = er1[v * 32 + lane];
      }
      float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const float u0 = bf_lo(uv[v].x), u1 = bf_hi(uv[v].x), u2 = bf_lo(uv[v].y),
                    u3 = bf_hi(uv[v].y), u4 = bf_lo(uv[v].z), u5 = bf_hi(uv[v].z),
                    u6 = bf_lo(uv[v].w), u7 = bf_hi(uv[v].w);
        a0 = fmaf(u0, bf_lo(x0[v].x), a0); a0 = fmaf(u1, bf_hi(x0[v].x), a0);
        a0 = fmaf(u2, bf_lo(x0[v].y), a0); a0 = fmaf(u3, bf_hi(x0[v].y), a0);
        a0 = fmaf(u4, bf_lo(x0[v].z), a0); a0 = fmaf(u5, bf_hi(x0[v].z), a0);
        a0 = fmaf(u6, bf_lo(x0[v].w), a0); a0 = fmaf(u7, bf_hi(x0[v].w), a0);
        a1 = fmaf(u0, bf_lo(x1[v].x), a1); a1 = fmaf(u1, bf_hi(x1[v].x), a1);
        a1 = fmaf(u2, bf_lo(x1[v].y), a1); a1 = fmaf(u3, bf_hi(x1[v].y), a1);
        a1 = fmaf(u4, bf_lo(x1[v].z), a1); a1 = fmaf(u5, bf_hi(x1[v].z), a1);
        a1 = fmaf(u6, bf_lo(x1[v].w), a1); a1 = fmaf(u7, bf_hi(x1[v].w), a1);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a0 += __shfl_xor_sync(kFull, a0, o);
        a1 += __shfl_xor_sync(kFull, a1, o);
      }
      if (lane == 0) {
        s_logit[e0] = a0;
        if (e1 < n) s_logit[e1] = a1;
      }
    }
    __syncthreads();
    if (warp == 0) {
      float lg[8], key[8], ex[8];
      float m = -CUDART_INF_F;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int e = lane + 32 * q;
        float l = -CUDART_INF_F, kv = -CUDART_INF_F;
        if (e < n) {
          const float raw = s_logit[e];
          kv = raw + (bias ? bias[e] : 0.0f);
          l = select_only ? raw : kv;
        }
        lg[q] = l;
        key[q] = kv;
        m = fmaxf(m, l);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
      float z = 0.0f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        ex[q] = (lane + 32 * q < n) ? expf(lg[q] - m) : 0.0f;
        z += ex[q];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
      const float inv_z = 1.0f / z;
      unsigned taken = 0;
      for (int k = 0; k < K; ++k) {
        float bv = -CUDART_INF_F;
        int bi = 0x7fffffff;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int e = lane + 32 * q;
          if (!((taken >> q) & 1u) && e < n && (key[q] > bv || bi == 0x7fffffff)) {
            bv = key[q];
            bi = e;
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ov = __shfl_xor_sync(kFull, bv, o);
          const int oi = __shfl_xor_sync(kFull, bi, o);
          if (ov > bv || (ov == bv && oi < bi)) {
            bv = ov;
            bi = oi;
          }
        }
        if ((bi & 31) == lane) {
          taken |= 1u << (bi >> 5);
          float g = 0.0f;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (q == (bi >> 5)) g = ex[q];
          idx[t * K + k] = bi;
          w[t * K + k] = g * inv_z;
        }
      }
    }
    __syncthreads();  // s_logit is free for the next token
  }
  if (!grid_step(&sync->select_done, G, status)) return;

  // ---- C. dispatch and gather -------------------------------------------------
  // warps 0-3: one token per thread (T <= 128), the experts it chose as bits
  for (int i = tid; i < 4 * 256; i += kFrThreads) (&wc[0][0])[i] = 0;
  int ek[32];
  uint32_t mask[NW];
#pragma unroll
  for (int v = 0; v < NW; ++v) mask[v] = 0;
  const bool ranker = warp < 4;  // warp-uniform
  const int t = tid;
  if (ranker) {
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      ek[k] = (t < T && k < K) ? __ldcg(idx + t * K + k) : -1;
#pragma unroll
      for (int v = 0; v < NW; ++v)
        if (ek[k] >= 0 && (ek[k] >> 5) == v) mask[v] |= 1u << (ek[k] & 31);
    }
  }
  __syncthreads();  // wc is zero
  if (ranker) {
#pragma unroll
    for (int v = 0; v < NW; ++v) {
      const uint32_t um = __reduce_or_sync(kFull, mask[v]);
      for (uint32_t m = um; m != 0; m &= m - 1) {
        const int b = __ffs(m) - 1;
        const unsigned bal = __ballot_sync(kFull, (mask[v] >> b) & 1u);
        if (lane == 0) wc[warp][v * 32 + b] = __popc(bal);
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < 256; e += kFrThreads) {
    int c = 0;
    if (e < n)
      for (int v = 0; v < 4; ++v) c += wc[v][e];
    tot[e] = c;
    if (blockIdx.x == 0 && e < n) counts[e] = c;
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive scan over the experts, eight entries a lane
    int v8[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v8[i] = tot[lane * 8 + i];
      sum += v8[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      tot[e] = run;
      if (blockIdx.x == 0 && e < n) offsets[e] = run;
      run += v8[i];
    }
    if (blockIdx.x == 0 && lane == 31) offsets[n] = incl;
  }
  __syncthreads();
  for (int e = tid; e < n; e += kFrThreads) {
    int run = tot[e];
    for (int v = 0; v < 4; ++v) {
      const int c = wc[v][e];
      wc[v][e] = run;
      run += c;
    }
  }
  __syncthreads();
  if (ranker) {
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int v = 0; v < NW; ++v) {
      const uint32_t um = __reduce_or_sync(kFull, mask[v]);
      for (uint32_t m = um; m != 0; m &= m - 1) {
        const int b = __ffs(m) - 1;
        const int e = v * 32 + b;
        const bool has = (mask[v] >> b) & 1u;
        const unsigned bal = __ballot_sync(kFull, has);
        if (has) {
          const int pos = wc[warp][e] + __popc(bal & lt);
          int kk = 0;
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (ek[k] == e) kk = k;
          if (blockIdx.x == 0) {
            perm[pos] = t * K + kk;
            inv[t * K + kk] = pos;
          }
          spos[t][kk] = pos;
        }
      }
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
      uint4* dst = reinterpret_cast<uint4*>(xperm + static_cast<int64_t>(spos[tt][kk]) * D);
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
  const int nw = (s.n_routed + 31) / 32;
#define MOE_FRONT_CASE(W)                                                                      \
  case W:                                                                                      \
    return launch_k(decode_front_kernel<NV, W>, grid, kFrThreads, 0, st, 1,                    \
                    static_cast<const bf16*>(u), static_cast<const bf16*>(E), bias,            \
                    static_cast<int>(s.T), s.n_routed, s.top_k, s.flags, idx, w, logits, counts, \
                    offsets, perm, inv, static_cast<bf16*>(xperm), sync, status);
  switch (nw) {
    MOE_FRONT_CASE(1) MOE_FRONT_CASE(2) MOE_FRONT_CASE(3) MOE_FRONT_CASE(4)
    MOE_FRONT_CASE(5) MOE_FRONT_CASE(6) MOE_FRONT_CASE(7) MOE_FRONT_CASE(8)
    default: return MOE_ERR_SHAPE;
  }
#undef MOE_FRONT_CASE
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
  if (cudaMemsetAsync(sync, 0, sizeof(FrontSync), st) != cudaSuccess) return MOE_ERR_CUDA;
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
