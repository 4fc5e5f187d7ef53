// Router of the DeepSeekMoE layer (§3.2, eqs. (10)-(11)): fp32 logits
// l_{t,i} = sum_j u_{t,j} e_{i,j} (+ b_i) on CUDA cores, softmax over the
// routed experts and top-K selection with warp shuffles.
//
// A CTA of 4 warps owns 32 tokens; a warp owns 8 tokens and lane L owns
// experts L, L+32, ... (EPT = ceil(N_r / 32) of them).  d is walked in
// 32-wide chunks staged in shared memory as fp32; every logit is one fp32
// FMA chain in increasing j, so equal centroids give bitwise-equal logits.
// The selection runs on logits (softmax is monotone), lower index first on
// ties; gates are exp(l - max) / sum, not renormalised over the top K.
#include <math_constants.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kRouterWarps = 4;
constexpr int kTokPerWarp = 8;
constexpr int kTokPerCta = kRouterWarps * kTokPerWarp;  // 32
constexpr int kChunk = 32;

// Stage rows [r0, r0+nr) x columns [j0, j0+32) of a row-major [nrows, d]
// matrix into dst[j][r] (fp32, zero outside the matrix).
template <typename TIn>
__device__ __forceinline__ void stage_transposed(const TIn* __restrict__ src, int64_t r0, int nr,
                                                 int64_t nrows, int d, int j0, float* dst,
                                                 int ld_dst) {
  constexpr int V = Vec16<TIn>::N;      // elements per 16-byte load
  constexpr int PER_ROW = kChunk / V;   // loads per row chunk
  const bool vec_ok = (d % V) == 0;
  for (int i = threadIdx.x; i < nr * PER_ROW; i += blockDim.x) {
    const int rr = i / PER_ROW;
    const int c = (i - rr * PER_ROW) * V;
    const int64_t row = r0 + rr;
    float v[V];
    const int j = j0 + c;
    if (row < nrows && vec_ok && j + V <= d) {
      Vec16<TIn>::load(src + row * d + j, v);
    } else {
#pragma unroll
      for (int q = 0; q < V; ++q)
        v[q] = (row < nrows && j + q < d) ? to_f32(src[row * d + j + q]) : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < V; ++q) dst[(c + q) * ld_dst + rr] = v[q];
  }
}

template <typename TIn, int EPT, bool STATS>
__global__ void __launch_bounds__(kRouterWarps * 32)
router_topk_kernel(const TIn* __restrict__ u, const TIn* __restrict__ E,
                   const float* __restrict__ bias, int64_t T, int d, int n, int K, int flags,
                   int32_t* __restrict__ idx, float* __restrict__ w, float* __restrict__ pstat) {
  constexpr int NP = EPT * 32;
  __shared__ __align__(16) float sU[kChunk][kTokPerCta];
  __shared__ __align__(16) float sE[kChunk][NP];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTokPerCta;

  float acc[kTokPerWarp][EPT];
#pragma unroll
  for (int i = 0; i < kTokPerWarp; ++i)
#pragma unroll
    for (int q = 0; q < EPT; ++q) acc[i][q] = 0.0f;

  for (int j0 = 0; j0 < d; j0 += kChunk) {
    stage_transposed<TIn>(u, t0, kTokPerCta, T, d, j0, &sU[0][0], kTokPerCta);
    stage_transposed<TIn>(E, 0, NP, n, d, j0, &sE[0][0], NP);
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < kChunk; ++j) {
      float ev[EPT];
#pragma unroll
      for (int q = 0; q < EPT; ++q) ev[q] = sE[j][lane + 32 * q];
      const float4 ua = *reinterpret_cast<const float4*>(&sU[j][warp * kTokPerWarp]);
      const float4 ub = *reinterpret_cast<const float4*>(&sU[j][warp * kTokPerWarp + 4]);
      const float uv[kTokPerWarp] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
#pragma unroll
      for (int i = 0; i < kTokPerWarp; ++i)
#pragma unroll
        for (int q = 0; q < EPT; ++q) acc[i][q] = fmaf(uv[i], ev[q], acc[i][q]);
    }
    __syncthreads();
  }

  float b[EPT];
#pragma unroll
  for (int q = 0; q < EPT; ++q) {
    const int e = lane + 32 * q;
    b[q] = (bias != nullptr && e < n) ? bias[e] : 0.0f;
  }
  const bool select_only = (flags & MOE_FLAG_BIAS_SELECT_ONLY) != 0;

  float pst[EPT];
#pragma unroll
  for (int q = 0; q < EPT; ++q) pst[q] = 0.0f;

#pragma unroll
  for (int i = 0; i < kTokPerWarp; ++i) {
    const int64_t t = t0 + warp * kTokPerWarp + i;
    if (t >= T) break;  // warp-uniform
    // softmax logits (with the bias unless it only steers the selection)
    // and selection keys
    float lg[EPT], key[EPT];
#pragma unroll
    for (int q = 0; q < EPT; ++q) {
      const int e = lane + 32 * q;
      const float biased = acc[i][q] + b[q];
      lg[q] = e < n ? (select_only ? acc[i][q] : biased) : -CUDART_INF_F;
      key[q] = e < n ? biased : -CUDART_INF_F;
    }
    float m = lg[0];
#pragma unroll
    for (int q = 1; q < EPT; ++q) m = fmaxf(m, lg[q]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float ex[EPT];
    float s = 0.0f;
#pragma unroll
    for (int q = 0; q < EPT; ++q) {
      ex[q] = expf(lg[q] - m);
      s += ex[q];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float inv_s = 1.0f / s;
    if (STATS) {
#pragma unroll
      for (int q = 0; q < EPT; ++q) pst[q] += ex[q] / s;
    }

    unsigned taken = 0;
    for (int k = 0; k < K; ++k) {
      float bv = -CUDART_INF_F;
      int bi = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < EPT; ++q) {
        const int e = lane + 32 * q;
        if (!((taken >> q) & 1u) && e < n && (key[q] > bv || bi == 0x7fffffff)) {
          bv = key[q];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      // the lane that owns the winner writes its index and gate
      if ((bi & 31) == lane) {
        float l_sel = 0.0f;
#pragma unroll
        for (int q = 0; q < EPT; ++q)
          if (q == (bi >> 5)) l_sel = ex[q];
        idx[t * K + k] = bi;
        w[t * K + k] = l_sel * inv_s;
      }
    }
  }

  if (STATS) {
    // per-CTA partial sums of the scores, reduced in a fixed order later
    __shared__ float red[kRouterWarps][NP];
#pragma unroll
    for (int q = 0; q < EPT; ++q) red[warp][lane + 32 * q] = pst[q];
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
      float a = 0.0f;
      for (int ww = 0; ww < kRouterWarps; ++ww) a += red[ww][e];
      pstat[static_cast<int64_t>(blockIdx.x) * n + e] = a;
    }
  }
}

template <typename TIn, bool STATS>
int launch_router_t(const TIn* u, const TIn* E, const float* bias, int64_t T, int d, int n, int K,
                    int flags, int32_t* idx, float* w, float* pstat, cudaStream_t st) {
  const int ept = (n + 31) / 32;
  const unsigned grid = static_cast<unsigned>((T + kTokPerCta - 1) / kTokPerCta);
  const dim3 block(kRouterWarps * 32);
#define MOE_ROUTER_CASE(N)                                                                \
  case N:                                                                                 \
    router_topk_kernel<TIn, N, STATS><<<grid, block, 0, st>>>(u, E, bias, T, d, n, K, flags, \
                                                               idx, w, pstat);            \
    break;
  switch (ept) {
    MOE_ROUTER_CASE(1)
    MOE_ROUTER_CASE(2)
    MOE_ROUTER_CASE(3)
    MOE_ROUTER_CASE(4)
    MOE_ROUTER_CASE(5)
    MOE_ROUTER_CASE(6)
    MOE_ROUTER_CASE(7)
    MOE_ROUTER_CASE(8)
    default:
      return MOE_ERR_SHAPE;
  }
#undef MOE_ROUTER_CASE
  count_launch();
  return check_launch();
}

}  // namespace

int router_num_ctas(int64_t T) { return static_cast<int>((T + kTokPerCta - 1) / kTokPerCta); }

int launch_router(int dtype, const void* u, const void* E, const float* bias, int64_t T, int d,
                  int n, int K, int flags, int32_t* idx, float* w, float* pstat,
                  cudaStream_t st) {
  if (T == 0) return MOE_OK;
  if (dtype == MOE_DTYPE_BF16) {
    if (pstat)
      return launch_router_t<bf16, true>(static_cast<const bf16*>(u), static_cast<const bf16*>(E),
                                         bias, T, d, n, K, flags, idx, w, pstat, st);
    return launch_router_t<bf16, false>(static_cast<const bf16*>(u), static_cast<const bf16*>(E),
                                        bias, T, d, n, K, flags, idx, w, pstat, st);
  }
  if (pstat)
    return launch_router_t<float, true>(static_cast<const float*>(u),
                                        static_cast<const float*>(E), bias, T, d, n, K, flags,
                                        idx, w, pstat, st);
  return launch_router_t<float, false>(static_cast<const float*>(u), static_cast<const float*>(E),
                                       bias, T, d, n, K, flags, idx, w, pstat, st);
}

}  // namespace moe
