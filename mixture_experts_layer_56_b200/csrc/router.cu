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

// Eight consecutive elements of a row as fp32 (zero outside the matrix).
template <typename TIn>
struct Row8;
template <>
struct Row8<bf16> {
  uint4 raw;
  __device__ __forceinline__ void load(const bf16* __restrict__ src, int64_t row, int64_t nrows,
                                       int d, int j) {
    if (row < nrows && j + 8 <= d) {
      raw = *reinterpret_cast<const uint4*>(src + row * d + j);
    } else {
      uint16_t h[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        h[q] = (row < nrows && j + q < d)
                   ? reinterpret_cast<const uint16_t*>(src)[row * d + j + q] : uint16_t(0);
      raw = make_uint4(h[0] | (uint32_t(h[1]) << 16), h[2] | (uint32_t(h[3]) << 16),
                       h[4] | (uint32_t(h[5]) << 16), h[6] | (uint32_t(h[7]) << 16));
    }
  }
  __device__ __forceinline__ float get(int q) const {
    const uint32_t w = q < 2 ? raw.x : q < 4 ? raw.y : q < 6 ? raw.z : raw.w;
    return __uint_as_float((q & 1) ? (w & 0xffff0000u) : (w << 16));
  }
};
template <>
struct Row8<float> {
  float4 lo, hi;
  __device__ __forceinline__ void load(const float* __restrict__ src, int64_t row, int64_t nrows,
                                       int d, int j) {
    if (row < nrows && j + 8 <= d && (d & 3) == 0) {
      lo = *reinterpret_cast<const float4*>(src + row * d + j);
      hi = *reinterpret_cast<const float4*>(src + row * d + j + 4);
    } else {
      float v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = (row < nrows && j + q < d) ? src[row * d + j + q] : 0.0f;
      lo = make_float4(v[0], v[1], v[2], v[3]);
      hi = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
  __device__ __forceinline__ float get(int q) const {
    const float4& v = q < 4 ? lo : hi;
    const int r = q & 3;
    return r == 0 ? v.x : r == 1 ? v.y : r == 2 ? v.z : v.w;
  }
};

// d-chunk staged per step: as long as shared memory allows (the global loads
// of the next chunk are in flight while the current one is multiplied).
template <int EPT>
constexpr int router_chunk() {
  return EPT <= 2 ? 128 : (EPT <= 4 ? 64 : 32);
}
template <int EPT>
constexpr int router_smem_bytes() {
  return router_chunk<EPT>() * (kTokPerCta + EPT * 32) * 4;
}

template <typename TIn, int EPT, bool STATS>
__global__ void __launch_bounds__(kRouterWarps * 32)
router_topk_kernel(const TIn* __restrict__ u, const TIn* __restrict__ E,
                   const float* __restrict__ bias, int64_t T, int d, int n, int K, int flags,
                   int32_t* __restrict__ idx, float* __restrict__ w, float* __restrict__ pstat) {
  constexpr int NP = EPT * 32;
  constexpr int KC = router_chunk<EPT>();
  constexpr int NT = kRouterWarps * 32;      // threads
  constexpr int UG = KC / 8 * kTokPerCta / NT;  // u items (8 columns each) per thread
  constexpr int EG = KC / 8 * NP / NT;          // E items per thread
  // one d-chunk of u (tokens) and E (experts), transposed to [j][row], fp32
  extern __shared__ __align__(16) float smem_f[];
  float (*sU)[kTokPerCta] = reinterpret_cast<float (*)[kTokPerCta]>(smem_f);
  float (*sE)[NP] = reinterpret_cast<float (*)[NP]>(smem_f + KC * kTokPerCta);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTokPerCta;

  // staging assignment: item i = tid + NT*k covers 8 columns of one row,
  // row = i % rows, column group = i / rows.  Within a warp the group is
  // fixed and the rows are consecutive, so the transposed stores hit 32
  // distinct banks.
  Row8<TIn> pu[UG];
  Row8<TIn> pe[EG];
  auto prefetch = [&](int j0) {
#pragma unroll
    for (int k = 0; k < UG; ++k) {
      const int i = tid + NT * k;
      pu[k].load(u, t0 + i % kTokPerCta, T, d, j0 + (i / kTokPerCta) * 8);
    }
#pragma unroll
    for (int k = 0; k < EG; ++k) {
      const int i = tid + NT * k;
      pe[k].load(E, i % NP, n, d, j0 + (i / NP) * 8);
    }
  };

  float acc[kTokPerWarp][EPT];
#pragma unroll
  for (int i = 0; i < kTokPerWarp; ++i)
#pragma unroll
    for (int q = 0; q < EPT; ++q) acc[i][q] = 0.0f;

  prefetch(0);
  for (int j0 = 0; j0 < d; j0 += KC) {
    __syncthreads();  // the previous chunk's reads are done
#pragma unroll
    for (int k = 0; k < UG; ++k) {
      const int i = tid + NT * k;
#pragma unroll
      for (int q = 0; q < 8; ++q) sU[(i / kTokPerCta) * 8 + q][i % kTokPerCta] = pu[k].get(q);
    }
#pragma unroll
    for (int k = 0; k < EG; ++k) {
      const int i = tid + NT * k;
#pragma unroll
      for (int q = 0; q < 8; ++q) sE[(i / NP) * 8 + q][i % NP] = pe[k].get(q);
    }
    __syncthreads();
    if (j0 + KC < d) prefetch(j0 + KC);  // in flight during the FMAs below
    const int jn = min(KC, d - j0);
#pragma unroll 8
    for (int j = 0; j < jn; ++j) {
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
#define MOE_ROUTER_CASE(N)                                                                  \
  case N: {                                                                                 \
    auto kern = router_topk_kernel<TIn, N, STATS>;                                          \
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,             \
                             router_smem_bytes<N>()) != cudaSuccess)                        \
      return MOE_ERR_CUDA;                                                                  \
    kern<<<grid, block, router_smem_bytes<N>(), st>>>(u, E, bias, T, d, n, K, flags, idx, w, \
                                                     pstat);                                \
    break;                                                                                  \
  }
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
