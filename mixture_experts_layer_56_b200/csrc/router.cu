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

constexpr int kRouterWarps = 8;   // 4 token groups x 2 halves of d
constexpr int kRouterThreads = kRouterWarps * 32;
constexpr int kTokPerWarp = 8;
constexpr int kTokPerCta = 4 * kTokPerWarp;  // 32
#ifndef MOE_ROUTER_LOOKAHEAD
#define MOE_ROUTER_LOOKAHEAD 2
#endif
constexpr int kRouterLookahead = MOE_ROUTER_LOOKAHEAD;  // shared-load lookahead (d-steps)

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

// d-chunk staged per step (the global loads of the next chunk are in flight
// while the current one is multiplied).
template <int EPT>
constexpr int router_chunk() {
  return EPT <= 4 ? 64 : 32;
}
template <int EPT>
constexpr int router_smem_bytes() {
  return router_chunk<EPT>() * (kTokPerCta + EPT * 32) * 4;
}

// The logits of the CTA's 32 tokens x NP experts are an outer-product
// register tile: thread h of a 128-thread half owns tokens 4*(h%8)..+3 and
// experts XPT*(h/8)..+XPT-1 (XPT = 2*EPT), so one d-step costs it one
// 16-byte load of token values, XPT/4 of expert values (each a single
// shared-memory wavefront per warp) and 4*XPT FMAs.  The two halves of the
// CTA sum the two halves of every d-chunk; their partial sums are added once
// at the end (first half + second half), in the same order for every
// expert, so equal centroids give equal logits.
template <typename TIn, int EPT, bool STATS>
__global__ void __launch_bounds__(kRouterThreads)
router_topk_kernel(const TIn* __restrict__ u, const TIn* __restrict__ E,
                   const float* __restrict__ bias, int64_t T, int d, int n, int K, int flags,
                   int32_t* __restrict__ idx, float* __restrict__ w, float* __restrict__ pstat) {
  constexpr int NP = EPT * 32;
  constexpr int XPT = 2 * EPT;                   // experts per thread
  constexpr int KC = router_chunk<EPT>();
  constexpr int NT = kRouterThreads;
  constexpr int UI = KC / 8 * kTokPerCta;        // u items (8 columns each) per chunk
  constexpr int EI = KC / 8 * NP;                // E items per chunk
  constexpr int UG = (UI + NT - 1) / NT;         // items per thread
  constexpr int EG = (EI + NT - 1) / NT;
  constexpr int LDL = NP + 1;                    // logits row length (floats)
  static_assert(KC * (kTokPerCta + NP) >= kTokPerCta * LDL, "logits fit the staging area");
  // one d-chunk of u and E transposed to [j][row] (fp32); afterwards the
  // [token][expert] logits
  extern __shared__ __align__(16) float smem_f[];
  float* sU = smem_f;                   // [KC][kTokPerCta]
  float* sE = smem_f + KC * kTokPerCta;  // [KC][NP]
  float* sL = smem_f;                   // [kTokPerCta][LDL]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int half = tid >> 7;            // which half of each chunk this thread sums
  const int hh = tid & 127;
  const int tg = hh & 7;                // tokens 4*tg .. 4*tg+3
  const int eg = hh >> 3;               // experts XPT*eg .. XPT*eg+XPT-1
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTokPerCta;

  // two register buffers of staged chunks: the global loads of chunk c+2
  // are issued while chunk c is multiplied
  struct Staged {
    Row8<TIn> pu[UG];
    Row8<TIn> pe[EG];
  };
  Staged bufA, bufB;
  auto prefetch = [&](Staged& b, int j0) {
#pragma unroll
    for (int k = 0; k < UG; ++k) {
      const int i = tid + NT * k;
      if (UI % NT == 0 || i < UI) b.pu[k].load(u, t0 + i % kTokPerCta, T, d, j0 + (i / kTokPerCta) * 8);
    }
#pragma unroll
    for (int k = 0; k < EG; ++k) {
      const int i = tid + NT * k;
      if (EI % NT == 0 || i < EI) b.pe[k].load(E, i % NP, n, d, j0 + (i / NP) * 8);
    }
  };

  float acc[4][XPT];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int m = 0; m < XPT; ++m) acc[i][m] = 0.0f;

  auto chunk = [&](Staged& b, int j0) {
    __syncthreads();  // the previous chunk's reads are done
    // transposed stores: within a warp the 8-column group is fixed and the
    // rows are consecutive, so each store hits 32 distinct banks
#pragma unroll
    for (int k = 0; k < UG; ++k) {
      const int i = tid + NT * k;
      if (UI % NT != 0 && i >= UI) continue;
#pragma unroll
      for (int q = 0; q < 8; ++q) sU[((i / kTokPerCta) * 8 + q) * kTokPerCta + i % kTokPerCta] = b.pu[k].get(q);
    }
#pragma unroll
    for (int k = 0; k < EG; ++k) {
      const int i = tid + NT * k;
      if (EI % NT != 0 && i >= EI) continue;
#pragma unroll
      for (int q = 0; q < 8; ++q) sE[((i / NP) * 8 + q) * NP + i % NP] = b.pe[k].get(q);
    }
    __syncthreads();
    if (j0 + 2 * KC < d) prefetch(b, j0 + 2 * KC);  // in flight during the next two chunks
    // columns past d were staged as zeros, so their products are 0.  The
    // shared-memory operands of step jj+1 are loaded before the FMAs of step
    // jj, so their latency overlaps the arithmetic.
    const int jb = half * (KC / 2);
    constexpr int LA = kRouterLookahead;  // d-steps of shared loads in flight
    float ut[LA + 1][4], ev[LA + 1][XPT];
    auto load_step = [&](int buf, int jj) {
      const float4 uv = *reinterpret_cast<const float4*>(sU + (jb + jj) * kTokPerCta + 4 * tg);
      ut[buf][0] = uv.x; ut[buf][1] = uv.y; ut[buf][2] = uv.z; ut[buf][3] = uv.w;
      if constexpr (XPT % 4 == 0) {
#pragma unroll
        for (int m = 0; m < XPT; m += 4) {
          const float4 e4 = *reinterpret_cast<const float4*>(sE + (jb + jj) * NP + XPT * eg + m);
          ev[buf][m] = e4.x; ev[buf][m + 1] = e4.y; ev[buf][m + 2] = e4.z; ev[buf][m + 3] = e4.w;
        }
      } else {
#pragma unroll
        for (int m = 0; m < XPT; m += 2) {
          const float2 e2 = *reinterpret_cast<const float2*>(sE + (jb + jj) * NP + XPT * eg + m);
          ev[buf][m] = e2.x; ev[buf][m + 1] = e2.y;
        }
      }
    };
#pragma unroll
    for (int l = 0; l < LA; ++l) load_step(l, l);
#pragma unroll
    for (int jj = 0; jj < KC / 2; ++jj) {
      const int cur = jj % (LA + 1);
      if (jj + LA < KC / 2) load_step((jj + LA) % (LA + 1), jj + LA);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < XPT; ++m) acc[i][m] = fmaf(ut[cur][i], ev[cur][m], acc[i][m]);
    }
  };

  prefetch(bufA, 0);
  if (KC < d) prefetch(bufB, KC);
  for (int j0 = 0; j0 < d; j0 += 2 * KC) {
    chunk(bufA, j0);
    if (j0 + KC < d) chunk(bufB, j0 + KC);
  }

  // logits = first-half sums + second-half sums, into [token][expert]
  __syncthreads();
  if (half == 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int m = 0; m < XPT; ++m) sL[(4 * tg + i) * LDL + XPT * eg + m] = acc[i][m];
  }
  __syncthreads();
  if (half == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int m = 0; m < XPT; ++m) {
        float* p = sL + (4 * tg + i) * LDL + XPT * eg + m;
        *p = acc[i][m] + *p;
      }
  }
  __syncthreads();

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

  // softmax and top-K: warp w takes tokens 4w..4w+3; lane L holds experts
  // L, L+32, ...
#pragma unroll 1
  for (int i = 0; i < kTokPerCta / kRouterWarps; ++i) {
    const int tl = warp * (kTokPerCta / kRouterWarps) + i;
    const int64_t t = t0 + tl;
    if (t >= T) break;  // warp-uniform
    // softmax logits (with the bias unless it only steers the selection)
    // and selection keys
    float lg[EPT], key[EPT];
#pragma unroll
    for (int q = 0; q < EPT; ++q) {
      const int e = lane + 32 * q;
      const float l = sL[tl * LDL + e];
      const float biased = l + b[q];
      lg[q] = e < n ? (select_only ? l : biased) : -CUDART_INF_F;
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
    __syncthreads();  // every warp is done reading the logits
    float* pred = smem_f;  // [kRouterWarps][NP]
#pragma unroll
    for (int q = 0; q < EPT; ++q) pred[warp * NP + lane + 32 * q] = pst[q];
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
      float a = 0.0f;
      for (int ww = 0; ww < kRouterWarps; ++ww) a += pred[ww * NP + e];
      pstat[static_cast<int64_t>(blockIdx.x) * n + e] = a;
    }
  }
}

template <typename TIn, bool STATS>
int launch_router_t(const TIn* u, const TIn* E, const float* bias, int64_t T, int d, int n, int K,
                    int flags, int32_t* idx, float* w, float* pstat, cudaStream_t st) {
  const int ept = (n + 31) / 32;
  const unsigned grid = static_cast<unsigned>((T + kTokPerCta - 1) / kTokPerCta);
  const dim3 block(kRouterThreads);
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
