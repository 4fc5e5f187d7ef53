// Router of the DeepSeekMoE layer (§3.2, eqs. (10)-(11)): fp32 logits
// l_{t,i} = sum_j u_{t,j} e_{i,j} (+ b_i) on CUDA cores, softmax over the
// routed experts and top-K selection with warp shuffles.  It serves the fp32
// layer and, with MOE_FLAG_ROUTER_SIMT, bf16; bf16 routes on the tensor cores
// by default (router_tc.cu), and launch_router below picks between them.
//
// A CTA owns 32 tokens and all experts.  A producer warp streams 128-byte
// column slices of u (32 rows) and E (NP rows) into a 4-stage shared-memory
// ring with TMA (128-byte swizzle, rows past the matrix read as zeros), so
// the loads of later slices are in flight while earlier ones are multiplied,
// without costing registers.  The 256 compute threads form two halves; each
// half sums one half of every slice, thread h owning the outer-product tile
// tokens {h%8 + 8i} x experts {h/8 + 16m}, so a warp's shared loads are one
// wavefront each.  Per logit every half is one fp32 FMA chain in increasing
// j and the two halves are added once at the end, the same order for every
// expert, so equal centroids give bitwise-equal logits.  The selection runs
// on logits (softmax is monotone), lower index first on ties; gates are
// exp(l - max) / sum, not renormalised over the top K.
#include <cuda.h>
#include <math_constants.h>

#include "common.cuh"
#include "gemm_sm100.h"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace moe {

namespace {

using namespace sm100;

constexpr int kRouterWarps = 8;                   // compute warps (two halves of 4)
constexpr int kRouterThreads = kRouterWarps * 32 + 32;  // + one producer warp
constexpr int kTokPerCta = 32;
constexpr int kRouterStages = 4;

template <int EPT>
constexpr int router_stage_bytes() {
  return (kTokPerCta + EPT * 32) * 128;
}
template <int EPT>
constexpr int router_smem_bytes() {
  return kRouterStages * router_stage_bytes<EPT>() + 1024;
}

// element v of a 16-byte chunk of 8 bf16 / 4 fp32 values, as fp32
template <typename TIn>
__device__ __forceinline__ float chunk_elem(const uint4& c, int v);
template <>
__device__ __forceinline__ float chunk_elem<bf16>(const uint4& c, int v) {
  const uint32_t w = v < 2 ? c.x : v < 4 ? c.y : v < 6 ? c.z : c.w;
  return __uint_as_float((v & 1) ? (w & 0xffff0000u) : (w << 16));
}
template <>
__device__ __forceinline__ float chunk_elem<float>(const uint4& c, int v) {
  return __uint_as_float(v == 0 ? c.x : v == 1 ? c.y : v == 2 ? c.z : c.w);
}

// 16-byte chunk ch of row `row` of a TMA tile with 128-byte rows and
// 128-byte swizzle (tile base 1024-byte aligned)
__device__ __forceinline__ uint4 lds_sw128(const uint8_t* tile, int row, int ch) {
  return *reinterpret_cast<const uint4*>(tile + row * 128 + ((ch ^ (row & 7)) << 4));
}

template <typename TIn, int EPT, bool STATS, int CS>
__global__ void __launch_bounds__(kRouterThreads)
router_topk_kernel(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmE,
                   const float* __restrict__ bias, int64_t T, int d, int n, int K, int flags,
                   int32_t* __restrict__ idx, float* __restrict__ w, float* __restrict__ pstat) {
  constexpr int NP = EPT * 32;
  constexpr int XPT = 2 * EPT;                 // experts per thread
  constexpr int VPC = 16 / sizeof(TIn);        // values per 16-byte chunk
  constexpr int KC = 8 * VPC;                  // columns per stage (128-byte rows)
  constexpr uint32_t U_BYTES = kTokPerCta * 128;
  constexpr uint32_t ST_BYTES = router_stage_bytes<EPT>();
  constexpr int LDL = NP + 1;                  // logits row length (floats)
  static_assert(kRouterStages * ST_BYTES >= kTokPerCta * LDL * 4, "logits fit the ring");

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * kRouterStages];
  __shared__ int abort_flag;
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* sL = reinterpret_cast<float*>(ring);  // [kTokPerCta][LDL], after the d loop
  const uint32_t ring_base = smem_addr(ring);
  const uint32_t bar_base = smem_addr(bars);
  auto full_bar = [&](int st) { return bar_base + 8u * st; };
  auto empty_bar = [&](int st) { return bar_base + 8u * (kRouterStages + st); };

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // a cluster of CS CTAs shares 32 tokens; CTA `rank` sums its share of d
  const uint32_t rank = CS > 1 ? cluster_ctarank() : 0;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x / CS) * kTokPerCta;
  const int nall = (d + KC - 1) / KC;
  const int cbeg = static_cast<int>(rank) * nall / CS;
  const int nchunks = (static_cast<int>(rank) + 1) * nall / CS - cbeg;
  volatile int* abort_p = &abort_flag;

  if (tid == 0) {
    for (int st = 0; st < kRouterStages; ++st) {
      mbar_init(full_bar(st), 1);
      mbar_init(empty_bar(st), kRouterWarps);
    }
    abort_flag = 0;
    fence_mbar_init();
    fence_async_shared();
  }
  __syncthreads();

  float acc[4][XPT];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int m = 0; m < XPT; ++m) acc[i][m] = 0.0f;

  if (warp == kRouterWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmU);
      tma_prefetch_desc(&tmE);
      for (int c = 0; c < nchunks; ++c) {
        const int st = c % kRouterStages;
        const uint32_t ph = (c / kRouterStages) & 1;
        if (!wait_bounded(empty_bar(st), ph ^ 1u, abort_p, nullptr)) break;
        const uint32_t sb = ring_base + st * ST_BYTES;
        mbar_arrive_expect_tx(full_bar(st), ST_BYTES);
        tma_load_2d(sb, &tmU, full_bar(st), (cbeg + c) * KC, static_cast<int32_t>(t0));
        tma_load_2d(sb + U_BYTES, &tmE, full_bar(st), (cbeg + c) * KC, 0);
      }
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------------- FMAs
    const int half = tid >> 7;  // which 4 of the 8 chunks of every slice
    const int hh = tid & 127;
    const int tg = hh & 7;      // tokens tg + 8i
    const int eg = hh >> 3;     // experts eg + 16m
    for (int c = 0; c < nchunks; ++c) {
      const int st = c % kRouterStages;
      const uint32_t ph = (c / kRouterStages) & 1;
      if (!wait_bounded(full_bar(st), ph, abort_p, nullptr)) break;
      const uint8_t* uT = ring + st * ST_BYTES;
      const uint8_t* eT = uT + U_BYTES;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int ch = half * 4 + q;
        uint4 ur[4], er[XPT];
#pragma unroll
        for (int i = 0; i < 4; ++i) ur[i] = lds_sw128(uT, tg + 8 * i, ch);
#pragma unroll
        for (int m = 0; m < XPT; ++m) er[m] = lds_sw128(eT, eg + 16 * m, ch);
#pragma unroll
        for (int v = 0; v < VPC; ++v) {
          float uf[4], ef[XPT];
#pragma unroll
          for (int i = 0; i < 4; ++i) uf[i] = chunk_elem<TIn>(ur[i], v);
#pragma unroll
          for (int m = 0; m < XPT; ++m) ef[m] = chunk_elem<TIn>(er[m], v);
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int m = 0; m < XPT; ++m) acc[i][m] = fmaf(uf[i], ef[m], acc[i][m]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(st));
    }
  }

  // logits = first-half sums + second-half sums, into [token][expert]
  __syncthreads();  // every stage consumed; the ring is free
  const int half = tid >> 7;
  const int hh = tid & 127;
  const int tg = hh & 7;
  const int eg = hh >> 3;
  if (warp < kRouterWarps && half == 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int m = 0; m < XPT; ++m) sL[(tg + 8 * i) * LDL + eg + 16 * m] = acc[i][m];
  }
  __syncthreads();
  if (warp < kRouterWarps && half == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int m = 0; m < XPT; ++m) {
        float* p = sL + (tg + 8 * i) * LDL + eg + 16 * m;
        *p = acc[i][m] + *p;
      }
  }
  __syncthreads();
  if (CS > 1) {
    // rank 0 adds the other CTAs' partial logits, in rank order, through
    // distributed shared memory
    cluster_sync_all();
    if (rank == 0) {
      const uint32_t base = smem_addr(sL);
      for (int i = tid; i < kTokPerCta * LDL; i += blockDim.x) {
        float a = sL[i];
        for (int r = 1; r < CS; ++r) a += ld_shared_cluster_f32(map_to_cta(base + 4u * i, r));
        sL[i] = a;
      }
    }
    cluster_sync_all();  // the peers' logits stay alive until read
    if (rank != 0) return;
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

  // softmax and top-K: warp w takes tokens 4w..4w+3; lane L holds experts
  // L, L+32, ...
#pragma unroll 1
  for (int i = 0; i < kTokPerCta / kRouterWarps; ++i) {
    const int tl = warp * (kTokPerCta / kRouterWarps) + i;
    const int64_t t = t0 + tl;
    if (warp >= kRouterWarps || t >= T) break;  // warp-uniform; the producer has no tokens
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
    float* pred = sL;  // [kRouterWarps][NP]
    if (warp < kRouterWarps) {
#pragma unroll
      for (int q = 0; q < EPT; ++q) pred[warp * NP + lane + 32 * q] = pst[q];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
      float a = 0.0f;
      for (int ww = 0; ww < kRouterWarps; ++ww) a += pred[ww * NP + e];
      pstat[static_cast<int64_t>(blockIdx.x / CS) * n + e] = a;
    }
  }
}

template <typename TIn, bool STATS>
int launch_router_t(const TIn* u, const TIn* E, const float* bias, int64_t T, int d, int n, int K,
                    int flags, int32_t* idx, float* w, float* pstat, cudaStream_t st) {
  const int ept = (n + 31) / 32;
  const unsigned grid = static_cast<unsigned>((T + kTokPerCta - 1) / kTokPerCta);
  const dim3 block(kRouterThreads);
  constexpr int VPC = 16 / sizeof(TIn);
  const CUtensorMapDataType dt =
      sizeof(TIn) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUtensorMap mu, me;
  if (!make_map_2d(&mu, dt, u, static_cast<uint64_t>(d), static_cast<uint64_t>(T),
                   static_cast<uint64_t>(d) * sizeof(TIn), 8 * VPC, kTokPerCta) ||
      !make_map_2d(&me, dt, E, static_cast<uint64_t>(d), static_cast<uint64_t>(n),
                   static_cast<uint64_t>(d) * sizeof(TIn), 8 * VPC, 32 * ept))
    return MOE_ERR_CUDA;
  // small batches: split d over a cluster of CS CTAs so that more SMs work
  const int nall = static_cast<int>((d + 8 * VPC - 1) / (8 * VPC));
  int cs = 1;
  while (cs < 8 && static_cast<int64_t>(grid) * cs * 2 <= 148 && cs * 2 <= nall) cs *= 2;
  auto launch = [&](auto kern, int smem) -> int {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid * cs, 1, 1);
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mu, me, bias, T, d, n, K, flags, idx, w, pstat) ==
                   cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
  };
  int rc = MOE_OK;
#define MOE_ROUTER_CASE(N)                                                                  \
  case N:                                                                                   \
    rc = cs == 8   ? launch(router_topk_kernel<TIn, N, STATS, 8>, router_smem_bytes<N>())    \
         : cs == 4 ? launch(router_topk_kernel<TIn, N, STATS, 4>, router_smem_bytes<N>())    \
         : cs == 2 ? launch(router_topk_kernel<TIn, N, STATS, 2>, router_smem_bytes<N>())    \
                   : launch(router_topk_kernel<TIn, N, STATS, 1>, router_smem_bytes<N>());   \
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
  if (rc) return rc;
  count_launch();
  return check_launch();
}

}  // namespace

int router_num_ctas(int64_t T) { return static_cast<int>((T + kTokPerCta - 1) / kTokPerCta); }

int launch_router(int dtype, const void* u, const void* E, const float* bias, int64_t T, int d,
                  int n, int K, int flags, int32_t* idx, float* w, float* pstat,
                  int32_t* status, cudaStream_t st, int32_t* chunk_counts, bool* counted) {
  if (counted) *counted = false;
  if (T == 0) return MOE_OK;
  if (dtype == MOE_DTYPE_BF16 && !(flags & MOE_FLAG_ROUTER_SIMT)) {
    if (counted) *counted = chunk_counts != nullptr;
    return launch_router_tc(u, E, bias, T, d, n, K, flags, idx, w, pstat, status, chunk_counts,
                            st);
  }
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
