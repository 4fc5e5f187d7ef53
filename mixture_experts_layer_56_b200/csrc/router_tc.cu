// Router of the DeepSeekMoE layer (§3.2, eqs. (10)-(11)) on the tensor
// cores: the logits l_{t,i} = u_t . e_i of 128 tokens against every routed
// expert are one tcgen05 MMA tile (M = 128 tokens, N = N_r rounded up to 16,
// K = d), bf16 x bf16 with fp32 accumulation in TMEM.  Each product of two
// bf16 values is exact in fp32, so the logits differ from a sequential fp32
// sum only in summation order.
//
// One CTA per 128 tokens, 4 warps.  Warp 0 streams 64-wide column slices
// of u (128 rows) and E (N rows, zero rows past N_r) into a shared-memory
// ring with TMA; warp 1 issues the MMAs; warp 2 owns the TMEM columns.
// Then every thread takes the token of its TMEM lane and works through its
// logits in 32-column chunks read from TMEM:
//   max and sum of the softmax (bias added unless it only steers the
//   selection), then K selection passes, each taking the largest key
//   l + b that comes after the previous pick in (value descending, index
//   ascending) order, so lower indices win ties.  Gates are
//   exp(l - max) / sum, not renormalised over the top K.
// With statistics on, each warp also sums the scores of its 32 tokens per
// expert (fixed token order) for the balance statistics of §3.3.
#include <cuda.h>
#include <math_constants.h>

#include "common.cuh"
#include "gemm_sm100.h"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace moe {

namespace {

using namespace sm100;

constexpr int kRtTokens = 128;  // tokens per CTA: one TMEM lane each
static_assert(kRtTokens == kDispatchChunk, "a router CTA counts exactly one dispatch chunk");
constexpr int kRtThreads = 128;
constexpr int kRtBK = 64;  // columns of d per stage (128 bytes of bf16)
constexpr int kRtMaxStages = 8;
constexpr int kRtSmemBudget = 200 * 1024;
constexpr int kRtTileBytes = kRtTokens * kRtBK * 2;

// 32 consecutive fp32 columns of this thread's TMEM lane from registers
// (shape 32x32b, x32); tmem_st_wait() before the columns are read back
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// 16 bytes / 4 bytes of a cluster peer's shared memory (mapa address)
__device__ __forceinline__ float4 ld_shared_cluster_v4(uint32_t cluster_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}
__device__ __forceinline__ int ld_shared_cluster_s32(uint32_t cluster_addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}

inline int rt_padded_experts(int n) { return (n + 15) / 16 * 16; }
inline int rt_stage_bytes(int np) { return kRtTileBytes + np * kRtBK * 2; }
inline int rt_stages(int np) {
  const int s = kRtSmemBudget / rt_stage_bytes(np);
  return s > kRtMaxStages ? kRtMaxStages : s;
}

// NCH > 0: a token's logits (NCH chunks of 32) stay in registers after one
// TMEM read, SEL = the bias only steers the selection.  NCH = 0: any expert
// count; the chunks are re-read from TMEM for every pass.  CS > 1: a cluster
// of CS CTAs shares one 128-token tile, rank r computing the logits over
// its share of d; rank 0 adds the partials in rank order and selects.
template <bool STATS, int NCH, bool SEL, int CS>
__global__ void __launch_bounds__(kRtThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmE,
                 const float* __restrict__ bias, int64_t T, int d, int n, int np, int K,
                 int flags, int stages, uint32_t tmem_cols, int32_t* __restrict__ idx,
                 float* __restrict__ w, float* __restrict__ pstat, int32_t* status,
                 int32_t* __restrict__ chunk_counts) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * kRtMaxStages + 2];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ float sbias[256];
  __shared__ int hist[256];  // this CTA's tokens per expert (chunk_counts)

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = smem_addr(smem);
  const uint32_t stage_bytes = static_cast<uint32_t>(kRtTileBytes + np * kRtBK * 2);
  const uint32_t bar_base = smem_addr(bars);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (kRtMaxStages + s); };
  const uint32_t done_bar = bar_base + 8u * (2 * kRtMaxStages);
  const uint32_t drain_bar = bar_base + 8u * (2 * kRtMaxStages + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int tile = static_cast<int>(blockIdx.x) / CS;
  const int m0 = tile * kRtTokens;
  const int crank = CS > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int nkb_all = d / kRtBK;
  const int kb0 = crank * nkb_all / CS, kb1 = (crank + 1) * nkb_all / CS;
  const int nkb = kb1 - kb0;
  volatile int* abort_p = &abort_flag;

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(done_bar, 1);
    mbar_init(drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    fence_async_shared();
  }
  if (warp == 2) {
    tmem_alloc(smem_addr(&tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmE);
  }
  pdl_wait();  // u, E, bias and the outputs belong to earlier stream work
  for (int e = tid; e < 256; e += kRtThreads) {
    sbias[e] = (bias != nullptr && e < n) ? bias[e] : 0.0f;
    hist[e] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  const uint32_t idesc = idesc_bf16_f32(kRtTokens, np);

  if (warp == 0) {
    // ---------------------------------------------------- TMA producer ----
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_p, status)) { ok = false; break; }
        const uint32_t sa = smem_base + stage * stage_bytes;
        mbar_arrive_expect_tx(full_bar(stage), stage_bytes);
        tma_load_2d(sa, &tmU, full_bar(stage), (kb0 + i) * kRtBK, m0);
        tma_load_2d(sa + kRtTileBytes, &tmE, full_bar(stage), (kb0 + i) * kRtBK, 0);
        issued |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == stages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) {
        for (int s = 0; s < stages; ++s)
          if (issued & (1u << s)) {
            int dummy = 0;
            wait_bounded(full_bar(s), (issued_parity >> s) & 1u, &dummy, nullptr);
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer ----
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!wait_bounded(full_bar(stage), phase, abort_p, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_base + stage * stage_bytes;
        const uint32_t sb = sa + kRtTileBytes;
#pragma unroll
        for (int k = 0; k < kRtBK / 16; ++k)
          mma_bf16(tmem_base, desc_kmajor_sw128(sa + k * 32), desc_kmajor_sw128(sb + k * 32), idesc,
                   (kb > 0 || k > 0) ? 1u : 0u);
        // only stages that are loaded again need an "empty" arrival; the
        // last round's would otherwise still be in flight when the CTA exits
        if (kb + stages < nkb) mma_commit(empty_bar(stage));
        if (++stage == stages) { stage = 0; phase ^= 1u; }
      }
      if (ok) {
        mma_commit(done_bar);
      } else {
        mma_commit(drain_bar);
        int dummy = 0;
        wait_bounded(drain_bar, 0, &dummy, nullptr);
      }
    }
    __syncwarp();
  }

  // ------------------------------------------------ softmax and top-K ------
  pdl_trigger();
  bool got = __all_sync(0xffffffffu, wait_bounded(done_bar, 0, abort_p, status) ? 1 : 0);
  tc_fence_after();
  const int r = warp * 32 + lane;
  const int64_t t = static_cast<int64_t>(m0) + r;
  const bool live = t < T;
  const uint32_t trow = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
  const int nch = (np + 31) / 32;
  const bool select_only = (flags & MOE_FLAG_BIAS_SELECT_ONLY) != 0;
  bool selects = true;  // this CTA runs the softmax and selection

  if constexpr (CS > 1) {
    // Each rank's partial logits go to its own shared memory (the ring is
    // free: every MMA that read it has completed).  Rank 0 adds the ranks'
    // partials in rank order and writes the sums into its TMEM, where the
    // selection below reads them.  Every CTA reaches both cluster barriers.
    // Only rows of real tokens move (one row at T = 1).
    __shared__ int got_flag;
    const int ldp = nch * 32 + 4;
    float* part = reinterpret_cast<float*>(smem);
    const bool warp_live = __any_sync(0xffffffffu, live);
    if (got && warp_live) {
      for (int c = 0; c < nch; ++c) {
        float x[32];
        tmem_ld32(trow + c * 32, x);
        tmem_ld_wait_regs(x);
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(part + r * ldp + c * 32 + j) =
              make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
      }
    }
    const bool cta_got = __syncthreads_and(got ? 1 : 0) != 0;
    if (tid == 0) got_flag = cta_got ? 1 : 0;
    cluster_sync_all();
    if (crank == 0) {
      int all = 1;
      for (int rk = 0; rk < CS; ++rk) all &= ld_shared_cluster_s32(map_to_cta(smem_addr(&got_flag), rk));
      got = all != 0;
      if (got && warp_live) {
        for (int c = 0; c < nch; ++c) {
          float x[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) x[j] = 0.0f;
          for (int rk = 0; rk < (live ? CS : 0); ++rk) {
            const uint32_t row = map_to_cta(smem_addr(part + r * ldp + c * 32), rk);
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float4 v = ld_shared_cluster_v4(row + j * 4);
              x[j] += v.x;
              x[j + 1] += v.y;
              x[j + 2] += v.z;
              x[j + 3] += v.w;
            }
          }
          tmem_st32(trow + c * 32, x);
        }
        tmem_st_wait();
      }
    }
    cluster_sync_all();  // the peers' partials stay until rank 0 has read them
    selects = crank == 0;
  }

  if (!selects) {
    // a peer rank: its share of the logits is with rank 0
  } else if (!got) {
    // results stay in range for the stages downstream; the status word says
    // that they are not to be used
    if (live)
      for (int k = 0; k < K; ++k) {
        idx[t * K + k] = k;
        w[t * K + k] = 0.0f;
        if (chunk_counts) atomicAdd(&hist[k], 1);
      }
  } else if (NCH == 0) {
    float m = -CUDART_INF_F;
#pragma unroll 1
    for (int c = 0; c < nch; ++c) {
      float x[32];
      tmem_ld32(trow + c * 32, x);
      tmem_ld_wait_regs(x);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int e = c * 32 + j;
        if (e < n) m = fmaxf(m, select_only ? x[j] : x[j] + sbias[e]);
      }
    }
    float z = 0.0f;
#pragma unroll 1
    for (int c = 0; c < nch; ++c) {
      float x[32];
      tmem_ld32(trow + c * 32, x);
      tmem_ld_wait_regs(x);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int e = c * 32 + j;
        if (e < n) z += expf((select_only ? x[j] : x[j] + sbias[e]) - m);
      }
    }
    const float inv_z = 1.0f / z;

    float pv = CUDART_INF_F;  // previous pick (key, index)
    int pe = -1;
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
      float bv = -CUDART_INF_F, blg = 0.0f;
      int bi = -1;
#pragma unroll 1
      for (int c = 0; c < nch; ++c) {
        float x[32];
        tmem_ld32(trow + c * 32, x);
        tmem_ld_wait_regs(x);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int e = c * 32 + j;
          const float key = x[j] + sbias[e];
          const bool after = key < pv || (key == pv && e > pe);
          if (e < n && after && (bi < 0 || key > bv)) {
            bv = key;
            bi = e;
            blg = select_only ? x[j] : key;
          }
        }
      }
      if (live) {
        idx[t * K + k] = bi;
        w[t * K + k] = expf(blg - m) * inv_z;
        if (chunk_counts && bi >= 0) atomicAdd(&hist[bi], 1);
      }
      pv = bv;
      pe = bi;
    }

    if (STATS) {
      // scores of this warp's 32 tokens, transposed through shared memory
      // (the ring is free: every MMA that read it has completed)
      const int ld = np + 1;
      float* sc = reinterpret_cast<float*>(smem) + warp * 32 * ld;
#pragma unroll 1
      for (int c = 0; c < nch; ++c) {
        float x[32];
        tmem_ld32(trow + c * 32, x);
        tmem_ld_wait_regs(x);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int e = c * 32 + j;
          if (e < np)
            sc[lane * ld + e] =
                (live && e < n) ? expf((select_only ? x[j] : x[j] + sbias[e]) - m) / z : 0.0f;
        }
      }
      __syncwarp();
      const int64_t g = static_cast<int64_t>(tile) * (kRtTokens / 32) + warp;
      if (g * 32 < T) {
        for (int e = lane; e < n; e += 32) {
          float a = 0.0f;
          for (int tok = 0; tok < 32; ++tok) a += sc[tok * ld + e];
          pstat[g * n + e] = a;
        }
      }
    }
  } else {
    // logits -> selection keys (and, with SEL, the softmax logits) in registers
    constexpr int NR = (NCH > 0 ? NCH : 1) * 32;
    float key[NR];
    float lg[SEL ? NR : 1];
#pragma unroll
    for (int c = 0; c < NR / 32; ++c) tmem_ld32(trow + c * 32, key + c * 32);
#pragma unroll
    for (int c = 0; c < NR / 32; ++c) tmem_ld_wait_regs(key + c * 32);
    // four interleaved chains (j mod 4) keep the scans short in latency
    constexpr int NB = 4;
    float mb[NB];
#pragma unroll
    for (int q = 0; q < NB; ++q) mb[q] = -CUDART_INF_F;
#pragma unroll
    for (int j = 0; j < NR; ++j) {
      if (SEL) lg[j] = j < n ? key[j] : -CUDART_INF_F;
      key[j] = j < n ? key[j] + sbias[j] : -CUDART_INF_F;
      mb[j % NB] = fmaxf(mb[j % NB], SEL ? lg[j] : key[j]);
    }
    const float m = fmaxf(fmaxf(mb[0], mb[1]), fmaxf(mb[2], mb[3]));
    float zb[NB];
#pragma unroll
    for (int q = 0; q < NB; ++q) zb[q] = 0.0f;
#pragma unroll
    for (int j = 0; j < NR; ++j) zb[j % NB] += expf((SEL ? lg[j] : key[j]) - m);
    const float z = (zb[0] + zb[1]) + (zb[2] + zb[3]);
    const float inv_z = 1.0f / z;

    if (STATS) {
      const int ld = np + 1;
      float* sc = reinterpret_cast<float*>(smem) + warp * 32 * ld;
#pragma unroll
      for (int j = 0; j < NR; ++j)
        if (j < np) sc[lane * ld + j] = (live && j < n) ? expf((SEL ? lg[j] : key[j]) - m) / z : 0.0f;
      __syncwarp();
      const int64_t g = static_cast<int64_t>(tile) * (kRtTokens / 32) + warp;
      if (g * 32 < T) {
        for (int e = lane; e < n; e += 32) {
          float a = 0.0f;
          for (int tok = 0; tok < 32; ++tok) a += sc[tok * ld + e];
          pstat[g * n + e] = a;
        }
      }
    }

    // K passes; each takes the largest remaining key (lower index first on
    // equal keys) and removes it from the next pass
    int prev = -1;
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
      float bv[NB], bl[NB];
      int bi[NB];
#pragma unroll
      for (int q = 0; q < NB; ++q) {
        bv[q] = -CUDART_INF_F;
        bl[q] = 0.0f;
        bi[q] = 0x7fffffff;
      }
#pragma unroll
      for (int j = 0; j < NR; ++j) {
        const int q = j % NB;
        const float kj = (j == prev) ? -CUDART_INF_F : key[j];
        key[j] = kj;
        if (kj > bv[q]) {
          bv[q] = kj;
          bi[q] = j;
          if (SEL) bl[q] = lg[j];
        }
      }
      // merge the chains: larger key, then lower index
      float v = bv[0], l = bl[0];
      int e = bi[0];
#pragma unroll
      for (int q = 1; q < NB; ++q) {
        if (bv[q] > v || (bv[q] == v && bi[q] < e)) {
          v = bv[q];
          e = bi[q];
          l = bl[q];
        }
      }
      if (live) {
        idx[t * K + k] = e;
        w[t * K + k] = expf((SEL ? l : v) - m) * inv_z;
        if (chunk_counts && e < n) atomicAdd(&hist[e], 1);
      }
      prev = e;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
  if (chunk_counts && crank == 0)
    for (int e = tid; e < n; e += kRtThreads)
      chunk_counts[static_cast<int64_t>(tile) * n + e] = hist[e];
}

}  // namespace

int launch_router_tc(const void* u, const void* E, const float* bias, int64_t T, int d, int n,
                     int K, int flags, int32_t* idx, float* w, float* pstat, int32_t* status,
                     int32_t* chunk_counts, cudaStream_t st) {
  if (T == 0) return MOE_OK;
  if (d % kRtBK != 0 || n < 1 || n > 256) return MOE_ERR_SHAPE;
  const int np = rt_padded_experts(n);
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(np)) cols *= 2;
  const int stages = rt_stages(np);
  const int smem = stages * rt_stage_bytes(np) + 1024;
  CUtensorMap mu, me;
  if (!make_map_2d(&mu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, u, static_cast<uint64_t>(d),
                   static_cast<uint64_t>(T), static_cast<uint64_t>(d) * 2, kRtBK, kRtTokens) ||
      !make_map_2d(&me, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, E, static_cast<uint64_t>(d),
                   static_cast<uint64_t>(n), static_cast<uint64_t>(d) * 2, kRtBK,
                   static_cast<uint32_t>(np)))
    return MOE_ERR_CUDA;
  const int64_t tiles = (T + kRtTokens - 1) / kRtTokens;
  // few tiles (short batches): split d over a cluster so that more SMs
  // stream u and E; with many tiles every SM is busy and the exchange of
  // partial logits would only add work
  static int sm_count[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  if (sm_count[dev] == 0 &&
      cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  int cs = 1;
  if (!pstat && tiles <= 16)
    while (cs < 8 && tiles * cs * 2 <= sm_count[dev] && d / kRtBK >= 2 * cs) cs *= 2;
  auto go = [&](auto kern, std::atomic<uint64_t>& optin, unsigned cl) -> int {
    // one opt-in size covering every expert count (smem never exceeds it)
    if (int rc = ensure_smem_optin(reinterpret_cast<const void*>(kern), kRtSmemBudget + 1024, optin))
      return rc;
    return launch_k(kern, dim3(static_cast<unsigned>(tiles) * cl), kRtThreads,
                    static_cast<size_t>(smem), st, cl, mu, me, bias, T, d, n, np, K, flags, stages,
                    cols, idx, w, pstat, status, chunk_counts);
  };
  const bool sel = (flags & MOE_FLAG_BIAS_SELECT_ONLY) != 0;
  const int nch = (np + 31) / 32;
  // register-resident variants up to 64 experts (128 without SEL)
  // (with statistics, beyond 64 experts the register variant would spill)
  const int v = (nch <= 2 || (nch <= 4 && !sel && !pstat)) ? nch : 0;
#define MOE_RT_GO(STATS, NCH, SEL)                                                   \
  {                                                                                  \
    static std::atomic<uint64_t> done1{0}, done2{0}, done4{0}, done8{0};            \
    if (STATS || cs == 1) return go(router_tc_kernel<STATS, NCH, SEL, 1>, done1, 1u); \
    if (cs == 2) return go(router_tc_kernel<STATS, NCH, SEL, (STATS ? 1 : 2)>, done2, 2u); \
    if (cs == 4) return go(router_tc_kernel<STATS, NCH, SEL, (STATS ? 1 : 4)>, done4, 4u); \
    return go(router_tc_kernel<STATS, NCH, SEL, (STATS ? 1 : 8)>, done8, 8u);        \
  }
#define MOE_RT_VARIANTS(STATS)                                      \
  if (v == 1 && sel) MOE_RT_GO(STATS, 1, true)                      \
  if (v == 1) MOE_RT_GO(STATS, 1, false)                            \
  if (v == 2 && sel) MOE_RT_GO(STATS, 2, true)                      \
  if (v == 2) MOE_RT_GO(STATS, 2, false)                            \
  if (v == 3) MOE_RT_GO(STATS, (STATS ? 0 : 3), false)              \
  if (v == 4) MOE_RT_GO(STATS, (STATS ? 0 : 4), false)              \
  MOE_RT_GO(STATS, 0, false)
  if (pstat) {
    MOE_RT_VARIANTS(true)
  } else {
    MOE_RT_VARIANTS(false)
  }
#undef MOE_RT_VARIANTS
#undef MOE_RT_GO
}

}  // namespace moe
