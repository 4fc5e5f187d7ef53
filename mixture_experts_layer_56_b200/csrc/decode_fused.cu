// The whole DeepSeekMoE layer (§3.2, eqs. (9)-(11)) for decode-sized batches
// (T <= kDecMaxT tokens) in one persistent kernel.
//
// At a handful of tokens the layer is a stream of the activated experts'
// weights (W1/W3/W2 of every routed expert some token chose, plus the shared
// experts, all read once), so what matters is that every SM streams weights
// all the time.  The work is cut into units: one unit is kDecUC = 64
// intermediate rows of one expert, i.e. one 128-row packed W13 block
// [gate 64 | up 64] and the matching 64 columns of W2.  CTAs take units from
// an atomic counter, so the units spread evenly over the SMs whatever the
// routing; each unit writes fp32 partial down projections into slots fixed by
// the unit, and the sums below run in a fixed order, so the result does not
// depend on which CTA took which unit.
//
// A unit on the tensor cores (weights as the M = 128 operand, the batch's
// tokens as N = 16 columns, fp32 accumulators in TMEM):
//   gate/up  D1[128 x 16] = W13 block [128 x d] . U^T, U = all tokens (bf16,
//            zero rows past T), in d/64 MMA steps; each ring stage brings a
//            W13 tile and the tokens' tile of the same 64 columns;
//   SwiGLU   a[r, t] = SiLU(D1[r, t]) * D1[64 + r, t]   (r < 64), bf16;
//   down     D2[m][128 x 16] = W2[m*128 .. +127, chunk cols] . a, d/128 tiles;
//   store    the columns of the unit's own tokens (its expert's tokens, or all
//            of them for a shared expert) as partial rows.
// Roles (8 warps): warp 0 the TMA producer (unit counter, W13 and W2 tiles into
// an 11-stage ring, running ahead into the next unit), warp 1 the MMA issuer,
// warp 2 the TMEM owner, warps 2-7 the routing of every token and warp 3 the
// expert tables (phase 2), then warps 4-7 the epilogue (TMEM lane quarters).
// The ring carries unit i's W13 tiles before unit i-1's W2 tiles, and D1 is
// double-buffered, so unit i's gate/up MMAs run while the epilogue turns
// unit i-1's D1 into a^T.
//
// Phases, all in this one launch (one CTA per SM):
//  1. Logits (with G = min(n, grid), CTA c < G takes experts c, c + G, ...):
//     expert i's row stays in registers while each warp takes two tokens,
//     u_t . e_i as fp32 FMA chains per lane plus a fixed shuffle tree; the
//     CTA publishes its logits and counts itself.
//  2. Routing and tables (warps 2-7 of every CTA, the same arithmetic in
//     each): once every logit CTA is counted, softmax of each token over the
//     routed experts (fixed-order max and sum) and its top K by rank among
//     the keys (larger first, lower index first on ties; gates not
//     renormalised); then each slot's rank within its expert in slot order
//     (warp match / popc, 32 slots at a time), the experts' offsets and the
//     active list from warp scans; the producer is released through an
//     mbarrier.
//  3. Units: the shared experts' units need no routing and come first; the
//     routed units (active experts in increasing index, chunks in order)
//     wait for the tables.
//  4. Combine: once every unit is done, h_t = u_t + sum_j g_j p_j over the
//     token's partial rows p_j (the shared units' with g = 1, then each
//     routed slot k's chunks with g = w[t,k]), in fp32: one CTA per (token,
//     256 columns), warp w summing rows w, w + 8, ... in order (coalesced
//     row segments, 8 rows' loads in flight), then the 8 warps' sums in warp
//     order; u is added last and h rounded once to bf16.
// Every wait is bounded: a wait that runs out records MOE_ERR_DEVICE_CHECK in
// the status word and the kernel winds down without writing h.
#include <cuda.h>
#include <math_constants.h>

#include "common.cuh"
#include "decode_fused.h"
#include "gemm_sm100.h"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace moe {

namespace {

using namespace sm100;

constexpr int kDecThreads = 256;                     // 8 warps
constexpr int kDecUC = 64;                           // intermediate rows per unit
constexpr int kDecN = 16;                            // token columns of an MMA
constexpr int kDecTileBytes = 128 * 64 * 2;          // one 128 x 64 bf16 TMA tile
constexpr int kDecUTileBytes = 16 * 64 * 2;          // the tokens' 64 columns (16 rows)
constexpr int kDecStageBytes = kDecTileBytes + kDecUTileBytes;
constexpr int kDecStages = 11;
constexpr int kDecQueue = 4;                         // unit descriptors in flight
constexpr int kRouteWarps = 6;                       // warps 2-7 route the tokens
constexpr int kDecMaxSlots = kDecMaxT * 32;          // routed (token, k) slots
constexpr uint32_t kDecTmemCols = 512;               // D1 (2 x 16) + D2 (16 per 128 rows of d)
static_assert(kDecMaxT <= kDecN, "the batch fits one MMA's columns");

// sync words of the decode scratch (zeroed before each launch)
struct DecSync {
  int unit_next;      // next unit to take
  int logit_ctas;     // CTAs whose logits are published
  int units_done;     // units whose partials are written
  int pad;
};

struct DecArgs {
  const bf16* u;        // [T, d]
  const bf16* E;        // [n, d]
  const float* bias;    // [n] or null
  bf16* h;              // [T, d]
  int32_t* idx;         // [T, K] (workspace)
  float* w;             // [T, K] (workspace)
  float* logits;        // [T, n] (workspace)
  float* part;          // partial rows [rows, d] (workspace)
  DecSync* sync;
  int32_t* status;
  int T, d, n, Ks, I, K, flags;
};

struct __align__(16) UnitDesc {
  int kind;      // 0 shared, 1 routed, -1 no more units
  int expert;    // routed expert e, or shared expert s
  int chunk;     // which kDecUC rows of I
  int slot;      // first partial row
  int8_t row_of[kDecN];  // token t -> its row within the unit's slots, or -1
};

__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, 128;" ::: "memory");  // the 4 epilogue warps
}

// The 4 epilogue warps vote: true when all of them pass true.  Each of them
// reaches every vote once, whatever its own wait saw, so they leave the unit
// loop together also when a wait runs out.
__device__ __forceinline__ bool epi_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

// The routing warps 2-7 vote (named barrier 2): true when all 192 threads
// pass true.
__device__ __forceinline__ bool route_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 2, 192, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

// a bounded mbarrier wait taken by a whole warp, with one result for it
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          int32_t* status) {
  return __all_sync(0xffffffffu, wait_bounded(bar, parity, abort, status) ? 1 : 0) != 0;
}

// bounded spin on a global word until it reaches `target` (acquire)
__device__ __forceinline__ bool spin_until(const int* p, int target, int32_t* status) {
  const uint64_t t0 = global_timer_ns();
  uint32_t spins = 0;
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    if (v >= target) return true;
    if ((++spins & 63u) == 0 && global_timer_ns() - t0 > kWaitTimeoutNs) {
      record_status(status, MOE_ERR_DEVICE_CHECK);
      return false;
    }
    __nanosleep(64);
  }
}

__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// Each weight tile is read once per launch: its L2 lines go first, so that
// the partial rows (written during the units, read back by the combine), the
// tokens' tiles and the router's inputs stay in L2 while the weights stream.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void tma_load_2d_evict_first(uint32_t dst, const CUtensorMap* map,
                                                        uint32_t bar, int32_t x, int32_t y,
                                                        uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// Softmax and top-K of tokens t0, t0 + tstep, ... < T, one warp; lane l holds
// experts l, l + 32, ..., l + 32 (NQ - 1) (NQ * 32 >= n).  keys: this warp's
// shared row of 4 * ceil(n / 4) floats.  Each selected expert e of token t
// goes to slot rank(e), its rank among the keys (larger first, lower index
// first on ties); gates are exp(l_e - max) / sum, not renormalised.
template <int NQ>
__device__ __forceinline__ void route_tokens(const float* logits, const float* bias, int n, int K,
                                             int T, int t0, int tstep, bool select_only,
                                             float* keys, int* sidx, float* sw, int32_t* gidx,
                                             float* gw) {
  const int lane = threadIdx.x & 31;
  const int n4 = (n + 3) & ~3;
  float b[NQ], nxt[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int e = lane + 32 * q;
    b[q] = (bias && e < n) ? bias[e] : 0.0f;
    nxt[q] = (t0 < T && e < n) ? __ldcg(logits + t0 * n + e) : 0.0f;
  }
#pragma unroll 1
  for (int t = t0; t < T; t += tstep) {
    float key[NQ], lg[NQ];
    float m = -CUDART_INF_F;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = lane + 32 * q;
      const float raw = nxt[q];
      nxt[q] = (t + tstep < T && e < n) ? __ldcg(logits + (t + tstep) * n + e) : 0.0f;
      key[q] = e < n ? raw + b[q] : -CUDART_INF_F;
      lg[q] = e < n ? (select_only ? raw : key[q]) : -CUDART_INF_F;
      if (e < n4) keys[e] = key[q];
      m = fmaxf(m, lg[q]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float ex[NQ], z = 0.0f;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      ex[q] = lane + 32 * q < n ? expf(lg[q] - m) : 0.0f;
      z += ex[q];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const float inv_z = 1.0f / z;
    __syncwarp();
    int rank[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) rank[q] = 0;
    const float4* k4 = reinterpret_cast<const float4*>(keys);
#pragma unroll 2
    for (int j4 = 0; j4 < n4 / 4; ++j4) {
      const float4 v = k4[j4];
      const int j = 4 * j4;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int e = lane + 32 * q;
        const float kq = key[q];
        rank[q] += static_cast<int>(v.x > kq) | (static_cast<int>(v.x == kq) & static_cast<int>(j < e));
        rank[q] += static_cast<int>(v.y > kq) | (static_cast<int>(v.y == kq) & static_cast<int>(j + 1 < e));
        rank[q] += static_cast<int>(v.z > kq) | (static_cast<int>(v.z == kq) & static_cast<int>(j + 2 < e));
        rank[q] += static_cast<int>(v.w > kq) | (static_cast<int>(v.w == kq) & static_cast<int>(j + 3 < e));
      }
    }
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = lane + 32 * q;
      if (e < n && rank[q] < K) {
        const float g = ex[q] * inv_z;
        sidx[t * K + rank[q]] = e;
        sw[t * K + rank[q]] = g;
        if (gidx) {
          gidx[t * K + rank[q]] = e;
          gw[t * K + rank[q]] = g;
        }
      }
    }
    __syncwarp();  // keys[] is rewritten for the next token
  }
}

// byte offset of element (row, k) in a K-major [rows x 64] bf16 tile with
// 128-byte swizzle (16-byte chunk k/8 of a row sits at chunk (k/8) ^ (row % 8))
__device__ __forceinline__ uint32_t sw128_off(int row, int k) {
  return static_cast<uint32_t>(row * 128 + ((((k >> 3) ^ (row & 7)) & 7) << 4) + (k & 7) * 2);
}

template <int NV>
__global__ void __launch_bounds__(kDecThreads, 1)
decode_layer_kernel(const __grid_constant__ CUtensorMap tmW13,
                    const __grid_constant__ CUtensorMap tmW13s,
                    const __grid_constant__ CUtensorMap tmW2,
                    const __grid_constant__ CUtensorMap tmW2s,
                    const __grid_constant__ CUtensorMap tmU, const DecArgs a) {
  constexpr int D = NV * 256;        // hidden size
  constexpr int KB13 = D / 64;       // gate/up k-blocks per unit
  constexpr int MT2 = D / 128;       // down row tiles per unit
  constexpr uint32_t IDESC = idesc_bf16_f32(128, kDecN);
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * kDecStages + 2 * kDecQueue + 6];
  __shared__ UnitDesc qdesc[kDecQueue];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int s_cnt[256], s_off[257], s_active[256];
  __shared__ int s_tok[kDecMaxSlots];             // tokens of each expert, increasing t
  __shared__ int s_rank[kDecMaxSlots];            // rank of token t within expert idx[t,k]
  __shared__ int s_idx[kDecMaxSlots];
  __shared__ float s_w[kDecMaxSlots];             // gates of the slots
  __shared__ __align__(16) float s_keys[kRouteWarps][256];  // each routing warp's token keys
  __shared__ int s_total, s_last;
  __shared__ float upx[64][kDecN + 1];            // the up rows of D1, for the SwiGLU

  // dynamic: ring (stage = a weight tile + the tokens' tile of the same k
  // columns) | a^T (one 16-row tile)
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* at = ring + kDecStages * kDecStageBytes;
  const uint32_t ring_base = smem_addr(ring);
  const uint32_t at_base = smem_addr(at);
  const uint32_t bar_base = smem_addr(bars);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (kDecStages + s); };
  auto qfull_bar = [&](int q) { return bar_base + 8u * (2 * kDecStages + q); };
  auto qempty_bar = [&](int q) { return bar_base + 8u * (2 * kDecStages + kDecQueue + q); };
  // gate/up done, one barrier per D1 buffer: the MMA thread commits unit
  // j + 1's gate/up before it waits for unit j's a^T, so a single barrier
  // could complete two phases before the epilogue tests unit j's parity
  const uint32_t gu_full0 = bar_base + 8u * (2 * kDecStages + 2 * kDecQueue);
  auto gu_full = [&](uint32_t j) { return gu_full0 + 8u * (j & 1u); };
  const uint32_t a_ready = gu_full0 + 16u;
  const uint32_t dn_full = gu_full0 + 24u;
  const uint32_t drain_bar = gu_full0 + 32u;
  const uint32_t tables_bar = gu_full0 + 40u;  // warp 3's expert tables are built

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.T, n = a.n, K = a.K, I = a.I, Ks = a.Ks;
  const int nc = I / kDecUC;
  const int S = Ks * nc;                      // shared units
  volatile int* abort_p = &abort_flag;

  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int q = 0; q < kDecQueue; ++q) {
      mbar_init(qfull_bar(q), 1);
      mbar_init(qempty_bar(q), 5);  // the MMA thread and the 4 epilogue warps
    }
    mbar_init(gu_full(0), 1);
    mbar_init(gu_full(1), 1);
    mbar_init(a_ready, 1);
    mbar_init(dn_full, 1);
    mbar_init(drain_bar, 1);
    mbar_init(tables_bar, 32);
    abort_flag = 0;
    fence_mbar_init();
    fence_async_shared();  // the initialised barriers, before TMA completes on them
  }
  if (warp == 2) {
    tmem_alloc(smem_addr(&tmem_slot), kDecTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // u, the weights and the zeroed sync words come from earlier stream work
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  // ---- 1. logits: CTA c takes experts c, c + n_lc, ... ---------------------
  const int n_lc = n < static_cast<int>(gridDim.x) ? n : static_cast<int>(gridDim.x);
  if (static_cast<int>(blockIdx.x) < n_lc) {
    const int t0 = warp, t1 = warp + kDecThreads / 32;  // T <= 16: two tokens per warp
    for (int e = blockIdx.x; e < n; e += n_lc) {
      const uint4* er = reinterpret_cast<const uint4*>(a.E + static_cast<int64_t>(e) * D);
      const uint4* u0 = reinterpret_cast<const uint4*>(a.u + static_cast<int64_t>(t0 < T ? t0 : 0) * D);
      const uint4* u1 = reinterpret_cast<const uint4*>(a.u + static_cast<int64_t>(t1 < T ? t1 : 0) * D);
      uint4 ev[NV], x0[NV], x1[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        ev[v] = __ldg(er + v * 32 + lane);
        x0[v] = __ldg(u0 + v * 32 + lane);
        x1[v] = __ldg(u1 + v * 32 + lane);
      }
      float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const uint4 y = ev[v], p = x0[v], q = x1[v];
        acc0 = fmaf(bf_lo(p.x), bf_lo(y.x), acc0); acc0 = fmaf(bf_hi(p.x), bf_hi(y.x), acc0);
        acc0 = fmaf(bf_lo(p.y), bf_lo(y.y), acc0); acc0 = fmaf(bf_hi(p.y), bf_hi(y.y), acc0);
        acc0 = fmaf(bf_lo(p.z), bf_lo(y.z), acc0); acc0 = fmaf(bf_hi(p.z), bf_hi(y.z), acc0);
        acc0 = fmaf(bf_lo(p.w), bf_lo(y.w), acc0); acc0 = fmaf(bf_hi(p.w), bf_hi(y.w), acc0);
        acc1 = fmaf(bf_lo(q.x), bf_lo(y.x), acc1); acc1 = fmaf(bf_hi(q.x), bf_hi(y.x), acc1);
        acc1 = fmaf(bf_lo(q.y), bf_lo(y.y), acc1); acc1 = fmaf(bf_hi(q.y), bf_hi(y.y), acc1);
        acc1 = fmaf(bf_lo(q.z), bf_lo(y.z), acc1); acc1 = fmaf(bf_hi(q.z), bf_hi(y.z), acc1);
        acc1 = fmaf(bf_lo(q.w), bf_lo(y.w), acc1); acc1 = fmaf(bf_hi(q.w), bf_hi(y.w), acc1);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        acc0 += __shfl_xor_sync(0xffffffffu, acc0, o);
        acc1 += __shfl_xor_sync(0xffffffffu, acc1, o);
      }
      if (lane == 0) {
        if (t0 < T) a.logits[t0 * n + e] = acc0;
        if (t1 < T) a.logits[t1 * n + e] = acc1;
      }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0)
      asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(&a.sync->logit_ctas) : "memory");
  }

  // ---- 2. units --------------------------------------------------------------
  if (warp == 0) {
    // ------------------------------------------------------- TMA producer ----
    if (lane == 0) {
      const uint64_t w_policy = l2_evict_first_policy();
      tma_prefetch_desc(&tmW13);
      tma_prefetch_desc(&tmW2);
      tma_prefetch_desc(&tmU);
      if (Ks > 0) {
        tma_prefetch_desc(&tmW13s);
        tma_prefetch_desc(&tmW2s);
      }
      int q = 0, stage = 0;
      uint32_t qphase = 0, sphase = 0;
      bool have_tables = false, ok = true;
      uint32_t issued = 0, issued_parity = 0;
      int prev_kind = -1, prev_expert = 0, prev_chunk = 0;  // the unit whose W2 is due
      while (ok) {
        const int u = atomicAdd(&a.sync->unit_next, 1);
        if (u >= S && !have_tables) {
          // the routed units need the expert tables (warp 3)
          if (!wait_bounded(tables_bar, 0, abort_p, a.status)) {
            ok = false;
            break;
          }
          have_tables = true;
        }
        UnitDesc ud;
        for (int t = 0; t < kDecN; ++t) ud.row_of[t] = -1;
        if (have_tables && u >= s_total) {
          ud.kind = -1;
          ud.expert = ud.chunk = ud.slot = 0;
        } else if (u < S) {
          ud.kind = 0;
          ud.expert = u / nc;
          ud.chunk = u - ud.expert * nc;
          ud.slot = u * T;
          for (int t = 0; t < T; ++t) ud.row_of[t] = static_cast<int8_t>(t);
        } else {
          const int j = (u - S) / nc;
          const int e = s_active[j];
          ud.kind = 1;
          ud.expert = e;
          ud.chunk = (u - S) - j * nc;
          ud.slot = S * T + s_off[e] * nc + ud.chunk * s_cnt[e];
          for (int r = 0; r < s_cnt[e]; ++r)
            ud.row_of[s_tok[s_off[e] + r]] = static_cast<int8_t>(r);
        }
        if (!wait_bounded(qempty_bar(q), qphase ^ 1u, abort_p, a.status)) { ok = false; break; }
        qdesc[q] = ud;
        mbar_arrive(qfull_bar(q));  // release: the descriptor and the tables
        if (++q == kDecQueue) { q = 0; qphase ^= 1u; }
        // the ring order is W13(unit i), then W2(unit i-1): the MMAs of unit
        // i's gate/up run while the epilogue turns unit i-1's into a^T
        // with_u: also the tokens' tile of the same 64 columns of d (rows past
        // T read as zeros), the B operand of the gate/up MMAs
        auto load = [&](const CUtensorMap* map, int x, int y, bool with_u) {
          if (!wait_bounded(empty_bar(stage), sphase ^ 1u, abort_p, a.status)) return false;
          const uint32_t dst = ring_base + stage * kDecStageBytes;
          mbar_arrive_expect_tx(full_bar(stage), kDecTileBytes + (with_u ? kDecUTileBytes : 0));
          tma_load_2d_evict_first(dst, map, full_bar(stage), x, y, w_policy);
          if (with_u) tma_load_2d(dst + kDecTileBytes, &tmU, full_bar(stage), x, 0);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (sphase << stage);
          if (++stage == kDecStages) { stage = 0; sphase ^= 1u; }
          return true;
        };
        if (ud.kind >= 0) {
          // this unit's W13 block: KB13 tiles of 64 columns of d
          const CUtensorMap* m13 = ud.kind == 0 ? &tmW13s : &tmW13;
          const int row13 = ud.expert * 2 * I + ud.chunk * 128;
          for (int st = 0; st < KB13 && ok; ++st) ok = load(m13, st * 64, row13, true);
        }
        if (ok && prev_kind >= 0) {
          // the previous unit's W2 rows: MT2 tiles of 128, columns chunk*64 .. +63
          const CUtensorMap* m2 = prev_kind == 0 ? &tmW2s : &tmW2;
          for (int m = 0; m < MT2 && ok; ++m)
            ok = load(m2, prev_chunk * kDecUC, prev_expert * D + m * 128, false);
        }
        if (ud.kind < 0) break;
        prev_kind = ud.kind;
        prev_expert = ud.expert;
        prev_chunk = ud.chunk;
      }
      if (!ok) {
        // a wait ran out: the others see the flag; let the loads in flight land
        *abort_p = 1;
        for (int s = 0; s < kDecStages; ++s)
          if (issued & (1u << s)) {
            int dummy = 0;
            wait_bounded(full_bar(s), (issued_parity >> s) & 1u, &dummy, nullptr);
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer ----
    if (lane == 0) {
      int q = 0, stage = 0;
      uint32_t qphase = 0, sphase = 0;
      uint32_t j = 0;          // units whose gate/up MMAs were issued
      bool ok = true;
      // unit j's down MMAs follow unit j+1's gate/up MMAs (the ring order)
      auto down = [&](uint32_t jj) {
        // the epilogue has read D1 of unit jj and written its a^T
        if (!wait_bounded(a_ready, jj & 1u, abort_p, a.status)) return false;
        tc_fence_after();
        for (int m = 0; m < MT2; ++m) {
          if (!wait_bounded(full_bar(stage), sphase, abort_p, a.status)) return false;
          tc_fence_after();
          const uint32_t sa = ring_base + stage * kDecStageBytes;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16(tmem_base + 2 * kDecN + m * kDecN, desc_kmajor_sw128(sa + k * 32),
                     desc_kmajor_sw128(at_base + k * 32), IDESC, k > 0 ? 1u : 0u);
          mma_commit(empty_bar(stage));
          if (++stage == kDecStages) { stage = 0; sphase ^= 1u; }
        }
        mma_commit(dn_full);
        return true;
      };
      while (ok) {
        if (!wait_bounded(qfull_bar(q), qphase, abort_p, a.status)) { ok = false; break; }
        const int kind = qdesc[q].kind;
        mbar_arrive(qempty_bar(q));
        if (++q == kDecQueue) { q = 0; qphase ^= 1u; }
        if (kind >= 0) {
          // gate/up of unit j: D1[j % 2] = W13 block . U^T
          const uint32_t d1 = tmem_base + (j & 1u) * kDecN;
          for (int kb = 0; kb < KB13; ++kb) {
            if (!wait_bounded(full_bar(stage), sphase, abort_p, a.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = ring_base + stage * kDecStageBytes;
            const uint32_t sb = sa + kDecTileBytes;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16(d1, desc_kmajor_sw128(sa + k * 32), desc_kmajor_sw128(sb + k * 32), IDESC,
                       (kb > 0 || k > 0) ? 1u : 0u);
            mma_commit(empty_bar(stage));
            if (++stage == kDecStages) { stage = 0; sphase ^= 1u; }
          }
          if (!ok) break;
          mma_commit(gu_full(j));
        }
        if (j > 0 && !down(j - 1)) { ok = false; break; }
        if (kind < 0) break;
        ++j;
      }
      if (!ok) {
        *abort_p = 1;
        // wait for every MMA already issued before TMEM is released
        mma_commit(drain_bar);
        int dummy = 0;
        wait_bounded(drain_bar, 0, &dummy, nullptr);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------- routing (warps 2-7) and tables (3) ----
    // the epilogue warps route too: their first wait (a unit's gate/up) is
    // further away than the routing
    const int pw = warp - 2;  // tokens pw, pw + 6, ...
    bool ok = true;
    if (tid == 64) ok = spin_until(&a.sync->logit_ctas, n_lc, a.status);
    ok = route_all(ok);  // warps 2-7 learn the outcome together
    if (!ok) {
      if (lane == 0) *abort_p = 1;
    } else {
      const bool select_only = (a.flags & MOE_FLAG_BIAS_SELECT_ONLY) != 0;
      int32_t* gidx = blockIdx.x == 0 ? a.idx : nullptr;  // one copy of idx / w in the workspace
      float* gw = blockIdx.x == 0 ? a.w : nullptr;
      if (n <= 32)
        route_tokens<1>(a.logits, a.bias, n, K, T, pw, kRouteWarps, select_only, s_keys[pw], s_idx, s_w,
                        gidx, gw);
      else if (n <= 64)
        route_tokens<2>(a.logits, a.bias, n, K, T, pw, kRouteWarps, select_only, s_keys[pw], s_idx, s_w,
                        gidx, gw);
      else if (n <= 128)
        route_tokens<4>(a.logits, a.bias, n, K, T, pw, kRouteWarps, select_only, s_keys[pw], s_idx, s_w,
                        gidx, gw);
      else
        route_tokens<8>(a.logits, a.bias, n, K, T, pw, kRouteWarps, select_only, s_keys[pw], s_idx, s_w,
                        gidx, gw);
      asm volatile("bar.sync 2, 192;" ::: "memory");  // every routing warp's slots are in s_idx / s_w
      if (warp == 3) {
        const int TK = T * K;
        for (int e = lane; e < n; e += 32) s_cnt[e] = 0;
        __syncwarp();
        // rank of slot i within its expert, in slot order (t, then k): 32
        // slots at a time, equal experts in one batch ranked by lane
        for (int i0 = 0; i0 < TK; i0 += 32) {
          const int i = i0 + lane;
          const bool act = i < TK;
          const int e = act ? s_idx[i] : -1 - lane;
          const unsigned peers = __match_any_sync(0xffffffffu, e);
          const int before = __popc(peers & ((1u << lane) - 1u));
          const int base = act ? s_cnt[e] : 0;
          __syncwarp();
          if (act) {
            s_rank[i] = base + before;
            if (before == 0) s_cnt[e] = base + __popc(peers);
          }
          __syncwarp();
        }
        // offsets and the active list: lane l takes experts 8l .. 8l+7
        int c[8], sum = 0, nact = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int e = lane * 8 + q;
          c[q] = e < n ? s_cnt[e] : 0;
          sum += c[q];
          nact += c[q] > 0 ? 1 : 0;
        }
        int incl = sum, inca = nact;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          const int ya = __shfl_up_sync(0xffffffffu, inca, o);
          if (lane >= o) {
            incl += y;
            inca += ya;
          }
        }
        int run = incl - sum, pos = inca - nact;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int e = lane * 8 + q;
          if (e < n) {
            s_off[e] = run;
            run += c[q];
            if (c[q] > 0) s_active[pos++] = e;
          }
        }
        if (lane == 31) {
          s_off[n] = incl;
          s_total = S + inca * nc;
        }
        __syncwarp();
        for (int i = lane; i < TK; i += 32) s_tok[s_off[s_idx[i]] + s_rank[i]] = i / K;
        __syncwarp();
        mbar_arrive(tables_bar);  // release: every lane's table writes
      }
    }
  }
  if (warp >= 4) {
    // ----------------------------------------------------------- epilogue ----
    const int q4 = warp - 4;            // TMEM lane quarter
    const int r = q4 * 32 + lane;       // TMEM lane: W13 block row / W2 row in a tile
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(q4 * 32) << 16);
    int q = 0;
    uint32_t qphase = 0, j = 0;
    while (true) {
      if (!epi_all(warp_wait(qfull_bar(q), qphase, abort_p, a.status))) break;
      const UnitDesc ud = qdesc[q];
      __syncwarp();
      if (lane == 0) mbar_arrive(qempty_bar(q));
      if (++q == kDecQueue) { q = 0; qphase ^= 1u; }
      if (ud.kind < 0) break;  // the same descriptor in every warp
      // D1 -> SwiGLU -> a^T (bf16, the B operand of the down MMAs)
      if (!epi_all(warp_wait(gu_full(j), (j >> 1) & 1u, abort_p, a.status))) break;
      tc_fence_after();
      float z[kDecN];
      tmem_ld16(tl + (j & 1u) * kDecN, z);
      tmem_ld_wait_regs16(z);
      if (q4 >= 2) {
#pragma unroll
        for (int t = 0; t < kDecN; ++t) upx[r - 64][t] = z[t];
      }
      epi_sync();
      if (q4 < 2) {
#pragma unroll
        for (int t = 0; t < kDecN; ++t) {
          const float av = t < T ? silu_mul(z[t], upx[r][t]) : 0.0f;
          *reinterpret_cast<bf16*>(at + sw128_off(t, r)) = __float2bfloat16_rn(av);
        }
      }
      fence_async_shared();  // a^T written by the generic proxy, read by the tensor cores
      tc_fence_before();
      epi_sync();
      if (tid == 128) mbar_arrive(a_ready);
      // D2 -> the unit's partial rows
      if (!epi_all(warp_wait(dn_full, j & 1u, abort_p, a.status))) break;
      tc_fence_after();
      float* base = a.part + static_cast<int64_t>(ud.slot) * D + r;
      for (int m = 0; m < MT2; ++m) {
        float y[kDecN];
        tmem_ld16(tl + 2 * kDecN + m * kDecN, y);
        tmem_ld_wait_regs16(y);
#pragma unroll
        for (int t = 0; t < kDecN; ++t) {
          const int row = ud.row_of[t];
          if (row >= 0) base[static_cast<int64_t>(row) * D + m * 128] = y[t];
        }
      }
      __threadfence();  // the partials, before the unit is counted
      tc_fence_before();
      epi_sync();
      if (tid == 128) atomicAdd(&a.sync->units_done, 1);
      ++j;
    }
  }

  // ---- 3. combine ------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kDecTmemCols);
  }
  if (*abort_p) {
    record_status(a.status, MOE_ERR_DEVICE_CHECK);
    return;
  }
  if (tid == 0) {
    // every CTA's producer built the tables before it ran out of units
    s_last = spin_until(&a.sync->units_done, s_total, a.status) ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // one CTA per (token, 256 columns): warp w sums the token's partial rows
  // w, w + 8, ... (shared units with gate 1, then each routed slot's chunks
  // with its gate) in that order, lane l over columns 8l .. 8l + 7, 8 rows'
  // loads in flight; then thread c adds the 8 warps' sums of column c in
  // warp order, adds u and rounds once.  The warps' sums go to the ring,
  // which the units no longer use.
  constexpr int kRows = 8;
  const int R = S + K * nc;
  float* wsum = reinterpret_cast<float*>(ring);  // [8 warps][256 columns]
  for (int item = blockIdx.x; item < T * NV; item += gridDim.x) {
    const int t = item / NV;
    const int col0 = (item - t * NV) * 256;
    const int col = col0 + lane * 8;
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
    for (int j0 = warp; j0 < R; j0 += 8 * kRows) {
      float4 p0[kRows], p1[kRows];
      float g[kRows];
#pragma unroll
      for (int q = 0; q < kRows; ++q) {
        const int jr = j0 + 8 * q;
        g[q] = 0.0f;
        if (jr < R) {
          int64_t row;
          if (jr < S) {
            row = static_cast<int64_t>(jr) * T + t;
            g[q] = 1.0f;
          } else {
            const int kk = (jr - S) / nc, c = (jr - S) - kk * nc;
            const int e = s_idx[t * K + kk];
            row = static_cast<int64_t>(S) * T + static_cast<int64_t>(s_off[e]) * nc +
                  static_cast<int64_t>(c) * s_cnt[e] + s_rank[t * K + kk];
            g[q] = s_w[t * K + kk];
          }
          const float4* src = reinterpret_cast<const float4*>(a.part + row * D + col);
          p0[q] = __ldcg(src);
          p1[q] = __ldcg(src + 1);
        }
      }
#pragma unroll
      for (int q = 0; q < kRows; ++q) {
        if (j0 + 8 * q < R) {
          acc[0] = fmaf(g[q], p0[q].x, acc[0]); acc[1] = fmaf(g[q], p0[q].y, acc[1]);
          acc[2] = fmaf(g[q], p0[q].z, acc[2]); acc[3] = fmaf(g[q], p0[q].w, acc[3]);
          acc[4] = fmaf(g[q], p1[q].x, acc[4]); acc[5] = fmaf(g[q], p1[q].y, acc[5]);
          acc[6] = fmaf(g[q], p1[q].z, acc[6]); acc[7] = fmaf(g[q], p1[q].w, acc[7]);
        }
      }
    }
    float4* dst = reinterpret_cast<float4*>(wsum + warp * 256 + lane * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    __syncthreads();
    {
      float v = wsum[tid];
#pragma unroll
      for (int w8 = 1; w8 < kDecThreads / 32; ++w8) v += wsum[w8 * 256 + tid];
      const int64_t o = static_cast<int64_t>(t) * D + col0 + tid;
      a.h[o] = __float2bfloat16_rn(__bfloat162float(a.u[o]) + v);
    }
    __syncthreads();  // wsum is rewritten by the next item
  }
}

constexpr int dec_smem_bytes(int) { return 1024 + kDecStages * kDecStageBytes + kDecN * 128; }

template <int NV>
int launch_decode_nv(const CUtensorMap& m13, const CUtensorMap& m13s, const CUtensorMap& m2,
                     const CUtensorMap& m2s, const CUtensorMap& mu, const DecArgs& a, int grid,
                     cudaStream_t st) {
  static std::atomic<uint64_t> optin{0};
  auto kern = decode_layer_kernel<NV>;
  const int smem = dec_smem_bytes(NV * 256);
  if (int rc = ensure_smem_optin(reinterpret_cast<const void*>(kern), smem, optin)) return rc;
  return launch_k(kern, grid, kDecThreads, smem, st, 1, m13, m13s, m2, m2s, mu, a);
}

}  // namespace

bool decode_fused_eligible(const moe_shape_t& s) {
  const bool d_ok = s.d == 256 || s.d == 512 || s.d == 1024 || s.d == 2048;
  const int32_t forced = MOE_FLAG_GEMM_SINGLE_CTA | MOE_FLAG_GEMM_CTA_PAIR |
                         MOE_FLAG_INJECT_WAIT_TIMEOUT;
  return s.dtype == MOE_DTYPE_BF16 && s.T >= 1 && s.T <= kDecMaxT && d_ok &&
         s.inter % kDecUC == 0 && s.top_k <= 32 && s.n_routed <= 256 && (s.flags & forced) == 0;
}

size_t decode_partial_rows(const moe_shape_t& s) {
  return static_cast<size_t>(s.n_shared + s.top_k) * (s.inter / kDecUC) * static_cast<size_t>(s.T);
}

size_t decode_sync_bytes() { return sizeof(DecSync); }

int launch_decode_fused(const moe_shape_t& s, const void* u, const void* E, const float* bias,
                        const void* W13, const void* W2, const void* W13_s, const void* W2_s,
                        void* h, int32_t* idx, float* w, float* logits, float* part, void* sync,
                        int32_t* status, int sms, cudaStream_t st) {
  const uint64_t d = static_cast<uint64_t>(s.d), I = static_cast<uint64_t>(s.inter);
  const uint64_t n = static_cast<uint64_t>(s.n_routed), ks = static_cast<uint64_t>(s.n_shared);
  CUtensorMap m13, m13s, m2, m2s;
  if (!make_map_2d(&m13, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W13, d, n * 2 * I, d * 2, 64, 128) ||
      !make_map_2d(&m2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W2, I, n * d, I * 2, 64, 128))
    return MOE_ERR_CUDA;
  if (ks > 0) {
    if (!make_map_2d(&m13s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W13_s, d, ks * 2 * I, d * 2, 64,
                     128) ||
        !make_map_2d(&m2s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W2_s, I, ks * d, I * 2, 64, 128))
      return MOE_ERR_CUDA;
  } else {
    m13s = m13;
    m2s = m2;
  }
  // the tokens as 16-row boxes of 64 columns (rows past T read as zeros)
  CUtensorMap mu;
  if (!make_map_2d(&mu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, u, d, static_cast<uint64_t>(s.T), d * 2,
                   64, kDecN))
    return MOE_ERR_CUDA;
  if (int rc = launch_zero_words(static_cast<int32_t*>(sync),
                                 static_cast<int>(sizeof(DecSync) / sizeof(int32_t)), st))
    return rc;
  DecArgs a{};
  a.u = static_cast<const bf16*>(u);
  a.E = static_cast<const bf16*>(E);
  a.bias = bias;
  a.h = static_cast<bf16*>(h);
  a.idx = idx;
  a.w = w;
  a.logits = logits;
  a.part = part;
  a.sync = static_cast<DecSync*>(sync);
  a.status = status;
  a.T = static_cast<int>(s.T);
  a.d = s.d;
  a.n = s.n_routed;
  a.Ks = s.n_shared;
  a.I = s.inter;
  a.K = s.top_k;
  a.flags = s.flags;
  switch (s.d) {
    case 256: return launch_decode_nv<1>(m13, m13s, m2, m2s, mu, a, sms, st);
    case 512: return launch_decode_nv<2>(m13, m13s, m2, m2s, mu, a, sms, st);
    case 1024: return launch_decode_nv<4>(m13, m13s, m2, m2s, mu, a, sms, st);
    case 2048: return launch_decode_nv<8>(m13, m13s, m2, m2s, mu, a, sms, st);
    default: return MOE_ERR_SHAPE;
  }
}

}  // namespace moe
