// The whole DeepSeekMoE layer (§3.2, eqs. (9)-(11)) for decode-sized batches
// (T <= kDecMaxT tokens) in one persistent kernel.
//
// At a handful of tokens the layer is a stream of the activated experts'
// weights (W1/W3/W2 of every routed expert some token chose, plus the shared
// experts, all read once), so what matters is that every SM streams weights
// all the time.  The work is cut into units: one unit is kDecUC intermediate
// rows of one expert (a 128-row packed W13 block [gate 64 | up 64] and the
// matching 64 columns of W2), for the tokens that chose that expert (all
// tokens for a shared expert).  A unit computes a = SiLU(W1 x) * (W3 x) for
// its 64 rows and its partial down projection W2[:, chunk] a, an fp32 row of
// d values per token, written to its own slot of the workspace.  CTAs take
// units from an atomic counter, so the units spread evenly whatever the
// routing; the partial slots are fixed by the unit and the sums below run in
// a fixed order, so the result is the same whichever CTA took which unit.
//
// Phases, all in this one launch (one CTA per SM, 8 compute warps plus a
// producer warp):
//  1. Router (CTAs 0 .. ceil(n/8)-1): logits u_t . e_i for 8 experts each,
//     all tokens, fp32 FMA chains; the CTA that finishes last runs softmax
//     and top-K for every token (lower expert index first on ties, gates not
//     renormalised) and publishes idx / w.
//  2. Units: the shared experts' units need no routing and come first; the
//     routed units (active experts in increasing index, chunks in order)
//     become known once the routing is published.  The producer warp takes
//     units, streams each unit's W13 block with bulk copies and its W2
//     columns with TMA into a 4-stage ring, running ahead into the next
//     unit; the compute warps take the units from a small queue.
//  3. Combine: once every unit is done, h_t = u_t + sum over the shared
//     partials + sum_k w[t,k] * (sum over expert idx[t,k]'s partials), in
//     fp32 in that order, rounded once to bf16.
// Every wait is bounded: a wait that runs out records MOE_ERR_DEVICE_CHECK in
// the status word and the kernel winds down without touching h.
#include <cuda.h>
#include <math_constants.h>

#include "common.cuh"
#include "decode_fused.h"
#include "gemm_sm100.h"
#include "sm100_ptx.cuh"

namespace moe {

namespace {

using namespace sm100;

constexpr int kDecWarps = 8;                         // compute warps
constexpr int kDecThreads = (kDecWarps + 1) * 32;    // + the producer warp
constexpr int kDecUC = 64;                           // intermediate rows per unit
constexpr int kDecStageBytes = 32 * 1024;
constexpr int kDecStages = 4;
constexpr int kDecQueue = 4;                         // unit descriptors in flight
constexpr int kDecW2Rows = 256;                      // W2 rows per TMA box
constexpr int kDecRouterExperts = 8;                 // experts per router CTA
constexpr int kDecMaxSlots = kDecMaxT * 32;          // routed (token, k) slots

// sync words at the start of the decode scratch (zeroed before each launch)
struct DecSync {
  int unit_next;     // next unit to take
  int route_arrive;  // router CTAs done with their logits
  int route_done;    // 1 once idx / w are published
  int units_done;    // units whose partials are written
};

struct DecArgs {
  const bf16* u;        // [T, d]
  const bf16* E;        // [n, d]
  const float* bias;    // [n] or null
  const bf16* W13;      // [n, 2I, d] packed
  const bf16* W13_s;    // [Ks, 2I, d] packed (null when Ks = 0)
  bf16* h;              // [T, d]
  int32_t* idx;         // [T, K] (workspace)
  float* w;             // [T, K] (workspace)
  float* logits;        // [T, n] (workspace)
  float* part;          // partial rows [rows, d] (workspace)
  DecSync* sync;
  int32_t* status;
  int T, d, n, Ks, I, K, flags;
};

struct UnitDesc {
  int kind;      // 0 shared, 1 routed, -1 no more units
  int expert;    // routed expert e, or shared expert s
  int chunk;     // which kDecUC rows of I
  int n_tok;
  int tok_off;   // into the token list (routed) or -1 (all tokens)
  int slot;      // first partial row
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kDecWarps * 32) : "memory");
}

// All compute warps vote: true when every one of them passes true.  Every
// compute warp reaches each vote exactly once, whatever its own wait saw, so
// they stay in step also when a wait runs out.
__device__ __forceinline__ bool consumer_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(kDecWarps * 32)
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

template <int NV>
__global__ void __launch_bounds__(kDecThreads, 1)
decode_layer_kernel(const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmW2s,
                    const DecArgs a) {
  constexpr int D = NV * 256;  // hidden size: NV 16-byte chunks per lane
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * kDecStages + 2 * kDecQueue];
  __shared__ UnitDesc qdesc[kDecQueue];
  __shared__ int abort_flag;
  __shared__ int s_cnt[256], s_off[257], s_active[256], s_nactive;
  __shared__ int s_tok[kDecMaxSlots];             // tokens of each expert, increasing t
  __shared__ int s_rank[kDecMaxSlots];            // rank of token t within expert idx[t,k]
  __shared__ int s_idx[kDecMaxSlots];
  __shared__ int s_total, s_tables_ok, s_last;
  __shared__ float zbuf[128][kDecMaxT];
  __shared__ float abuf[kDecUC][kDecMaxT];

  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* uf = reinterpret_cast<float*>(ring + kDecStages * kDecStageBytes);  // [T][D] fp32
  const uint32_t ring_base = smem_addr(ring);
  const uint32_t bar_base = smem_addr(bars);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (kDecStages + s); };
  auto qfull_bar = [&](int q) { return bar_base + 8u * (2 * kDecStages + q); };
  auto qempty_bar = [&](int q) { return bar_base + 8u * (2 * kDecStages + kDecQueue + q); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.T, n = a.n, K = a.K, I = a.I, Ks = a.Ks;
  const int nc = I / kDecUC;
  const int S = Ks * nc;                      // shared units
  const int rs = 16384 / D;                   // W13 rows per 32 KB stage
  const int n13 = 128 / rs;                   // W13 stages per unit
  const int n2 = (D + kDecW2Rows - 1) / kDecW2Rows;  // W2 boxes per unit
  volatile int* abort_p = &abort_flag;

  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kDecWarps);
    }
    for (int q = 0; q < kDecQueue; ++q) {
      mbar_init(qfull_bar(q), 1);
      mbar_init(qempty_bar(q), kDecWarps);
    }
    abort_flag = 0;
    s_tables_ok = 0;
    fence_mbar_init();
    fence_async_shared();
  }
  pdl_wait();  // u, the weights and the zeroed sync words come from earlier stream work
  pdl_trigger();
  // the batch's token rows, widened to fp32 once
  for (int i = tid; i < T * (D / 8); i += kDecThreads) {
    const int t = i / (D / 8), c = i - t * (D / 8);
    const uint4 v = reinterpret_cast<const uint4*>(a.u + static_cast<int64_t>(t) * D)[c];
    float* dst = uf + t * D + c * 8;
    reinterpret_cast<float4*>(dst)[0] = make_float4(bf_lo(v.x), bf_hi(v.x), bf_lo(v.y), bf_hi(v.y));
    reinterpret_cast<float4*>(dst)[1] = make_float4(bf_lo(v.z), bf_hi(v.z), bf_lo(v.w), bf_hi(v.w));
  }
  __syncthreads();

  // ---- 1. router -----------------------------------------------------------
  const int n_rctas = (n + kDecRouterExperts - 1) / kDecRouterExperts;
  if (static_cast<int>(blockIdx.x) < n_rctas) {
    if (warp < kDecWarps) {
      const int e = blockIdx.x * kDecRouterExperts + warp;
      if (e < n) {
        const uint4* er = reinterpret_cast<const uint4*>(a.E + static_cast<int64_t>(e) * D);
        float ev[NV][8];
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          const uint4 x = er[v * 32 + lane];
          ev[v][0] = bf_lo(x.x); ev[v][1] = bf_hi(x.x); ev[v][2] = bf_lo(x.y); ev[v][3] = bf_hi(x.y);
          ev[v][4] = bf_lo(x.z); ev[v][5] = bf_hi(x.z); ev[v][6] = bf_lo(x.w); ev[v][7] = bf_hi(x.w);
        }
        for (int t = 0; t < T; ++t) {
          float acc = 0.0f;
#pragma unroll
          for (int v = 0; v < NV; ++v) {
            const float4* up = reinterpret_cast<const float4*>(uf + t * D + (v * 32 + lane) * 8);
            const float4 p0 = up[0], p1 = up[1];
            acc = fmaf(p0.x, ev[v][0], acc); acc = fmaf(p0.y, ev[v][1], acc);
            acc = fmaf(p0.z, ev[v][2], acc); acc = fmaf(p0.w, ev[v][3], acc);
            acc = fmaf(p1.x, ev[v][4], acc); acc = fmaf(p1.y, ev[v][5], acc);
            acc = fmaf(p1.z, ev[v][6], acc); acc = fmaf(p1.w, ev[v][7], acc);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          if (lane == 0) a.logits[t * n + e] = acc;
        }
      }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&a.sync->route_arrive, 1) == n_rctas - 1;
    __syncthreads();
    if (s_last) {
      // the last router CTA: softmax and top-K of every token, warp per token
      __threadfence();
      const bool select_only = (a.flags & MOE_FLAG_BIAS_SELECT_ONLY) != 0;
      for (int t = warp; t < T && warp < kDecWarps; t += kDecWarps) {
        float lg[8], key[8], ex[8];
        float m = -CUDART_INF_F;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int e = lane + 32 * q;
          float l = -CUDART_INF_F, kv = -CUDART_INF_F;
          if (e < n) {
            const float raw = __ldcg(a.logits + t * n + e);
            const float b = a.bias ? a.bias[e] : 0.0f;
            kv = raw + b;
            l = select_only ? raw : kv;
          }
          lg[q] = l;
          key[q] = kv;
          m = fmaxf(m, l);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float z = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          ex[q] = (lane + 32 * q < n) ? expf(lg[q] - m) : 0.0f;
          z += ex[q];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
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
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
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
            a.idx[t * K + k] = bi;
            a.w[t * K + k] = g * inv_z;
          }
        }
      }
      __threadfence();
      __syncthreads();
      if (tid == 0) {
        asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(&a.sync->route_done), "r"(1)
                     : "memory");
      }
    }
  }

  // ---- 2. units --------------------------------------------------------------
  if (warp == kDecWarps) {
    // ------------------------------------------------------- producer warp ----
    if (lane == 0) {
      tma_prefetch_desc(&tmW2);
      if (Ks > 0) tma_prefetch_desc(&tmW2s);
      int q = 0, stage = 0;
      uint32_t qphase = 0, sphase = 0;
      bool have_tables = false, ok = true;
      uint32_t issued = 0, issued_parity = 0;
      while (ok) {
        const int u = atomicAdd(&a.sync->unit_next, 1);
        if (u >= S && !have_tables) {
          // the routed units need the routing: build the expert tables
          if (!spin_until(&a.sync->route_done, 1, a.status)) { *abort_p = 1; ok = false; break; }
          for (int e = 0; e < n; ++e) s_cnt[e] = 0;
          for (int i = 0; i < T * K; ++i) {
            const int e = __ldcg(a.idx + i);
            s_idx[i] = e;
            s_rank[i] = s_cnt[e]++;  // i runs in increasing t: ranks follow t
          }
          int run = 0, na = 0;
          for (int e = 0; e < n; ++e) {
            s_off[e] = run;
            run += s_cnt[e];
            if (s_cnt[e] > 0) s_active[na++] = e;
          }
          s_off[n] = run;
          for (int i = 0; i < T * K; ++i) s_tok[s_off[s_idx[i]] + s_rank[i]] = i / K;
          s_nactive = na;
          s_total = S + na * nc;
          s_tables_ok = 1;
          have_tables = true;
        }
        UnitDesc ud;
        if (have_tables && u >= s_total) {
          ud.kind = -1;
        } else if (u < S) {
          ud.kind = 0;
          ud.expert = u / nc;
          ud.chunk = u - ud.expert * nc;
          ud.n_tok = T;
          ud.tok_off = -1;
          ud.slot = u * T;
        } else {
          const int j = (u - S) / nc;
          const int e = s_active[j];
          ud.kind = 1;
          ud.expert = e;
          ud.chunk = (u - S) - j * nc;
          ud.n_tok = s_cnt[e];
          ud.tok_off = s_off[e];
          ud.slot = S * T + s_off[e] * nc + ud.chunk * s_cnt[e];
        }
        if (!wait_bounded(qempty_bar(q), qphase ^ 1u, abort_p, a.status)) { ok = false; break; }
        qdesc[q] = ud;
        mbar_arrive(qfull_bar(q));  // release: the descriptor and the tables
        if (++q == kDecQueue) { q = 0; qphase ^= 1u; }
        if (ud.kind < 0) break;
        // the unit's weights: its W13 block in n13 bulk copies, then W2's
        // columns chunk*64 .. +63 in n2 boxes of 256 rows
        const bf16* w13 = ud.kind == 0
                              ? a.W13_s + (static_cast<int64_t>(ud.expert) * 2 * I + ud.chunk * 128) * D
                              : a.W13 + (static_cast<int64_t>(ud.expert) * 2 * I + ud.chunk * 128) * D;
        for (int st = 0; st < n13 + n2 && ok; ++st) {
          if (!wait_bounded(empty_bar(stage), sphase ^ 1u, abort_p, a.status)) { ok = false; break; }
          const uint32_t dst = ring_base + stage * kDecStageBytes;
          if (st < n13) {
            mbar_arrive_expect_tx(full_bar(stage), kDecStageBytes);
            bulk_load(dst, w13 + static_cast<int64_t>(st) * rs * D, kDecStageBytes, full_bar(stage));
          } else {
            const int box = st - n13;
            mbar_arrive_expect_tx(full_bar(stage), kDecW2Rows * 128);
            tma_load_2d(dst, ud.kind == 0 ? &tmW2s : &tmW2, full_bar(stage), ud.chunk * kDecUC,
                        ud.expert * D + box * kDecW2Rows);
          }
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (sphase << stage);
          if (++stage == kDecStages) { stage = 0; sphase ^= 1u; }
        }
      }
      if (!ok) {
        // a wait ran out: tell the compute warps, and let the copies in flight land
        *abort_p = 1;
        for (int s = 0; s < kDecStages; ++s)
          if (issued & (1u << s)) {
            int dummy = 0;
            wait_bounded(full_bar(s), (issued_parity >> s) & 1u, &dummy, nullptr);
          }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- compute warps ----
    int q = 0, stage = 0;
    uint32_t qphase = 0, sphase = 0;
    while (true) {
      if (!consumer_all(warp_wait(qfull_bar(q), qphase, abort_p, a.status))) break;
      const UnitDesc ud = qdesc[q];
      __syncwarp();
      if (lane == 0) mbar_arrive(qempty_bar(q));
      if (++q == kDecQueue) { q = 0; qphase ^= 1u; }
      if (ud.kind < 0) break;
      bool ok = true;
      // gate/up rows: warp w takes rows w, w + 8, ... of each stage
      for (int st = 0; st < n13; ++st) {
        if (!consumer_all(warp_wait(full_bar(stage), sphase, abort_p, a.status))) { ok = false; break; }
        const uint8_t* tile = ring + stage * kDecStageBytes;
        for (int rl = warp; rl < rs; rl += kDecWarps) {
          const uint4* row = reinterpret_cast<const uint4*>(tile + rl * D * 2);
          float wv[NV][8];
#pragma unroll
          for (int v = 0; v < NV; ++v) {
            const uint4 x = row[v * 32 + lane];
            wv[v][0] = bf_lo(x.x); wv[v][1] = bf_hi(x.x); wv[v][2] = bf_lo(x.y); wv[v][3] = bf_hi(x.y);
            wv[v][4] = bf_lo(x.z); wv[v][5] = bf_hi(x.z); wv[v][6] = bf_lo(x.w); wv[v][7] = bf_hi(x.w);
          }
          for (int i = 0; i < ud.n_tok; ++i) {
            const int t = ud.tok_off < 0 ? i : s_tok[ud.tok_off + i];
            float acc = 0.0f;
#pragma unroll
            for (int v = 0; v < NV; ++v) {
              const float4* up = reinterpret_cast<const float4*>(uf + t * D + (v * 32 + lane) * 8);
              const float4 p0 = up[0], p1 = up[1];
              acc = fmaf(p0.x, wv[v][0], acc); acc = fmaf(p0.y, wv[v][1], acc);
              acc = fmaf(p0.z, wv[v][2], acc); acc = fmaf(p0.w, wv[v][3], acc);
              acc = fmaf(p1.x, wv[v][4], acc); acc = fmaf(p1.y, wv[v][5], acc);
              acc = fmaf(p1.z, wv[v][6], acc); acc = fmaf(p1.w, wv[v][7], acc);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) zbuf[st * rs + rl][i] = acc;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(stage));
        if (++stage == kDecStages) { stage = 0; sphase ^= 1u; }
      }
      if (!ok) break;  // the same decision in every compute warp
      consumer_sync();  // zbuf complete
      // SwiGLU of the unit's 64 rows (packed block: gate rows 0-63, up 64-127)
      for (int i = tid; i < kDecUC * ud.n_tok; i += kDecWarps * 32) {
        const int j = i / ud.n_tok, tt = i - j * ud.n_tok;
        abuf[j][tt] = silu_mul(zbuf[j][tt], zbuf[64 + j][tt]);
      }
      consumer_sync();
      // partial down projection: thread r takes W2 row box*256 + r
      for (int bx = 0; bx < n2; ++bx) {
        if (!consumer_all(warp_wait(full_bar(stage), sphase, abort_p, a.status))) { ok = false; break; }
        const uint8_t* tile = ring + stage * kDecStageBytes;
        const int r = tid;  // 0 .. 255
        const int jrow = bx * kDecW2Rows + r;
        if (jrow < D) {
          float wv[64];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            // 128-byte swizzle: 16-byte chunk c of row r sits at c ^ (r & 7)
            const uint4 x = *reinterpret_cast<const uint4*>(tile + r * 128 + ((c ^ (r & 7)) << 4));
            wv[c * 8 + 0] = bf_lo(x.x); wv[c * 8 + 1] = bf_hi(x.x);
            wv[c * 8 + 2] = bf_lo(x.y); wv[c * 8 + 3] = bf_hi(x.y);
            wv[c * 8 + 4] = bf_lo(x.z); wv[c * 8 + 5] = bf_hi(x.z);
            wv[c * 8 + 6] = bf_lo(x.w); wv[c * 8 + 7] = bf_hi(x.w);
          }
          for (int i = 0; i < ud.n_tok; ++i) {
            float acc = 0.0f;
#pragma unroll
            for (int k = 0; k < kDecUC; ++k) acc = fmaf(wv[k], abuf[k][i], acc);
            a.part[static_cast<int64_t>(ud.slot + i) * D + jrow] = acc;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(stage));
        if (++stage == kDecStages) { stage = 0; sphase ^= 1u; }
      }
      if (!ok) break;
      __threadfence();  // this thread's partials, before the unit is counted
      consumer_sync();
      if (tid == 0) atomicAdd(&a.sync->units_done, 1);
    }
  }

  // ---- 3. combine ------------------------------------------------------------
  __syncthreads();
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
  const int cols4 = D / 4;
  for (int g = blockIdx.x * kDecThreads + tid; g < T * cols4; g += gridDim.x * kDecThreads) {
    const int t = g / cols4;
    const int col = (g - t * cols4) * 4;
    const uint2 uv = *reinterpret_cast<const uint2*>(a.u + static_cast<int64_t>(t) * D + col);
    float4 acc = make_float4(bf_lo(uv.x), bf_hi(uv.x), bf_lo(uv.y), bf_hi(uv.y));
    float4 sh = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int su = 0; su < S; ++su) {
      const float4 p = __ldcg(reinterpret_cast<const float4*>(
          a.part + static_cast<int64_t>(su * T + t) * D + col));
      sh.x += p.x; sh.y += p.y; sh.z += p.z; sh.w += p.w;
    }
    acc.x += sh.x; acc.y += sh.y; acc.z += sh.z; acc.w += sh.w;
    for (int k = 0; k < K; ++k) {
      const int e = s_idx[t * K + k];
      const int cnt = s_cnt[e];
      const int64_t base = static_cast<int64_t>(S) * T + static_cast<int64_t>(s_off[e]) * nc +
                           s_rank[t * K + k];
      float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int c = 0; c < nc; ++c) {
        const float4 p = __ldcg(reinterpret_cast<const float4*>(
            a.part + (base + static_cast<int64_t>(c) * cnt) * D + col));
        y.x += p.x; y.y += p.y; y.z += p.z; y.w += p.w;
      }
      const float wk = __ldcg(a.w + t * K + k);
      acc.x = fmaf(wk, y.x, acc.x); acc.y = fmaf(wk, y.y, acc.y);
      acc.z = fmaf(wk, y.z, acc.z); acc.w = fmaf(wk, y.w, acc.w);
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&lo);
    o.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(a.h + static_cast<int64_t>(t) * D + col) = o;
  }
}


constexpr int dec_smem_bytes(int D) { return 1024 + kDecStages * kDecStageBytes + kDecMaxT * D * 4; }

template <int NV>
int launch_decode_nv(const CUtensorMap& m2, const CUtensorMap& m2s, const DecArgs& a, int grid,
                     cudaStream_t st) {
  static std::atomic<uint64_t> optin{0};
  auto kern = decode_layer_kernel<NV>;
  const int smem = dec_smem_bytes(NV * 256);
  if (int rc = ensure_smem_optin(reinterpret_cast<const void*>(kern), smem, optin)) return rc;
  return launch_k(kern, grid, kDecThreads, smem, st, 1, m2, m2s, a);
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
  CUtensorMap m2, m2s;
  if (!make_map_2d(&m2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W2, I,
                   static_cast<uint64_t>(s.n_routed) * d, I * 2, kDecUC, kDecW2Rows))
    return MOE_ERR_CUDA;
  if (s.n_shared > 0) {
    if (!make_map_2d(&m2s, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W2_s, I,
                     static_cast<uint64_t>(s.n_shared) * d, I * 2, kDecUC, kDecW2Rows))
      return MOE_ERR_CUDA;
  } else {
    m2s = m2;
  }
  if (cudaMemsetAsync(sync, 0, sizeof(DecSync), st) != cudaSuccess) return MOE_ERR_CUDA;
  DecArgs a{};
  a.u = static_cast<const bf16*>(u);
  a.E = static_cast<const bf16*>(E);
  a.bias = bias;
  a.W13 = static_cast<const bf16*>(W13);
  a.W13_s = static_cast<const bf16*>(W13_s);
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
    case 256: return launch_decode_nv<1>(m2, m2s, a, sms, st);
    case 512: return launch_decode_nv<2>(m2, m2s, a, sms, st);
    case 1024: return launch_decode_nv<4>(m2, m2s, a, sms, st);
    case 2048: return launch_decode_nv<8>(m2, m2s, a, sms, st);
    default: return MOE_ERR_SHAPE;
  }
}

}  // namespace moe
