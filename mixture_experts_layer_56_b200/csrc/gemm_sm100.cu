// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM),
// fed by TMA, for the SwiGLU experts of the DeepSeekMoE layer (§3.2,
// eq. (9); the expert FFN is W2 (SiLU(W1 x) * W3 x)).
//
// One persistent kernel computes, for every group g (the shared-expert group,
// then routed expert e = 0..N_r-1), D_g = A_g * B_g^T over 128-row x BN-column
// tiles:
//   gate/up launch: A = gathered token rows [n_e, d], B = packed W13_e [2I, d];
//                   epilogue a = SiLU(D[:, gate]) * D[:, up] -> bf16 [n_e, I]
//   down launch:    A = a [n_e, I],  B = W2_e [d, I];  epilogue D -> y
// The shared experts form one group whose FFN has width K_s*I (their sum is
// one wider SwiGLU FFN, the segmentation identity of §3.1).
//
// Roles (256 threads): warp 0 lane 0 issues TMA loads into a STAGES-deep
// shared-memory ring; warp 1 lane 0 issues tcgen05.mma into one of two TMEM
// accumulators; warp 2 owns the TMEM allocation; warps 4-7 drain a finished
// accumulator (tcgen05.ld), apply the epilogue and store rows < n_e directly
// to global memory, so tiles never write into a neighbouring expert's rows.
// Groups are unpadded: A rows past a group's end are read (and ignored) or
// zero-filled by TMA past the tensor's end.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "gemm_sm100.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace sm100 {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 384;  // 4 role warps + 8 epilogue warps
constexpr int kMaxGroups = 257;  // 256 routed + 1 shared

// Stage layout by the N tile BN and the A rows a stage holds, AR: 128, or 64
// / 32 for batches whose groups have at most that many rows (fewer than 128
// tokens).  The MMA still reads 128 rows of A from the stage's start; the
// rows past AR are other bytes of the same stage (AR * 128 + BN * 128 >=
// 16 KB), their accumulator rows never stored.  Smaller A leaves room for
// more stages of B, the weights that decode-sized batches stream.
template <int BN, int AR> struct Cfg {
  static constexpr int kBytes = AR * BK * 2 + BN * BK * 2;
  static constexpr int STAGES = (216 * 1024) / kBytes < 32 ? (216 * 1024) / kBytes : 32;
  static_assert(kBytes >= BM * BK * 2, "the MMA's 128 rows of A stay inside the stage");
};
template <> struct Cfg<256, 128> { static constexpr int STAGES = 4; };
template <> struct Cfg<128, 128> { static constexpr int STAGES = 6; };
template <> struct Cfg<64, 128>  { static constexpr int STAGES = 8; };

template <int BN, int AR>
constexpr int smem_bytes() {
  return Cfg<BN, AR>::STAGES * (AR * BK * 2 + BN * BK * 2) + 1024;
}

// When every group fits one row block (decode-sized batches) each B tile is
// read by one tile only: its L2 lines go first, so that the rows of A, the
// outputs and the next kernels' inputs stay in L2 while the weights stream.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void tma_load_3d_evict_first(uint32_t dst, const CUtensorMap* map,
                                                        uint32_t bar, int32_t x, int32_t y,
                                                        int32_t z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z), "l"(policy)
      : "memory");
}

struct TileInfo {
  int g;        // group index (0 = shared when present)
  int shared;   // 1 for the shared-expert group
  int m_blk;
  int n_blk;
};

__device__ __forceinline__ TileInfo decode_tile(int tile, const int32_t* tile_start, int G, int hs,
                                                int nt_r, int nt_s) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  TileInfo t;
  t.g = lo;
  t.shared = (hs && lo == 0) ? 1 : 0;
  const int nt = t.shared ? nt_s : nt_r;
  const int local = tile - tile_start[lo];
  t.m_blk = local / nt;
  t.n_blk = local - t.m_blk * nt;
  return t;
}

template <int BN, int EPI, int AR>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
                    const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
                    const GroupedGemmArgs args) {
  constexpr int STAGES = Cfg<BN, AR>::STAGES;
  constexpr uint32_t A_BYTES = AR * BK * 2;
  constexpr uint32_t B_BYTES = BN * BK * 2;
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);
  // SwiGLU epilogues drain with 8 warps (two per TMEM lane quarter, one per
  // half of the columns); plain ones with 4
  constexpr int EPI_WARPS = EPI == kEpiSwiGLU ? 8 : 4;

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * STAGES + 5];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int32_t tile_start[kMaxGroups + 1];
  __shared__ int32_t grp_row0[kMaxGroups];
  __shared__ int32_t grp_rows[kMaxGroups];
  __shared__ int b_once;  // every group fits one row block: each B tile is read once

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = smem_addr(smem);
  const uint32_t bar_base = smem_addr(bars);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar_base + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar_base + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar_base + 8u * (2 * STAGES + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int hs = args.shared_rows > 0 ? 1 : 0;
  const int G = args.n_routed + hs;
  volatile int* abort_p = &abort_flag;

  // ---- per-CTA setup: barriers, TMEM, group tile prefix ------------------
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), EPI_WARPS);  // one arrive per epilogue warp
    }
    mbar_init(drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    fence_async_shared();
  }
  if (warp == 2) {
    tmem_alloc(smem_addr(&tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();  // offsets, operands and outputs belong to earlier stream work
  pdl_trigger();
  for (int g = tid; g < G; g += kThreads) {
    int rows, row0, nt;
    if (hs && g == 0) {
      rows = args.shared_rows; row0 = 0; nt = args.nt_shared;
    } else {
      const int e = g - hs;
      row0 = args.offsets[e];
      rows = args.offsets[e + 1] - row0;
      nt = args.nt_routed;
    }
    grp_row0[g] = row0;
    grp_rows[g] = rows;
    tile_start[g + 1] = ((rows + BM - 1) / BM) * nt;
  }
  __syncthreads();
  if (warp == 0) {
    const int per = (G + 31) / 32;
    const int beg = min(lane * per, G);
    const int end = min(beg + per, G);
    int sum = 0;
    for (int i = beg; i < end; ++i) sum += tile_start[i + 1];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - sum;
    bool big = false;
    for (int i = beg; i < end; ++i) {
      run += tile_start[i + 1];
      tile_start[i + 1] = run;
      big = big || grp_rows[i] > BM;
    }
    big = __any_sync(0xffffffffu, big);
    if (lane == 0) {
      tile_start[0] = 0;
      b_once = big ? 0 : 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  const int total_tiles = tile_start[G];
  const int n_long = (hs && args.kb_shared > args.kb_routed) ? tile_start[1] : 0;
  const int workers = static_cast<int>(gridDim.x);

  if (warp == 0) {
    // ---------------------------------------------------- TMA producer ----
    if (lane == 0) {
      tma_prefetch_desc(&tmA_r);
      tma_prefetch_desc(&tmB_r);
      if (hs) {
        tma_prefetch_desc(&tmA_s);
        tma_prefetch_desc(&tmB_s);
      }
      const uint32_t a_bytes =
          static_cast<uint32_t>(args.a_rows > 0 && args.a_rows < AR ? args.a_rows : AR) * BK * 2;
      const uint64_t b_policy = l2_evict_first_policy();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;
      bool ok = true;
      if (args.inject_wait_timeout) {
        // slot 0 is released only after a load into it has been consumed,
        // and none was issued: this wait runs out
        if (!wait_bounded(empty_bar(0), 0u, abort_p, args.status, kInjectedWaitNs)) ok = false;
      }
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        const TileInfo ti = decode_tile(place_tile(tile, total_tiles, workers, n_long), tile_start, G, hs,
                                        args.nt_routed, args.nt_shared);
        const CUtensorMap* ma = ti.shared ? &tmA_s : &tmA_r;
        const CUtensorMap* mb = ti.shared ? &tmB_s : &tmB_r;
        const int row = grp_row0[ti.g] + ti.m_blk * BM;
        const int nrow = ti.n_blk * BN;
        const int nkb = ti.shared ? args.kb_shared : args.kb_routed;
        const int zbase = ti.shared ? 0 : ti.g - hs;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_p, args.status)) { ok = false; break; }
          const uint32_t sa = smem_base + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(full_bar(stage), a_bytes + B_BYTES);
          tma_load_2d(sa, ma, full_bar(stage), kb * BK, row);
          if (b_once)
            tma_load_3d_evict_first(sa + A_BYTES, mb, full_bar(stage),
                                    (kb % args.kb_per_expert) * BK, nrow,
                                    zbase + kb / args.kb_per_expert, b_policy);
          else
            tma_load_3d(sa + A_BYTES, mb, full_bar(stage), (kb % args.kb_per_expert) * BK, nrow,
                        zbase + kb / args.kb_per_expert);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // let every load already in flight land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s)) {
            int dummy = 0;
            wait_bounded(full_bar(s), (issued_parity >> s) & 1u, &dummy, nullptr);
          }
      } else {
        // the last round's "empty" arrivals land in this CTA's shared memory:
        // wait for them so that none is still in flight when the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s)) {
            int dummy = 0;
            wait_bounded(empty_bar(s), (issued_parity >> s) & 1u, &dummy, nullptr);
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer ----
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++it) {
        const TileInfo ti = decode_tile(place_tile(tile, total_tiles, workers, n_long), tile_start, G, hs,
                                        args.nt_routed, args.nt_shared);
        const int nkb = ti.shared ? args.kb_shared : args.kb_routed;
        const int acc = it & 1;
        const uint32_t ap = (it >> 1) & 1;
        if (!wait_bounded(tempty_bar(acc), ap ^ 1u, abort_p, args.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_bounded(full_bar(stage), phase, abort_p, args.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            mma_bf16(d_tmem, desc_kmajor_sw128(sa + k * 32), desc_kmajor_sw128(sb + k * 32), IDESC,
                     (kb > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok) mma_commit(tfull_bar(acc));
      }
      if (!ok) {
        // wait for every MMA already issued before TMEM is released
        mma_commit(drain_bar);
        int dummy = 0;
        wait_bounded(drain_bar, 0, &dummy, nullptr);
      }
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 4 + EPI_WARPS) {
    // ------------------------------------------------------- epilogue -----
    const int q = warp & 3;          // TMEM lane quarter of this warp
    const int hcol = (warp - 4) >> 2;  // which half of the tile's columns it drains
    const int r = q * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      const TileInfo ti = decode_tile(place_tile(tile, total_tiles, workers, n_long), tile_start, G, hs,
                                        args.nt_routed, args.nt_shared);
      const int acc = it & 1;
      const uint32_t ap = (it >> 1) & 1;
      if (!wait_bounded(tfull_bar(acc), ap, abort_p, args.status)) break;
      tc_fence_after();
      const int rows_valid = grp_rows[ti.g] - ti.m_blk * BM;
      const int64_t orow = static_cast<int64_t>(grp_row0[ti.g]) + ti.m_blk * BM + r;
      const bool live = r < rows_valid;
      // routed rows of the plain epilogue may be remapped (token-slot order)
      const int64_t prow = (EPI == kEpiPlain && !ti.shared && args.row_map_r != nullptr && live)
                               ? static_cast<int64_t>(args.row_map_r[orow])
                               : orow;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      if (EPI == kEpiSwiGLU) {
        bf16* out = static_cast<bf16*>(ti.shared ? args.out_s : args.out_r);
        const int64_t ld = ti.shared ? args.ld_s : args.ld_r;
        const int64_t col0 = static_cast<int64_t>(ti.n_blk) * (BN / 2);
#pragma unroll 1
        for (int c = hcol * (BN / 128); c < (hcol + 1) * (BN / 128); ++c) {  // 8 warps
          const int pair = c >> 1, half = c & 1;
          const int gcol = pair * 128 + half * 32;
          float gv[32], uv[32];
          tmem_ld32(taddr + gcol, gv);
          tmem_ld32(taddr + gcol + 64, uv);
          tmem_ld_wait();
          if (live) {
            bf16* dst = out + orow * ld + col0 + pair * 64 + half * 32;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float o[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) o[j] = silu_mul(gv[v * 8 + j], uv[v * 8 + j]);
              Vec16<bf16>::store(dst + v * 8, o);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {  // 4 warps
          float x[32];
          tmem_ld32(taddr + c * 32, x);
          tmem_ld_wait();
          if (live) {
            const int64_t col = static_cast<int64_t>(ti.n_blk) * BN + c * 32;
            if (ti.shared) {
              float* dst = static_cast<float*>(args.out_s) + orow * args.ld_s + col;
#pragma unroll
              for (int v = 0; v < 8; ++v) Vec16<float>::store(dst + v * 4, x + v * 4);
            } else {
              bf16* dst = static_cast<bf16*>(args.out_r) + prow * args.ld_r + col;
#pragma unroll
              for (int v = 0; v < 4; ++v) Vec16<bf16>::store(dst + v * 8, x + v * 8);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// --------------------------------------------------------------------------
// host side
// --------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_map_bf16(CUtensorMap* map, int rank, const void* base, uint64_t inner, uint64_t rows,
                   uint64_t depth, uint64_t row_stride_bytes, uint64_t depth_stride_bytes,
                   uint32_t box_rows, uint32_t box_k) {
  auto fn = encode_fn();
  if (!fn || !base || inner == 0 || rows == 0 || depth == 0 || (rank != 2 && rank != 3))
    return false;
  if (rank == 2 && depth != 1) return false;
  cuuint64_t dims[3] = {inner, rows, depth};
  cuuint64_t strides[2] = {row_stride_bytes, depth_stride_bytes};
  if (box_k != 64 && box_k != 32) return false;
  cuuint32_t box[3] = {box_k, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult res = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    box_k == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                 uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn || !base || inner == 0 || rows == 0) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult res = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

template <int BN, int EPI, int AR>
static int launch_impl(const GemmMaps& m, const GroupedGemmArgs& args, int grid,
                       cudaStream_t stream) {
  static std::atomic<uint64_t> optin{0};
  auto kern = grouped_gemm_kernel<BN, EPI, AR>;
  constexpr int smem = smem_bytes<BN, AR>();
  if (int rc = ensure_smem_optin(reinterpret_cast<const void*>(kern), smem, optin)) return rc;
  return launch_k(kern, grid, kThreads, smem, stream, 1, m.a_r, m.a_s, m.b_r, m.b_s, args);
}

// the stage layout for the A rows of the batch (a_rows 0 means 128)
template <int BN, int EPI>
static int launch_rows(const GemmMaps& m, const GroupedGemmArgs& args, int grid,
                       cudaStream_t stream) {
  const int ar = args.a_rows > 0 ? args.a_rows : BM;
  if constexpr (BN >= 128) {
    if (ar <= 32) return launch_impl<BN, EPI, 32>(m, args, grid, stream);
  }
  if (ar <= 64) return launch_impl<BN, EPI, 64>(m, args, grid, stream);
  return launch_impl<BN, EPI, 128>(m, args, grid, stream);
}

int launch_grouped_gemm(int BN, int epi, const GemmMaps& maps, const GroupedGemmArgs& args,
                        int grid, cudaStream_t stream) {
  if (grid <= 0) return MOE_OK;
  if (epi == kEpiSwiGLU) {
    if (BN == 256) return launch_rows<256, kEpiSwiGLU>(maps, args, grid, stream);
    if (BN == 128) return launch_rows<128, kEpiSwiGLU>(maps, args, grid, stream);
  } else {
    if (BN == 256) return launch_rows<256, kEpiPlain>(maps, args, grid, stream);
    if (BN == 128) return launch_rows<128, kEpiPlain>(maps, args, grid, stream);
    if (BN == 64) return launch_rows<64, kEpiPlain>(maps, args, grid, stream);
  }
  return MOE_ERR_SHAPE;
}

}  // namespace sm100
}  // namespace moe
