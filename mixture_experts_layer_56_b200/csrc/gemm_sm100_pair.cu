// Grouped expert GEMM on CTA pairs (tcgen05 cta_group::2): the same
// computation as gemm_sm100.cu (gate/up + SwiGLU, or down projection, over
// the shared group and the routed experts of the DeepSeekMoE layer, §3.2
// eq. (9)) with 256-row tiles split over the two SMs of a cluster.
//
// The leader CTA (rank 0) issues every MMA of the pair: M = 256 (rows 0..127
// from its own shared memory, 128..255 from the peer's), N = BN (B rows
// split in halves the same way), accumulating 128 rows x BN fp32 columns in
// each CTA's TMEM.  Each CTA loads its own A rows and B half with TMA; all
// transaction bytes land on the leader's "full" barrier, whose expected
// count the leader sets for both.  The leader's commits arrive on the
// "empty" and "accumulator full" barriers of both CTAs at once; both
// epilogues release an accumulator on the leader's "accumulator empty"
// barrier.  Per CTA and k-block this moves 16 KB of A and BN*64 B of B,
// against 16 KB + BN*128 B for one CTA computing half the tile alone.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_sm100.h"
#include "sm100_ptx.cuh"

namespace moe {
namespace sm100 {

namespace {

constexpr int PBM = 256;   // rows per pair tile
constexpr int HBM_ROWS = 128;  // rows per CTA
constexpr int PBK = 64;
constexpr int kPairThreads = 384;  // 4 role warps + 8 epilogue warps
constexpr int kPairMaxGroups = 257;

// Epilogue staging: every epilogue warp owns 32 rows x (128 + 16) bytes of
// shared memory; rows are padded by 16 bytes so that 32 lanes writing one
// row each hit distinct banks.
constexpr int kStageRowBytes = 128;
constexpr int kStagePitch = kStageRowBytes + 16;
constexpr int kWarpStageBytes = 32 * kStagePitch;

template <int EPI> constexpr int pair_epi_warps() { return 8; }

// pipeline depth: as many 256-row k-block stages as fit beside the staging
template <int BN, int EPI>
constexpr int pair_stages() {
  return (216 * 1024 - pair_epi_warps<EPI>() * kWarpStageBytes) /
         (HBM_ROWS * PBK * 2 + (BN / 2) * PBK * 2);
}

template <int BN, int EPI>
constexpr int pair_smem_bytes() {
  return pair_stages<BN, EPI>() * (HBM_ROWS * PBK * 2 + (BN / 2) * PBK * 2) +
         pair_epi_warps<EPI>() * kWarpStageBytes + 1024;
}

// A warp's 32 rows of ROW_BYTES bytes each (lane r holds row r in `v`) go
// to global memory through its shared staging area, as full row segments:
// ROW_BYTES / 16 lanes write one row, so one store instruction covers
// 512 / ROW_BYTES rows with whole 32-byte sectors.  `dst` is lane r's row
// start (nullptr: row r is not written).
template <int ROW_BYTES>
__device__ __forceinline__ void warp_store_rows(uint8_t* stage, const uint4* v, uint8_t* dst,
                                                int lane) {
  constexpr int CH = ROW_BYTES / 16;  // 16-byte chunks per row
  constexpr int RPI = 32 / CH;        // rows per store instruction
#pragma unroll
  for (int c = 0; c < CH; ++c)
    *reinterpret_cast<uint4*>(stage + lane * kStagePitch + c * 16) = v[c];
  __syncwarp();
#pragma unroll
  for (int it = 0; it < CH; ++it) {
    const int row = it * RPI + lane / CH;
    const int c = lane % CH;
    uint8_t* rdst = reinterpret_cast<uint8_t*>(
        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dst), row));
    const uint4 x = *reinterpret_cast<const uint4*>(stage + row * kStagePitch + c * 16);
    if (rdst != nullptr) *reinterpret_cast<uint4*>(rdst + c * 16) = x;
  }
  __syncwarp();
}

struct PairTile {
  int g, shared, m_blk, n_blk;
};

// A group's tiles run in column chunks of `cn` N tiles: all of its row blocks
// against the first cn N tiles, then the next cn, and so on (cn >= nt: plain
// row-major order).  The workers in flight then share one chunk of B, which
// L2 can hold while the row blocks of A stream past, where row-major order
// sweeps the whole of a wide group's B once per few row blocks.  (A group a
// tile falls in always has tiles, so mt > 0.)
__device__ __forceinline__ PairTile decode_pair_tile(int tile, const int32_t* tile_start, int G,
                                                     int hs, int nt_r, int nt_s, int cn) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  PairTile t;
  t.g = lo;
  t.shared = (hs && lo == 0) ? 1 : 0;
  const int nt = t.shared ? nt_s : nt_r;
  const int local = tile - tile_start[lo];
  const int mt = (tile_start[lo + 1] - tile_start[lo]) / nt;  // row blocks of the group
  const int cw = cn < nt ? cn : nt;                          // chunk width
  const int c = local / (cw * mt);
  const int rem = local - c * cw * mt;
  const int wc = min(cw, nt - c * cw);                       // N tiles of this chunk
  t.m_blk = rem / wc;
  t.n_blk = c * cw + (rem - t.m_blk * wc);
  return t;
}

constexpr int kRowMajor = 1 << 24;  // chunk width that never splits a group

template <int BN, int EPI>
__global__ void __launch_bounds__(kPairThreads, 1)
grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA_r,
                         const __grid_constant__ CUtensorMap tmA_s,
                         const __grid_constant__ CUtensorMap tmB_r,
                         const __grid_constant__ CUtensorMap tmB_s, const GroupedGemmArgs args) {
  constexpr int STAGES = pair_stages<BN, EPI>();
  constexpr uint32_t A_BYTES = HBM_ROWS * PBK * 2;
  constexpr uint32_t B_BYTES = (BN / 2) * PBK * 2;
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  constexpr uint32_t IDESC = idesc_bf16_f32(PBM, BN);
  // epilogues drain with 8 warps: two per TMEM lane quarter, one per half
  // of the tile's columns
  constexpr int EPI_WARPS = pair_epi_warps<EPI>();
  constexpr uint16_t kBoth = 0x3;

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * STAGES + 5];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int32_t tile_start[kPairMaxGroups + 1];
  __shared__ int32_t grp_row0[kPairMaxGroups];
  __shared__ int32_t grp_rows[kPairMaxGroups];

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
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = static_cast<int>(cluster_id_x());
  const int nclusters = static_cast<int>(num_clusters_x());
  const int hs = args.shared_rows > 0 ? 1 : 0;
  const int G = args.n_routed + hs;
  volatile int* abort_p = &abort_flag;

  // ---- setup --------------------------------------------------------------
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);   // the leader's arrive (+ both CTAs' bytes)
      mbar_init(empty_bar(s), 1);  // one multicast commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);   // one multicast commit
      mbar_init(tempty_bar(a), 2 * EPI_WARPS);  // epilogue warps of both CTAs (leader's copy)
    }
    mbar_init(drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    fence_async_shared();
  }
  if (warp == 2) {
    tmem_alloc_pair(smem_addr(&tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  pdl_wait();  // offsets, operands and outputs belong to earlier stream work
  pdl_trigger();
  for (int g = tid; g < G; g += kPairThreads) {
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
    tile_start[g + 1] = ((rows + PBM - 1) / PBM) * nt;
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
    for (int i = beg; i < end; ++i) {
      run += tile_start[i + 1];
      tile_start[i + 1] = run;
    }
    if (lane == 0) tile_start[0] = 0;
  }
  tc_fence_before();
  cluster_sync_all();  // barrier inits and TMEM allocations visible to the pair
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  const int total_tiles = tile_start[G];
  const int n_long = (hs && args.kb_shared > args.kb_routed) ? tile_start[1] : 0;

  if (warp == 0) {
    // ---------------------------------------------------- TMA producer ----
    if (lane == 0) {
      tma_prefetch_desc(&tmA_r);
      tma_prefetch_desc(&tmB_r);
      if (hs) {
        tma_prefetch_desc(&tmA_s);
        tma_prefetch_desc(&tmB_s);
      }
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      if (args.inject_wait_timeout) {
        // slot 0 is released only after a load into it has been consumed,
        // and none was issued: this wait runs out
        if (!wait_bounded(empty_bar(0), 0u, abort_p, args.status, kInjectedWaitNs)) ok = false;
      }
      for (int tile = cluster; tile < total_tiles && ok; tile += nclusters) {
        const PairTile ti =
            decode_pair_tile(place_tile(tile, total_tiles, nclusters, n_long), tile_start, G, hs,
                             args.nt_routed, args.nt_shared, kRowMajor);
        const CUtensorMap* ma = ti.shared ? &tmA_s : &tmA_r;
        const CUtensorMap* mb = ti.shared ? &tmB_s : &tmB_r;
        const int row = grp_row0[ti.g] + ti.m_blk * PBM + static_cast<int>(rank) * HBM_ROWS;
        const int nrow = ti.n_blk * BN + static_cast<int>(rank) * (BN / 2);
        const int nkb = ti.shared ? args.kb_shared : args.kb_routed;
        const int zbase = ti.shared ? 0 : ti.g - hs;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_p, args.status)) { ok = false; break; }
          const uint32_t sa = smem_base + stage * STAGE_BYTES;
          const uint32_t fb = leader ? full_bar(stage) : map_to_cta(full_bar(stage), 0);
          if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
          tma_load_2d_pair(sa, ma, fb, kb * PBK, row);
          tma_load_3d_pair(sa + A_BYTES, mb, fb, (kb % args.kb_per_expert) * PBK, nrow,
                           zbase + kb / args.kb_per_expert);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (ok) {
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
    // ----------------------------------------- MMA issuer (leader only) ----
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = cluster; tile < total_tiles && ok; tile += nclusters, ++it) {
        const PairTile ti =
            decode_pair_tile(place_tile(tile, total_tiles, nclusters, n_long), tile_start, G, hs,
                             args.nt_routed, args.nt_shared, kRowMajor);
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
          for (int k = 0; k < PBK / 16; ++k) {
            mma_bf16_pair(d_tmem, desc_kmajor_sw128(sa + k * 32), desc_kmajor_sw128(sb + k * 32),
                          IDESC, (kb > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit_pair(empty_bar(stage), kBoth);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok) mma_commit_pair(tfull_bar(acc), kBoth);
      }
      if (!ok) {
        // wait for every MMA already issued before TMEM is released
        mma_commit_pair(drain_bar, 0x1);
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
    const uint32_t tempty_leader0 = map_to_cta(tempty_bar(0), 0);
    const uint32_t tempty_leader1 = map_to_cta(tempty_bar(1), 0);
    int it = 0;
    for (int tile = cluster; tile < total_tiles; tile += nclusters, ++it) {
      const PairTile ti =
          decode_pair_tile(place_tile(tile, total_tiles, nclusters, n_long), tile_start, G, hs,
                             args.nt_routed, args.nt_shared, kRowMajor);
      const int acc = it & 1;
      const uint32_t ap = (it >> 1) & 1;
      if (!wait_bounded(tfull_bar(acc), ap, abort_p, args.status)) break;
      tc_fence_after();
      const int my0 = ti.m_blk * PBM + static_cast<int>(rank) * HBM_ROWS;
      const int rows_valid = grp_rows[ti.g] - my0;
      const int64_t orow = static_cast<int64_t>(grp_row0[ti.g]) + my0 + r;
      const bool live = r < rows_valid;
      // routed rows of the plain epilogue may be remapped (token-slot order)
      const int64_t prow = (EPI == kEpiPlain && !ti.shared && args.row_map_r != nullptr && live)
                               ? static_cast<int64_t>(args.row_map_r[orow])
                               : orow;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      uint8_t* stage = smem + STAGES * STAGE_BYTES + (warp - 4) * kWarpStageBytes;
      if (EPI == kEpiSwiGLU) {
        // this warp's output columns: 64 (BN = 256) or 32 (BN = 128)
        constexpr int OC = BN / 4;
        bf16* out = static_cast<bf16*>(ti.shared ? args.out_s : args.out_r);
        const int64_t ld = ti.shared ? args.ld_s : args.ld_r;
        const int64_t col0 = static_cast<int64_t>(ti.n_blk) * (BN / 2) + hcol * OC;
        uint4 packed[OC / 8];
#pragma unroll
        for (int h = 0; h < OC / 32; ++h) {
          // packed blocks of 128 columns are [gate 64 | up 64]; this warp's
          // gate columns start at 128*hcol (BN = 256) or 32*hcol (BN = 128)
          const int gcol = (BN == 256 ? hcol * 128 : hcol * 32) + h * 32;
          const int ucol = gcol + 64;
          float gv[32], uv[32];
          tmem_ld32(taddr + gcol, gv);
          tmem_ld32(taddr + ucol, uv);
          tmem_ld_wait();
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            float o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) o[j] = silu_mul(gv[v * 8 + j], uv[v * 8 + j]);
            Vec16<bf16>::store(reinterpret_cast<bf16*>(&packed[h * 4 + v]), o);
          }
        }
        uint8_t* dst = live ? reinterpret_cast<uint8_t*>(out + orow * ld + col0) : nullptr;
        warp_store_rows<OC * 2>(stage, packed, dst, lane);
      } else if (ti.shared) {
        // fp32 shared-expert output: chunks of 32 columns (128 bytes a row);
        // the TMEM load of chunk c+1 is in flight while chunk c is stored
        constexpr int WC = BN / 2;
        constexpr int NCH = WC / 32;
        const int c0 = hcol * WC;
        float x[32];
        tmem_ld32(taddr + c0, x);
        tmem_ld_wait_regs(x);
#pragma unroll 1
        for (int c = 0; c < NCH; ++c) {
          uint4 packed[8];
#pragma unroll
          for (int v = 0; v < 8; ++v)
            packed[v] = make_uint4(__float_as_uint(x[4 * v]), __float_as_uint(x[4 * v + 1]),
                                   __float_as_uint(x[4 * v + 2]), __float_as_uint(x[4 * v + 3]));
          if (c + 1 < NCH) tmem_ld32(taddr + c0 + (c + 1) * 32, x);
          const int64_t col = static_cast<int64_t>(ti.n_blk) * BN + c0 + c * 32;
          uint8_t* dst = live ? reinterpret_cast<uint8_t*>(static_cast<float*>(args.out_s) +
                                                           orow * args.ld_s + col)
                              : nullptr;
          warp_store_rows<128>(stage, packed, dst, lane);
          if (c + 1 < NCH) tmem_ld_wait_regs(x);
        }
      } else {
        // bf16 routed output: chunks of up to 64 columns (128 bytes a row),
        // next chunk's TMEM load overlapping this chunk's stores
        constexpr int WC = BN / 2;
        constexpr int CW = WC < 64 ? WC : 64;
        constexpr int NCH = WC / CW;
        const int c0 = hcol * WC;
        float x[CW];
#pragma unroll
        for (int h = 0; h < CW / 32; ++h) tmem_ld32(taddr + c0 + h * 32, x + h * 32);
#pragma unroll
        for (int h = 0; h < CW / 32; ++h) tmem_ld_wait_regs(x + h * 32);
#pragma unroll 1
        for (int c = 0; c < NCH; ++c) {
          uint4 packed[CW / 8];
#pragma unroll
          for (int v = 0; v < CW / 8; ++v)
            Vec16<bf16>::store(reinterpret_cast<bf16*>(&packed[v]), x + v * 8);
          if (c + 1 < NCH) {
#pragma unroll
            for (int h = 0; h < CW / 32; ++h)
              tmem_ld32(taddr + c0 + (c + 1) * CW + h * 32, x + h * 32);
          }
          const int64_t col = static_cast<int64_t>(ti.n_blk) * BN + c0 + c * CW;
          uint8_t* dst = live ? reinterpret_cast<uint8_t*>(static_cast<bf16*>(args.out_r) +
                                                           prow * args.ld_r + col)
                              : nullptr;
          warp_store_rows<CW * 2>(stage, packed, dst, lane);
          if (c + 1 < NCH) {
#pragma unroll
            for (int h = 0; h < CW / 32; ++h) tmem_ld_wait_regs(x + h * 32);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
    }
  }

  tc_fence_before();
  cluster_sync_all();  // no CTA of the pair leaves while the other still works
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Wide pair tiles: 256 rows x 512 columns per CTA pair.  Per 64-wide k-block
// each CTA takes in its 128 rows of A (16 KB) and 256 rows of B (32 KB: its
// 128-row share of each of two 256-column slices) and the leader issues two
// M = 256, N = 256 pair MMAs, one per slice.  That is 48 bytes of tiles per
// clock of full-rate tensor work where 256-column tiles need 64.  The
// accumulator fills all 512 TMEM columns, so it is not double-buffered;
// its two 256-column halves are released separately instead: the next
// tile's first MMAs into half 0 start as soon as the epilogue has drained
// half 0, while it drains half 1.
// ---------------------------------------------------------------------------
constexpr int kWideBN = 512;
constexpr int kWideHalf = 256;
constexpr int kWideEpiWarps = 8;
// column chunk of the tile order: 8 tiles of 512 columns, 32 MB of B at
// K = 4096 (the large layer's shared gate/up group is 24 tiles wide); it took
// that layer's gate/up DRAM reads from 15.6 to 12.8 GB per launch
constexpr int kWideChunk = 8;

// Stage size and count by the k-block width BKW (kWideBK): 64 gives three
// 48 KB stages beside the epilogue staging.
template <int BKW>
constexpr int wide_stage_bytes() {
  return HBM_ROWS * BKW * 2 + (kWideBN / 2) * BKW * 2;
}
template <int BKW>
constexpr int wide_stages() {
  return (216 * 1024 - kWideEpiWarps * kWarpStageBytes) / wide_stage_bytes<BKW>();
}
template <int BKW>
constexpr int wide_smem_bytes() {
  return wide_stages<BKW>() * wide_stage_bytes<BKW>() + kWideEpiWarps * kWarpStageBytes + 1024;
}

template <int BKW>
__device__ __forceinline__ uint64_t wide_desc(uint32_t saddr) {
  return BKW == 64 ? desc_kmajor_sw128(saddr) : desc_kmajor_sw64(saddr);
}

template <int EPI, int BKW>
__global__ void __launch_bounds__(kPairThreads, 1)
grouped_gemm_pair_wide_kernel(const __grid_constant__ CUtensorMap tmA_r,
                              const __grid_constant__ CUtensorMap tmA_s,
                              const __grid_constant__ CUtensorMap tmB_r,
                              const __grid_constant__ CUtensorMap tmB_s,
                              const GroupedGemmArgs args) {
  constexpr int STAGES = wide_stages<BKW>();
  constexpr uint32_t A_BYTES = HBM_ROWS * BKW * 2;
  constexpr uint32_t BH_BYTES = 128 * BKW * 2;  // this CTA's rows of one 256-column slice
  constexpr uint32_t STAGE_BYTES = A_BYTES + 2 * BH_BYTES;
  constexpr uint32_t TMEM_COLS = 512;
  constexpr uint32_t IDESC = idesc_bf16_f32(PBM, kWideHalf);
  constexpr int EPI_WARPS = kWideEpiWarps;
  constexpr uint16_t kBoth = 0x3;

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * STAGES + 5];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int32_t tile_start[kPairMaxGroups + 1];
  __shared__ int32_t grp_row0[kPairMaxGroups];
  __shared__ int32_t grp_rows[kPairMaxGroups];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = smem_addr(smem);
  const uint32_t bar_base = smem_addr(bars);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto tfull_bar = [&](int h) { return bar_base + 8u * (2 * STAGES + h); };
  auto tempty_bar = [&](int h) { return bar_base + 8u * (2 * STAGES + 2 + h); };
  const uint32_t drain_bar = bar_base + 8u * (2 * STAGES + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = static_cast<int>(cluster_id_x());
  const int nclusters = static_cast<int>(num_clusters_x());
  const int hs = args.shared_rows > 0 ? 1 : 0;
  const int G = args.n_routed + hs;
  volatile int* abort_p = &abort_flag;

  // ---- setup --------------------------------------------------------------
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);   // the leader's arrive (+ both CTAs' bytes)
      mbar_init(empty_bar(s), 1);  // one multicast commit
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(tfull_bar(h), 1);                 // one multicast commit
      mbar_init(tempty_bar(h), 2 * EPI_WARPS);    // epilogue warps of both CTAs (leader's copy)
    }
    mbar_init(drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    fence_async_shared();
  }
  if (warp == 2) {
    tmem_alloc_pair(smem_addr(&tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  pdl_wait();  // offsets, operands and outputs belong to earlier stream work
  pdl_trigger();
  for (int g = tid; g < G; g += kPairThreads) {
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
    tile_start[g + 1] = ((rows + PBM - 1) / PBM) * nt;
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
    for (int i = beg; i < end; ++i) {
      run += tile_start[i + 1];
      tile_start[i + 1] = run;
    }
    if (lane == 0) tile_start[0] = 0;
  }
  tc_fence_before();
  cluster_sync_all();  // barrier inits and TMEM allocations visible to the pair
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  const int total_tiles = tile_start[G];
  const int n_long = (hs && args.kb_shared > args.kb_routed) ? tile_start[1] : 0;

  if (warp == 0) {
    // ---------------------------------------------------- TMA producer ----
    if (lane == 0) {
      tma_prefetch_desc(&tmA_r);
      tma_prefetch_desc(&tmB_r);
      if (hs) {
        tma_prefetch_desc(&tmA_s);
        tma_prefetch_desc(&tmB_s);
      }
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      if (args.inject_wait_timeout) {
        // slot 0 is released only after a load into it has been consumed,
        // and none was issued: this wait runs out
        if (!wait_bounded(empty_bar(0), 0u, abort_p, args.status, kInjectedWaitNs)) ok = false;
      }
      for (int tile = cluster; tile < total_tiles && ok; tile += nclusters) {
        const PairTile ti =
            decode_pair_tile(place_tile(tile, total_tiles, nclusters, n_long), tile_start, G, hs,
                             args.nt_routed, args.nt_shared, kWideChunk);
        const CUtensorMap* ma = ti.shared ? &tmA_s : &tmA_r;
        const CUtensorMap* mb = ti.shared ? &tmB_s : &tmB_r;
        const int row = grp_row0[ti.g] + ti.m_blk * PBM + static_cast<int>(rank) * HBM_ROWS;
        const int nrow = ti.n_blk * kWideBN + static_cast<int>(rank) * 128;
        const int nkb = ti.shared ? args.kb_shared : args.kb_routed;
        const int zbase = ti.shared ? 0 : ti.g - hs;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_p, args.status)) { ok = false; break; }
          const uint32_t sa = smem_base + stage * STAGE_BYTES;
          const uint32_t fb = leader ? full_bar(stage) : map_to_cta(full_bar(stage), 0);
          const int kx = (kb % args.kb_per_expert) * BKW;
          const int kz = zbase + kb / args.kb_per_expert;
          if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
          tma_load_2d_pair(sa, ma, fb, kb * BKW, row);
          tma_load_3d_pair(sa + A_BYTES, mb, fb, kx, nrow, kz);
          tma_load_3d_pair(sa + A_BYTES + BH_BYTES, mb, fb, kx, nrow + kWideHalf, kz);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (ok) {
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
    // ----------------------------------------- MMA issuer (leader only) ----
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = cluster; tile < total_tiles && ok; tile += nclusters, ++it) {
        const PairTile ti =
            decode_pair_tile(place_tile(tile, total_tiles, nclusters, n_long), tile_start, G, hs,
                             args.nt_routed, args.nt_shared, kWideChunk);
        const int nkb = ti.shared ? args.kb_shared : args.kb_routed;
        const uint32_t tp = static_cast<uint32_t>(it & 1);
        for (int kb = 0; kb < nkb && ok; ++kb) {
          if (!wait_bounded(full_bar(stage), phase, abort_p, args.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_base + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          for (int h = 0; h < 2; ++h) {
            if (kb == 0) {
              // the epilogue has drained this half of the previous tile
              if (!wait_bounded(tempty_bar(h), tp ^ 1u, abort_p, args.status)) { ok = false; break; }
              tc_fence_after();
            }
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(h * kWideHalf);
#pragma unroll
            for (int k = 0; k < BKW / 16; ++k) {
              mma_bf16_pair(d_tmem, wide_desc<BKW>(sa + k * 32),
                            wide_desc<BKW>(sb + h * BH_BYTES + k * 32), IDESC,
                            (kb > 0 || k > 0) ? 1u : 0u);
            }
            if (kb == nkb - 1) mma_commit_pair(tfull_bar(h), kBoth);
          }
          if (!ok) break;
          mma_commit_pair(empty_bar(stage), kBoth);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // wait for every MMA already issued before TMEM is released
        mma_commit_pair(drain_bar, 0x1);
        int dummy = 0;
        wait_bounded(drain_bar, 0, &dummy, nullptr);
      }
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 4 + EPI_WARPS) {
    // ------------------------------------------------------- epilogue -----
    const int q = warp & 3;             // TMEM lane quarter of this warp
    const int hc = (warp - 4) >> 2;     // which 128 columns of a half it drains
    const int r = q * 32 + lane;
    const uint32_t tempty_leader0 = map_to_cta(tempty_bar(0), 0);
    const uint32_t tempty_leader1 = map_to_cta(tempty_bar(1), 0);
    uint8_t* stage = smem + STAGES * STAGE_BYTES + (warp - 4) * kWarpStageBytes;
    int it = 0;
    bool ok = true;
    for (int tile = cluster; tile < total_tiles && ok; tile += nclusters, ++it) {
      const PairTile ti =
          decode_pair_tile(place_tile(tile, total_tiles, nclusters, n_long), tile_start, G, hs,
                           args.nt_routed, args.nt_shared, kWideChunk);
      const uint32_t tp = static_cast<uint32_t>(it & 1);
      const int my0 = ti.m_blk * PBM + static_cast<int>(rank) * HBM_ROWS;
      const int rows_valid = grp_rows[ti.g] - my0;
      const int64_t orow = static_cast<int64_t>(grp_row0[ti.g]) + my0 + r;
      const bool live = r < rows_valid;
      // routed rows of the plain epilogue may be remapped (token-slot order)
      const int64_t prow = (EPI == kEpiPlain && !ti.shared && args.row_map_r != nullptr && live)
                               ? static_cast<int64_t>(args.row_map_r[orow])
                               : orow;
      for (int h = 0; h < 2; ++h) {
        if (!wait_bounded(tfull_bar(h), tp, abort_p, args.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(h * kWideHalf + hc * 128);
        if (EPI == kEpiSwiGLU) {
          // these 128 accumulator columns are one packed block [gate 64 | up 64]
          bf16* out = static_cast<bf16*>(ti.shared ? args.out_s : args.out_r);
          const int64_t ld = ti.shared ? args.ld_s : args.ld_r;
          const int64_t col0 = static_cast<int64_t>(ti.n_blk) * (kWideBN / 2) + h * 128 + hc * 64;
          uint4 packed[8];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float gv[32], uv[32];
            tmem_ld32(taddr + hh * 32, gv);
            tmem_ld32(taddr + 64 + hh * 32, uv);
            tmem_ld_wait();
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float o[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) o[j] = silu_mul(gv[v * 8 + j], uv[v * 8 + j]);
              Vec16<bf16>::store(reinterpret_cast<bf16*>(&packed[hh * 4 + v]), o);
            }
          }
          // the half's accumulator is in registers: release it before the stores
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(h ? tempty_leader1 : tempty_leader0);
          uint8_t* dst = live ? reinterpret_cast<uint8_t*>(out + orow * ld + col0) : nullptr;
          warp_store_rows<128>(stage, packed, dst, lane);
        } else if (ti.shared) {
          // fp32 shared-expert output: 4 chunks of 32 columns (128 bytes a row)
          const int64_t colb = static_cast<int64_t>(ti.n_blk) * kWideBN + h * kWideHalf + hc * 128;
          float x[32];
          tmem_ld32(taddr, x);
          tmem_ld_wait_regs(x);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint4 packed[8];
#pragma unroll
            for (int v = 0; v < 8; ++v)
              packed[v] = make_uint4(__float_as_uint(x[4 * v]), __float_as_uint(x[4 * v + 1]),
                                     __float_as_uint(x[4 * v + 2]), __float_as_uint(x[4 * v + 3]));
            if (c + 1 < 4) tmem_ld32(taddr + (c + 1) * 32, x);
            uint8_t* dst = live ? reinterpret_cast<uint8_t*>(static_cast<float*>(args.out_s) +
                                                             orow * args.ld_s + colb + c * 32)
                                : nullptr;
            warp_store_rows<128>(stage, packed, dst, lane);
            if (c + 1 < 4) tmem_ld_wait_regs(x);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(h ? tempty_leader1 : tempty_leader0);
        } else {
          // bf16 routed output: 2 chunks of 64 columns (128 bytes a row),
          // both read from TMEM and packed first, so that the half is
          // released before the stores
          const int64_t colb = static_cast<int64_t>(ti.n_blk) * kWideBN + h * kWideHalf + hc * 128;
          uint4 packed[2][8];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            float x[64];
            tmem_ld32(taddr + c * 64, x);
            tmem_ld32(taddr + c * 64 + 32, x + 32);
            tmem_ld_wait_regs(x);
            tmem_ld_wait_regs(x + 32);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              Vec16<bf16>::store(reinterpret_cast<bf16*>(&packed[c][v]), x + v * 8);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(h ? tempty_leader1 : tempty_leader0);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint8_t* dst = live ? reinterpret_cast<uint8_t*>(static_cast<bf16*>(args.out_r) +
                                                             prow * args.ld_r + colb + c * 64)
                                : nullptr;
            warp_store_rows<128>(stage, packed[c], dst, lane);
          }
        }
      }
    }
  }

  tc_fence_before();
  cluster_sync_all();  // no CTA of the pair leaves while the other still works
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

template <int EPI>
int launch_wide_impl(const GemmMaps& m, const GroupedGemmArgs& args, int clusters,
                     cudaStream_t stream) {
  static std::atomic<uint64_t> optin{0};
  auto kern = grouped_gemm_pair_wide_kernel<EPI, kWideBK>;
  constexpr int smem = wide_smem_bytes<kWideBK>();
  if (int rc = ensure_smem_optin(reinterpret_cast<const void*>(kern), smem, optin)) return rc;
  return launch_k(kern, dim3(2 * clusters), kPairThreads, smem, stream, 2, m.a_r, m.a_s, m.b_r,
                  m.b_s, args);
}

template <int BN, int EPI>
int launch_pair_impl(const GemmMaps& m, const GroupedGemmArgs& args, int clusters,
                     cudaStream_t stream) {
  static std::atomic<uint64_t> optin{0};
  auto kern = grouped_gemm_pair_kernel<BN, EPI>;
  if (int rc = ensure_smem_optin(reinterpret_cast<const void*>(kern), pair_smem_bytes<BN, EPI>(),
                                 optin))
    return rc;
  return launch_k(kern, dim3(2 * clusters), kPairThreads, pair_smem_bytes<BN, EPI>(), stream, 2,
                  m.a_r, m.a_s, m.b_r, m.b_s, args);
}

}  // namespace

int launch_grouped_gemm_pair(int BN, int epi, const GemmMaps& maps, const GroupedGemmArgs& args,
                             int clusters, cudaStream_t stream) {
  if (clusters <= 0) return MOE_OK;
  if (BN == kWideBN)
    return epi == kEpiSwiGLU ? launch_wide_impl<kEpiSwiGLU>(maps, args, clusters, stream)
                             : launch_wide_impl<kEpiPlain>(maps, args, clusters, stream);
  if (epi == kEpiSwiGLU) {
    if (BN == 256) return launch_pair_impl<256, kEpiSwiGLU>(maps, args, clusters, stream);
    if (BN == 128) return launch_pair_impl<128, kEpiSwiGLU>(maps, args, clusters, stream);
  } else {
    if (BN == 256) return launch_pair_impl<256, kEpiPlain>(maps, args, clusters, stream);
    if (BN == 128) return launch_pair_impl<128, kEpiPlain>(maps, args, clusters, stream);
    if (BN == 64) return launch_pair_impl<64, kEpiPlain>(maps, args, clusters, stream);
  }
  return MOE_ERR_SHAPE;
}

}  // namespace sm100
}  // namespace moe
