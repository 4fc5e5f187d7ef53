// Host interface of the tcgen05 grouped expert GEMM (gemm_sm100.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {
namespace sm100 {

enum { kEpiSwiGLU = 0, kEpiPlain = 1 };

// One launch covers the shared-expert group (when shared_rows > 0) and the
// n_routed routed groups whose rows are offsets[e] .. offsets[e+1]-1.
struct GroupedGemmArgs {
  const int32_t* offsets;  // device, [n_routed + 1]
  int32_t n_routed;
  int32_t shared_rows;     // rows of the shared group (T) or 0
  int32_t kb_routed;       // 64-wide k-blocks of a routed tile
  int32_t kb_shared;       // 64-wide k-blocks of a shared tile
  int32_t kb_per_expert;   // B's third coordinate advances every kb_per_expert k-blocks
  int32_t nt_routed;       // BN-wide N tiles per routed group
  int32_t nt_shared;       // BN-wide N tiles of the shared group
  void* out_r;             // routed output (bf16), row stride ld_r elements
  int64_t ld_r;
  const int32_t* row_map_r;  // routed output row of position p: row_map_r[p] (NULL: p)
  void* out_s;             // shared output: bf16 (SwiGLU) or fp32 (plain)
  int64_t ld_s;
  int32_t* status;         // workspace status word
  // Rows in the A maps' box (single-CTA kernel; 0 means 128).  Smaller for
  // batches of fewer than 128 tokens, where no group has more rows: the
  // tile's other A rows are left as they are in shared memory and their
  // accumulator rows are never stored.
  int32_t a_rows;
  // Failure injection (MOE_FLAG_INJECT_WAIT_TIMEOUT): before its first load
  // the TMA producer waits, with a 1 ms limit, for a shared-memory slot that
  // nothing releases; the kernel then gives up like on any expired wait.
  int32_t inject_wait_timeout;
};

// Tile placement of the persistent GEMMs.  Worker w (a CTA, or a CTA pair)
// takes positions w, w + workers, ...; position v computes tile
// place_tile(v, ...).  Tiles are numbered with the shared-expert group first,
// and its n_long tiles may be longer (the down GEMM's K is K_s * I there).
// With three or more positions per worker the long tiles stay first (they
// start early).  With at most two, they go to the last positions of the
// workers that get one position fewer, so that no worker adds a long tile
// to a full share of short ones.
__device__ __forceinline__ int place_tile(int v, int total, int workers, int n_long) {
  const int q = total / workers, r = total - q * workers;
  if (n_long == 0 || q < 1 || q > 2 || n_long > workers - r) return v;
  const int p0 = (q - 1) * workers + r;  // first position of a short worker's last round
  if (v >= p0 && v < p0 + n_long) return v - p0;
  return v < p0 ? v + n_long : v;
}

// A maps: rank 2 {K, rows}; B maps: rank 3 {K, N rows, experts}; bf16, box
// {64, 128 (A) or BN (B)}, 128-byte swizzle.
struct GemmMaps {
  CUtensorMap a_r, a_s, b_r, b_s;
};

// box_k: 64 (128-byte rows, 128-byte swizzle) or 32 (64-byte rows, 64-byte
// swizzle).
bool make_map_bf16(CUtensorMap* map, int rank, const void* base, uint64_t inner, uint64_t rows,
                   uint64_t depth, uint64_t row_stride_bytes, uint64_t depth_stride_bytes,
                   uint32_t box_rows, uint32_t box_k = 64);

// Rank-2 map with 128-byte swizzle: box {box_inner, box_rows}; the box's
// inner extent must be 128 bytes.
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                 uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows);

int launch_grouped_gemm(int BN, int epi, const GemmMaps& maps, const GroupedGemmArgs& args,
                        int grid, cudaStream_t stream);

// The same GEMM on 2-CTA clusters with 256-row tiles (gemm_sm100_pair.cu).
// B maps must have box rows BN / 2 (128 for BN = 512, the wide tiles of
// 256 x 512 whose B rows come in two 128-row boxes per k-block).  The wide
// tiles step through K in blocks of kWideBK (maps with box_k = kWideBK; the
// args' k-block counts in those units): 64, three 48 KB stages.  32-wide
// k-blocks (64-byte swizzle, seven 24 KB stages) measured slower: 54.5%
// tensor-pipe against 72.6% on the 16B-shaped down GEMM.  `clusters` CTA
// pairs are launched.
constexpr int kWideBK = 64;
int launch_grouped_gemm_pair(int BN, int epi, const GemmMaps& maps, const GroupedGemmArgs& args,
                             int clusters, cudaStream_t stream);

}  // namespace sm100
}  // namespace moe
