// Dispatch, gather, combine, weight packing, the fp32 expert path and the
// balance-statistic reduction of the DeepSeekMoE layer.  All memory-bound
// kernels move 16-byte vectors; nothing here uses atomics, so every output
// is bitwise reproducible.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kDispThreads = kDispatchChunk;  // one thread per token
constexpr int kDispWarps = kDispThreads / 32;

// ---------------------------------------------------------------------------
// dispatch ("each token is computed only by its K experts", §2 after eq. (5))
//
// Tokens are cut into chunks of kDispatchChunk.  Pass 1 counts, per chunk
// and expert, the tokens that chose the expert (warp ballots, no atomics).
// The scan turns the counts into offsets and per-chunk bases.  Pass 2
// recomputes the ballots and ranks each (t, e) by the tokens before it, so
// the permutation lists every expert's tokens in increasing t.
// ---------------------------------------------------------------------------
template <int NW>
__device__ __forceinline__ void token_mask(const int32_t* __restrict__ idx, int64_t t, int64_t T,
                                           int K, uint32_t (&mask)[NW]) {
#pragma unroll
  for (int w = 0; w < NW; ++w) mask[w] = 0;
  if (t >= T) return;
  for (int k = 0; k < K; ++k) {
    const int e = idx[t * K + k];
#pragma unroll
    for (int w = 0; w < NW; ++w)
      if ((e >> 5) == w) mask[w] |= 1u << (e & 31);
  }
}

// wc[warp][e] = number of this warp's tokens that chose e
template <int NW>
__device__ __forceinline__ void warp_counts(const uint32_t (&mask)[NW], int n, int warp, int lane,
                                            int (*wc)[256]) {
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    for (int b = 0; b < 32; ++b) {
      const int e = w * 32 + b;
      if (e >= n) break;
      const unsigned bal = __ballot_sync(kFull, (mask[w] >> b) & 1u);
      if (lane == 0) wc[warp][e] = __popc(bal);
    }
  }
}

template <int NW>
__global__ void __launch_bounds__(kDispThreads)
dispatch_count_kernel(const int32_t* __restrict__ idx, int64_t T, int K, int n,
                      int32_t* __restrict__ chunk_counts) {
  __shared__ int wc[kDispWarps][256];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kDispThreads + threadIdx.x;
  uint32_t mask[NW];
  token_mask<NW>(idx, t, T, K, mask);
  warp_counts<NW>(mask, n, warp, lane, wc);
  __syncthreads();
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    int s = 0;
#pragma unroll 8
    for (int w = 0; w < kDispWarps; ++w) s += wc[w][e];
    chunk_counts[static_cast<int64_t>(blockIdx.x) * n + e] = s;
  }
}

__global__ void __launch_bounds__(256)
dispatch_scan_kernel(const int32_t* __restrict__ chunk_counts, int64_t nchunks, int n,
                     int32_t* __restrict__ chunk_base, int32_t* __restrict__ counts,
                     int32_t* __restrict__ offsets) {
  __shared__ int tot[256];
  pdl_wait();
  pdl_trigger();
  __shared__ int off[257];
  const int e = threadIdx.x;
  // pass 1: tokens per expert (loads batched so that 8 are in flight)
  int run = 0;
  if (e < n) {
    int64_t c = 0;
    for (; c + 8 <= nchunks; c += 8) {
      int v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = chunk_counts[(c + i) * n + e];
#pragma unroll
      for (int i = 0; i < 8; ++i) run += v[i];
    }
    for (; c < nchunks; ++c) run += chunk_counts[c * n + e];
    counts[e] = run;
  }
  tot[e] = e < n ? run : 0;
  __syncthreads();
  // exclusive scan over experts (Hillis-Steele on 256 entries)
  int x = tot[e];
  for (int o = 1; o < 256; o <<= 1) {
    __syncthreads();
    const int y = e >= o ? tot[e - o] : 0;
    __syncthreads();
    x += y;
    tot[e] = x;
  }
  __syncthreads();
  off[e + 1] = x;
  if (e == 0) off[0] = 0;
  __syncthreads();
  // pass 2: where each chunk's tokens of expert e start
  if (e < n) {
    int base = off[e];
    offsets[e] = base;
    int64_t c = 0;
    for (; c + 8 <= nchunks; c += 8) {
      int v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = chunk_counts[(c + i) * n + e];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        chunk_base[(c + i) * n + e] = base;
        base += v[i];
      }
    }
    for (; c < nchunks; ++c) {
      chunk_base[c * n + e] = base;
      base += chunk_counts[c * n + e];
    }
  }
  if (e == 0) offsets[n] = off[n];
}

template <int NW, int KMAX>
__global__ void __launch_bounds__(kDispThreads)
dispatch_scatter_kernel(const int32_t* __restrict__ idx, int64_t T, int K, int n,
                        const int32_t* __restrict__ chunk_base, int32_t* __restrict__ perm,
                        int32_t* __restrict__ inv) {
  __shared__ int wc[kDispWarps][256];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kDispThreads + threadIdx.x;
  // this token's experts, kept in registers
  int ek[KMAX];
#pragma unroll
  for (int k = 0; k < KMAX; ++k) ek[k] = (t < T && k < K) ? idx[t * K + k] : -1;
  uint32_t mask[NW];
#pragma unroll
  for (int w = 0; w < NW; ++w) mask[w] = 0;
#pragma unroll
  for (int k = 0; k < KMAX; ++k)
#pragma unroll
    for (int w = 0; w < NW; ++w)
      if (ek[k] >= 0 && (ek[k] >> 5) == w) mask[w] |= 1u << (ek[k] & 31);
  warp_counts<NW>(mask, n, warp, lane, wc);
  __syncthreads();
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    int run = chunk_base[static_cast<int64_t>(blockIdx.x) * n + e];
    for (int w = 0; w < kDispWarps; ++w) {
      const int c = wc[w][e];
      wc[w][e] = run;
      run += c;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    for (int b = 0; b < 32; ++b) {
      const int e = w * 32 + b;
      if (e >= n) break;
      const bool has = (mask[w] >> b) & 1u;
      const unsigned bal = __ballot_sync(kFull, has);
      if (has) {
        const int pos = wc[warp][e] + __popc(bal & lt);
        int kk = 0;
#pragma unroll
        for (int k = 0; k < KMAX; ++k)
          if (ek[k] == e) kk = k;
        const int64_t slot = t * K + kk;
        perm[pos] = static_cast<int32_t>(slot);
        inv[slot] = pos;
      }
    }
  }
}

// Scatter plus gather, for one chunk of kDispatchChunk tokens: the scatter
// above (warps 0-3, one thread per token), then every warp of the block copies
// the chunk's token rows of u to their K positions of xperm.  Each row of u is
// read once and written K times, where a separate gather would read it K
// times; the expert GEMMs then read xperm as before.
constexpr int kSgThreads = 512;
constexpr int kSgCopyUnroll = 8;  // 16-byte vectors a lane holds per row piece

template <int NW, int KMAX, typename TE>
__global__ void __launch_bounds__(kSgThreads)
dispatch_scatter_gather_kernel(const int32_t* __restrict__ idx, int64_t T, int K, int n,
                               const int32_t* __restrict__ chunk_base, int32_t* __restrict__ perm,
                               int32_t* __restrict__ inv, const TE* __restrict__ u, int d,
                               TE* __restrict__ xperm, int parts) {
  // `parts` blocks share a chunk: each ranks the chunk's tokens (cheap), the
  // first of them writes perm / inv, and each copies every parts-th row
  __shared__ int wc[kDispWarps][256];
  __shared__ int spos[kDispatchChunk][KMAX];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = static_cast<int>(blockIdx.x) / parts;
  const int part = static_cast<int>(blockIdx.x) - chunk * parts;
  const int64_t t0 = static_cast<int64_t>(chunk) * kDispatchChunk;
  const bool ranker = warp < kDispWarps;  // warp-uniform
  const int64_t t = t0 + threadIdx.x;
  int ek[KMAX];
  uint32_t mask[NW];
#pragma unroll
  for (int w = 0; w < NW; ++w) mask[w] = 0;
  if (ranker) {
#pragma unroll
    for (int k = 0; k < KMAX; ++k) ek[k] = (t < T && k < K) ? idx[t * K + k] : -1;
#pragma unroll
    for (int k = 0; k < KMAX; ++k)
#pragma unroll
      for (int w = 0; w < NW; ++w)
        if (ek[k] >= 0 && (ek[k] >> 5) == w) mask[w] |= 1u << (ek[k] & 31);
    warp_counts<NW>(mask, n, warp, lane, wc);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    int run = chunk_base[static_cast<int64_t>(chunk) * n + e];
    for (int w = 0; w < kDispWarps; ++w) {
      const int c = wc[w][e];
      wc[w][e] = run;
      run += c;
    }
  }
  __syncthreads();
  if (ranker) {
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      for (int b = 0; b < 32; ++b) {
        const int e = w * 32 + b;
        if (e >= n) break;
        const bool has = (mask[w] >> b) & 1u;
        const unsigned bal = __ballot_sync(kFull, has);
        if (has) {
          const int pos = wc[warp][e] + __popc(bal & lt);
          int kk = 0;
#pragma unroll
          for (int k = 0; k < KMAX; ++k)
            if (ek[k] == e) kk = k;
          const int64_t slot = t * K + kk;
          if (part == 0) {
            perm[pos] = static_cast<int32_t>(slot);
            inv[slot] = pos;
          }
          spos[threadIdx.x][kk] = pos;
        }
      }
    }
  }
  __syncthreads();
  // copy: warp w of part p takes the chunk's tokens p * 16 + w, + 16 * parts, ...
  constexpr int V = Vec16<TE>::N;
  constexpr int U = kSgCopyUnroll;
  constexpr int W = kSgThreads / 32;
  const int nv = d / V;
  const int64_t rem = T - t0;
  const int nt = rem < kDispatchChunk ? static_cast<int>(rem) : kDispatchChunk;
  for (int tl = part * W + warp; tl < nt; tl += W * parts) {
    const uint4* src = reinterpret_cast<const uint4*>(u + (t0 + tl) * static_cast<int64_t>(d));
    for (int c0 = lane; c0 < nv; c0 += 32 * U) {
      uint4 v[U];
#pragma unroll
      for (int j = 0; j < U; ++j)
        if (c0 + 32 * j < nv) v[j] = src[c0 + 32 * j];
      for (int kk = 0; kk < K; ++kk) {
        uint4* dst = reinterpret_cast<uint4*>(xperm + static_cast<int64_t>(spos[tl][kk]) * d);
#pragma unroll
        for (int j = 0; j < U; ++j)
          if (c0 + 32 * j < nv) dst[c0 + 32 * j] = v[j];
      }
    }
  }
}

// The whole dispatch in one block, for batches of at most kDispatchChunk
// tokens (decode): counts, the scan over experts and the scatter.  Each warp
// visits only the experts its own tokens chose (a handful at decode sizes).
template <int NW, int KMAX>
__global__ void __launch_bounds__(kDispThreads)
dispatch_single_kernel(const int32_t* __restrict__ idx, int64_t T, int K, int n,
                       int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                       int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  __shared__ int wc[kDispWarps][256];
  __shared__ int tot[256];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = threadIdx.x;
  for (int i = threadIdx.x; i < kDispWarps * 256; i += blockDim.x) (&wc[0][0])[i] = 0;
  int ek[KMAX];
#pragma unroll
  for (int k = 0; k < KMAX; ++k) ek[k] = (t < T && k < K) ? idx[t * K + k] : -1;
  uint32_t mask[NW], um[NW];
#pragma unroll
  for (int w = 0; w < NW; ++w) mask[w] = 0;
#pragma unroll
  for (int k = 0; k < KMAX; ++k)
#pragma unroll
    for (int w = 0; w < NW; ++w)
      if (ek[k] >= 0 && (ek[k] >> 5) == w) mask[w] |= 1u << (ek[k] & 31);
#pragma unroll
  for (int w = 0; w < NW; ++w) um[w] = __reduce_or_sync(kFull, mask[w]);
  __syncthreads();  // wc is zero
  // wc[warp][e] = this warp's tokens that chose e
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    for (uint32_t m = um[w]; m != 0; m &= m - 1) {
      const int b = __ffs(m) - 1;
      const unsigned bal = __ballot_sync(kFull, (mask[w] >> b) & 1u);
      if (lane == 0) wc[warp][w * 32 + b] = __popc(bal);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 256; e += blockDim.x) {
    int c = 0;
    if (e < n)
      for (int w = 0; w < kDispWarps; ++w) c += wc[w][e];
    tot[e] = c;
    if (e < n) counts[e] = c;
  }
  __syncthreads();
  // exclusive scan over the experts: one warp, eight entries a lane
  if (warp == 0) {
    int v[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = tot[lane * 8 + i];
      sum += v[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      tot[e] = run;
      if (e < n) offsets[e] = run;
      run += v[i];
    }
    if (lane == 31) offsets[n] = incl;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    int run = tot[e];
    for (int w = 0; w < kDispWarps; ++w) {
      const int c = wc[w][e];
      wc[w][e] = run;
      run += c;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    for (uint32_t m = um[w]; m != 0; m &= m - 1) {
      const int b = __ffs(m) - 1;
      const int e = w * 32 + b;
      const bool has = (mask[w] >> b) & 1u;
      const unsigned bal = __ballot_sync(kFull, has);
      if (has) {
        const int pos = wc[warp][e] + __popc(bal & lt);
        int kk = 0;
#pragma unroll
        for (int k = 0; k < KMAX; ++k)
          if (ek[k] == e) kk = k;
        const int64_t slot = t * K + kk;
        perm[pos] = static_cast<int32_t>(slot);
        inv[slot] = pos;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// gather: xperm[p] = u[perm[p] / K]  (the rows each expert multiplies)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256)
gather_rows_kernel(const T* __restrict__ u, const int32_t* __restrict__ perm, int64_t rows, int d,
                   int K, T* __restrict__ xperm) {
  constexpr int V = Vec16<T>::N;
  pdl_wait();
  pdl_trigger();
  constexpr int U = 4;  // 16-byte loads in flight per lane before the stores
  const int lane = threadIdx.x & 31;
  const int nv = d / V;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t p = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       p < rows; p += warps) {
    const int64_t t = perm[p] / K;
    const uint4* src = reinterpret_cast<const uint4*>(u + t * d);
    uint4* dst = reinterpret_cast<uint4*>(xperm + p * d);
    for (int c0 = lane; c0 < nv; c0 += 32 * U) {
      uint4 v[U];
#pragma unroll
      for (int k = 0; k < U; ++k)
        if (c0 + 32 * k < nv) v[k] = src[c0 + 32 * k];
#pragma unroll
      for (int k = 0; k < U; ++k)
        if (c0 + 32 * k < nv) dst[c0 + 32 * k] = v[k];
    }
  }
}

// ---------------------------------------------------------------------------
// combine (eq. (9)): h_t = u_t + ysh_t + sum_k w[t,k] * y[inv[t*K+k]], in
// fp32, in exactly this order (one fused multiply-add per k), rounded once.
// One warp per token; the K expert rows of a column block are loaded in
// batches of kCombineBatch before any of them is used, so their DRAM
// latencies overlap instead of forming a chain.
// ---------------------------------------------------------------------------
constexpr int kCombineBatch = 4;

template <typename T>
__global__ void __launch_bounds__(256, 4)
combine_kernel(const T* __restrict__ u, const float* __restrict__ ysh, const T* __restrict__ y,
               const float* __restrict__ w, const int32_t* __restrict__ inv, int64_t Tn, int d,
               int K, T* __restrict__ h) {
  // one warp per (token, block of 32*V columns)
  pdl_wait();
  pdl_trigger();
  constexpr int V = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int nblk = (d + 32 * V - 1) / (32 * V);
  const int64_t units = Tn * nblk;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t wu = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       wu < units; wu += warps) {
    const int64_t t = wu / nblk;
    const int c = static_cast<int>(wu - t * nblk) * 32 * V + lane * V;
    const bool live = c < d;
    // lane k < K holds row inv[t*K+k] (or the token-slot row t*K+k) and
    // gate w[t*K+k]; shuffles hand them to every lane
    const int my_row = lane < K ? (inv ? inv[t * K + lane] : static_cast<int>(t * K + lane)) : 0;
    const float my_w = lane < K ? w[t * K + lane] : 0.0f;
    float acc[V], tmp[V];
    if (live) {
      Vec16<T>::load(u + t * d + c, acc);
#pragma unroll
      for (int i = 0; i < V; i += 4) {
        Vec16<float>::load(ysh + t * d + c + i, tmp);
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i + j] += tmp[j];
      }
    }
    for (int k0 = 0; k0 < K; k0 += kCombineBatch) {
      uint4 raw[kCombineBatch];
      float wk[kCombineBatch];
#pragma unroll
      for (int kk = 0; kk < kCombineBatch; ++kk) {
        const int k = k0 + kk;
        const int64_t r = __shfl_sync(kFull, my_row, k & 31);
        wk[kk] = __shfl_sync(kFull, my_w, k & 31);
        if (live && k < K) raw[kk] = *reinterpret_cast<const uint4*>(y + r * d + c);
      }
#pragma unroll
      for (int kk = 0; kk < kCombineBatch; ++kk) {
        if (live && k0 + kk < K) {
          Vec16<T>::load(reinterpret_cast<const T*>(&raw[kk]), tmp);
#pragma unroll
          for (int j = 0; j < V; ++j) acc[j] = fmaf(wk[kk], tmp[j], acc[j]);
        }
      }
    }
    if (live) Vec16<T>::store(h + t * d + c, acc);
  }
}

// ---------------------------------------------------------------------------
// W13 packing: packed row 128b + j = W1 row 64b + j (j < 64), W3 row 64b + j - 64
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256)
pack_w13_kernel(const T* __restrict__ W1, const T* __restrict__ W3, T* __restrict__ W13,
                int64_t total_rows, int I, int d) {
  constexpr int V = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t pr = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       pr < total_rows; pr += warps) {
    const int64_t e = pr / (2 * I);
    const int r = static_cast<int>(pr - e * 2 * I);
    const int blk = r >> 7, j = r & 127;
    const T* src = (j < 64 ? W1 : W3) + (e * I + blk * 64 + (j & 63)) * static_cast<int64_t>(d);
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(W13 + pr * d);
    for (int c = lane; c < d / V; c += 32) d4[c] = s4[c];
  }
}

// ---------------------------------------------------------------------------
// fp32 expert FFN on CUDA cores (the float32 layer; correctness path).
// D = A * B^T over 64-row tiles; B(n, k) lives at
// B + (zbase + k / kpe) * zstride + n * ldb + k % kpe.
// ---------------------------------------------------------------------------
struct F32Gemm {
  const float* A_r;
  const float* A_s;
  int64_t lda_r, lda_s;
  const float* B_r;
  const float* B_s;
  int64_t ldb, zstride_r, zstride_s;
  int kpe;
  int k_r, k_s;       // reduction length of routed / shared tiles
  int nb_r, nb_s;     // B rows per routed expert / of the shared group
  float* out_r;
  float* out_s;
  int64_t ldo_r, ldo_s;
  const int32_t* offsets;
  int n_routed;
  int64_t shared_rows;
};

template <int SWIGLU>
__global__ void __launch_bounds__(256)
ffn_f32_gemm_kernel(F32Gemm p) {
  constexpr int BMr = 64, BKc = 16;
  constexpr int BNr = SWIGLU ? 128 : 64;  // B rows per tile
  __shared__ float As[BKc][BMr];
  __shared__ float Bs[BKc][BNr];
  __shared__ int s_start[258];
  __shared__ int s_g;

  const int tid = threadIdx.x;
  const int hs = p.shared_rows > 0 ? 1 : 0;
  const int G = p.n_routed + hs;
  // m-tile prefix over groups (shared group first)
  if (tid == 0) {
    int acc = 0;
    for (int g = 0; g < G; ++g) {
      s_start[g] = acc;
      const int64_t rows = (hs && g == 0) ? p.shared_rows
                                          : (p.offsets[g - hs + 1] - p.offsets[g - hs]);
      acc += static_cast<int>((rows + BMr - 1) / BMr);
    }
    s_start[G] = acc;
    int g = -1;
    for (int i = 0; i < G; ++i)
      if (s_start[i] <= static_cast<int>(blockIdx.x) && static_cast<int>(blockIdx.x) < s_start[i + 1]) g = i;
    s_g = g;
  }
  __syncthreads();
  const int g = s_g;
  if (g < 0) return;
  const bool shared = hs && g == 0;
  const int e = g - hs;
  const int64_t grow0 = shared ? 0 : p.offsets[e];
  const int64_t grows = shared ? p.shared_rows : p.offsets[e + 1] - p.offsets[e];
  const int m0 = (blockIdx.x - s_start[g]) * BMr;
  const int n0 = blockIdx.y * BNr;
  if (n0 >= (shared ? p.nb_s : p.nb_r)) return;
  const float* A = shared ? p.A_s : p.A_r;
  const int64_t lda = shared ? p.lda_s : p.lda_r;
  const float* B = shared ? p.B_s : p.B_r;
  const int64_t zstride = shared ? p.zstride_s : p.zstride_r;
  const int zbase = shared ? 0 : e;
  const int Kd = shared ? p.k_s : p.k_r;

  // thread (ty, tx): rows ty*4..+3; columns tx*4..+3 (and +64 for SwiGLU up)
  const int ty = tid / 16, tx = tid % 16;
  float acc[4][SWIGLU ? 8 : 4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < (SWIGLU ? 8 : 4); ++j) acc[i][j] = 0.0f;

  for (int k0 = 0; k0 < Kd; k0 += BKc) {
    for (int i = tid; i < BKc * BMr; i += 256) {
      const int r = i / BKc, kk = i % BKc;
      const int64_t row = grow0 + m0 + r;
      As[kk][r] = (m0 + r < grows && k0 + kk < Kd) ? A[row * lda + k0 + kk] : 0.0f;
    }
    for (int i = tid; i < BKc * BNr; i += 256) {
      const int r = i / BKc, kk = i % BKc;
      const int k = k0 + kk;
      Bs[kk][r] = k < Kd ? B[static_cast<int64_t>(zbase + k / p.kpe) * zstride +
                             static_cast<int64_t>(n0 + r) * p.ldb + (k % p.kpe)]
                         : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BKc; ++kk) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float a = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a, Bs[kk][tx * 4 + j], acc[i][j]);
          if (SWIGLU) acc[i][4 + j] = fmaf(a, Bs[kk][64 + tx * 4 + j], acc[i][4 + j]);
        }
      }
    }
    __syncthreads();
  }
  float* out = shared ? p.out_s : p.out_r;
  const int64_t ldo = shared ? p.ldo_s : p.ldo_r;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = m0 + ty * 4 + i;
    if (r >= grows) continue;
    const int64_t orow = grow0 + r;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (SWIGLU) {
        const float gt = acc[i][j], up = acc[i][4 + j];
        out[orow * ldo + (n0 / 2) + tx * 4 + j] = gt / (1.0f + expf(-gt)) * up;
      } else {
        out[orow * ldo + n0 + tx * 4 + j] = acc[i][j];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// balance statistics, §3.3 eqs. (12)-(13)
// ---------------------------------------------------------------------------
__global__ void balance_reduce_kernel(const float* __restrict__ pstat, int nblocks,
                                      const int32_t* __restrict__ counts, int64_t T, int n, int K,
                                      float* __restrict__ f, float* __restrict__ P) {
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int b = 0; b < nblocks; ++b) s += pstat[static_cast<int64_t>(b) * n + e];
    P[e] = s / static_cast<float>(T);
    f[e] = static_cast<float>(counts[e]) * (static_cast<float>(n) /
                                            (static_cast<float>(K) * static_cast<float>(T)));
  }
}

inline unsigned grid_for_rows(int64_t rows, int rows_per_block) {
  const int64_t b = (rows + rows_per_block - 1) / rows_per_block;
  return static_cast<unsigned>(b < 148 * 32 ? (b < 1 ? 1 : b) : 148 * 32);
}

}  // namespace

int launch_dispatch(const int32_t* idx, int64_t T, int K, int n, int32_t* chunk_counts,
                    int32_t* chunk_base, int32_t* counts, int32_t* offsets, int32_t* perm,
                    int32_t* inv, cudaStream_t st, bool counts_ready, const DispatchGather* dg,
                    bool* gathered) {
  if (gathered) *gathered = false;
  const int64_t nch = dispatch_num_chunks(T);
  const int nw = (n + 31) / 32;
  if (T == 0) {
    // no tokens: counts and offsets are all zero
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * n, st) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (n + 1), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (nch == 1) {
    // one block does it all
#define MOE_SINGLE_CASE(W)                                                                   \
  case W:                                                                                    \
    return K <= 8    ? launch_k(dispatch_single_kernel<W, 8>, 1, kDispThreads, 0, st, 1, idx, T, K, \
                                n, counts, offsets, perm, inv)                               \
           : K <= 16 ? launch_k(dispatch_single_kernel<W, 16>, 1, kDispThreads, 0, st, 1, idx, T,  \
                                K, n, counts, offsets, perm, inv)                            \
                     : launch_k(dispatch_single_kernel<W, 32>, 1, kDispThreads, 0, st, 1, idx, T,  \
                                K, n, counts, offsets, perm, inv);
    switch (nw) {
      MOE_SINGLE_CASE(1) MOE_SINGLE_CASE(2) MOE_SINGLE_CASE(3) MOE_SINGLE_CASE(4)
      MOE_SINGLE_CASE(5) MOE_SINGLE_CASE(6) MOE_SINGLE_CASE(7) MOE_SINGLE_CASE(8)
      default: return MOE_ERR_SHAPE;
    }
#undef MOE_SINGLE_CASE
  }
  const dim3 grid(static_cast<unsigned>(nch));
  int rc = MOE_ERR_SHAPE;
#define MOE_DISPATCH_CASE(W)                                                                 \
  case W:                                                                                    \
    rc = launch_k(dispatch_count_kernel<W>, grid, kDispThreads, 0, st, 1, idx, T, K, n,      \
                  chunk_counts);                                                             \
    break;
  if (counts_ready) {
    rc = MOE_OK;
  } else {
    switch (nw) {
      MOE_DISPATCH_CASE(1) MOE_DISPATCH_CASE(2) MOE_DISPATCH_CASE(3) MOE_DISPATCH_CASE(4)
      MOE_DISPATCH_CASE(5) MOE_DISPATCH_CASE(6) MOE_DISPATCH_CASE(7) MOE_DISPATCH_CASE(8)
      default: return MOE_ERR_SHAPE;
    }
  }
#undef MOE_DISPATCH_CASE
  if (rc) return rc;
  if (int r2 = launch_k(dispatch_scan_kernel, 1, 256, 0, st, 1, static_cast<const int32_t*>(chunk_counts),
                        nch, n, chunk_base, counts, offsets))
    return r2;
  if (dg && dg->xperm) {
    // scatter and gather in one launch; enough blocks share each chunk's
    // copies that the grid covers every SM about twice
    const int bf = dg->dtype == MOE_DTYPE_BF16;
    const int64_t want = (2 * 148 + nch - 1) / nch;
    const int parts = static_cast<int>(want < 1 ? 1 : (want > 8 ? 8 : want));
    const dim3 sg_grid(static_cast<unsigned>(nch * parts));
    rc = MOE_ERR_SHAPE;
#define MOE_SG_LAUNCH(W, KM, TE)                                                             \
  launch_k(dispatch_scatter_gather_kernel<W, KM, TE>, sg_grid, kSgThreads, 0, st, 1, idx, T, K, \
           n, static_cast<const int32_t*>(chunk_base), perm, inv, static_cast<const TE*>(dg->u), \
           dg->d, static_cast<TE*>(dg->xperm), parts)
#define MOE_SG_CASE(W)                                                                       \
  case W:                                                                                    \
    rc = bf ? (K <= 8 ? MOE_SG_LAUNCH(W, 8, bf16)                                            \
                      : K <= 16 ? MOE_SG_LAUNCH(W, 16, bf16) : MOE_SG_LAUNCH(W, 32, bf16))   \
            : (K <= 8 ? MOE_SG_LAUNCH(W, 8, float)                                           \
                      : K <= 16 ? MOE_SG_LAUNCH(W, 16, float) : MOE_SG_LAUNCH(W, 32, float)); \
    break;
    switch (nw) {
      MOE_SG_CASE(1) MOE_SG_CASE(2) MOE_SG_CASE(3) MOE_SG_CASE(4)
      MOE_SG_CASE(5) MOE_SG_CASE(6) MOE_SG_CASE(7) MOE_SG_CASE(8)
      default: return MOE_ERR_SHAPE;
    }
#undef MOE_SG_CASE
#undef MOE_SG_LAUNCH
    if (rc == MOE_OK && gathered) *gathered = true;
    return rc;
  }
  rc = MOE_ERR_SHAPE;
#define MOE_SCATTER_CASE(W)                                                                  \
  case W:                                                                                    \
    rc = K <= 8    ? launch_k(dispatch_scatter_kernel<W, 8>, grid, kDispThreads, 0, st, 1, idx, T, \
                              K, n, static_cast<const int32_t*>(chunk_base), perm, inv)      \
         : K <= 16 ? launch_k(dispatch_scatter_kernel<W, 16>, grid, kDispThreads, 0, st, 1, idx,   \
                              T, K, n, static_cast<const int32_t*>(chunk_base), perm, inv)   \
                   : launch_k(dispatch_scatter_kernel<W, 32>, grid, kDispThreads, 0, st, 1, idx,   \
                              T, K, n, static_cast<const int32_t*>(chunk_base), perm, inv);  \
    break;
  switch (nw) {
    MOE_SCATTER_CASE(1) MOE_SCATTER_CASE(2) MOE_SCATTER_CASE(3) MOE_SCATTER_CASE(4)
    MOE_SCATTER_CASE(5) MOE_SCATTER_CASE(6) MOE_SCATTER_CASE(7) MOE_SCATTER_CASE(8)
    default: return MOE_ERR_SHAPE;
  }
#undef MOE_SCATTER_CASE
  return rc;
}

__global__ void zero_words_kernel(int32_t* p, int n) {
  pdl_wait();     // the kernel before may still count on these words
  pdl_trigger();  // the next kernel's set-up may overlap the writes below
  for (int i = threadIdx.x; i < n; i += blockDim.x) p[i] = 0;
}

int launch_zero_words(int32_t* p, int n, cudaStream_t st) {
  return launch_k(zero_words_kernel, 1, 32, 0, st, 1, p, n);
}

int launch_gather(int dtype, const void* u, const int32_t* perm, int64_t rows, int d, int K,
                  void* xperm, cudaStream_t st) {
  if (rows == 0) return MOE_OK;
  const unsigned grid = grid_for_rows(rows, 8);
  if (dtype == MOE_DTYPE_BF16)
    return launch_k(gather_rows_kernel<bf16>, grid, 256, 0, st, 1, static_cast<const bf16*>(u),
                    perm, rows, d, K, static_cast<bf16*>(xperm));
  return launch_k(gather_rows_kernel<float>, grid, 256, 0, st, 1, static_cast<const float*>(u),
                  perm, rows, d, K, static_cast<float*>(xperm));
}

int launch_combine(int dtype, const void* u, const float* ysh, const void* y, const float* w,
                   const int32_t* inv, int64_t T, int d, int K, void* h, cudaStream_t st) {
  if (T == 0) return MOE_OK;
  const int V = dtype == MOE_DTYPE_BF16 ? 8 : 4;
  const unsigned grid = grid_for_rows(T * ((d + 32 * V - 1) / (32 * V)), 8);
  if (dtype == MOE_DTYPE_BF16)
    return launch_k(combine_kernel<bf16>, grid, 256, 0, st, 1, static_cast<const bf16*>(u), ysh,
                    static_cast<const bf16*>(y), w, inv, T, d, K, static_cast<bf16*>(h));
  return launch_k(combine_kernel<float>, grid, 256, 0, st, 1, static_cast<const float*>(u), ysh,
                  static_cast<const float*>(y), w, inv, T, d, K, static_cast<float*>(h));
}

int launch_pack_w13(int dtype, const void* W1, const void* W3, void* W13, int n_experts, int I,
                    int d, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(n_experts) * 2 * I;
  if (rows == 0) return MOE_OK;
  const unsigned grid = grid_for_rows(rows, 8);
  if (dtype == MOE_DTYPE_BF16)
    pack_w13_kernel<bf16><<<grid, 256, 0, st>>>(static_cast<const bf16*>(W1),
                                                static_cast<const bf16*>(W3),
                                                static_cast<bf16*>(W13), rows, I, d);
  else
    pack_w13_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(W1),
                                                 static_cast<const float*>(W3),
                                                 static_cast<float*>(W13), rows, I, d);
  count_launch();
  return check_launch();
}

int launch_ffn_f32(const float* xperm, const float* u, const int32_t* offsets, int n_routed,
                   int64_t T, int n_shared, int d, int I, const float* W13, const float* W2,
                   const float* W13_s, const float* W2_s, float* act, float* act_s, float* y,
                   float* ysh, int max_routed_mtiles, cudaStream_t st) {
  const int64_t shared_rows = n_shared > 0 ? T : 0;
  const int sh_tiles = static_cast<int>((shared_rows + 63) / 64);
  const unsigned gx = static_cast<unsigned>(max_routed_mtiles + sh_tiles);
  if (gx == 0) return MOE_OK;
  // gate/up: A = xperm | u, B = W13 [n, 2I, d] | W13_s as [K_s*2I, d]
  F32Gemm p{};
  p.A_r = xperm; p.A_s = u; p.lda_r = d; p.lda_s = d;
  p.B_r = W13; p.B_s = W13_s; p.ldb = d;
  p.zstride_r = static_cast<int64_t>(2) * I * d; p.zstride_s = 0;
  p.kpe = d; p.k_r = d; p.k_s = d;
  p.nb_r = 2 * I; p.nb_s = 2 * I * n_shared;
  p.out_r = act; p.out_s = act_s; p.ldo_r = I; p.ldo_s = static_cast<int64_t>(I) * n_shared;
  p.offsets = offsets; p.n_routed = n_routed; p.shared_rows = shared_rows;
  const int nbmax = p.nb_s > p.nb_r ? p.nb_s : p.nb_r;
  ffn_f32_gemm_kernel<1><<<dim3(gx, (nbmax + 127) / 128), 256, 0, st>>>(p);
  count_launch();
  if (int rc = check_launch()) return rc;
  // down: A = act | act_s, B = W2 [n, d, I] | W2_s [K_s, d, I] (K spans experts)
  F32Gemm q{};
  q.A_r = act; q.A_s = act_s; q.lda_r = I; q.lda_s = static_cast<int64_t>(I) * n_shared;
  q.B_r = W2; q.B_s = W2_s; q.ldb = I;
  q.zstride_r = static_cast<int64_t>(d) * I; q.zstride_s = static_cast<int64_t>(d) * I;
  q.kpe = I; q.k_r = I; q.k_s = I * n_shared;
  q.nb_r = d; q.nb_s = d;
  q.out_r = y; q.out_s = ysh; q.ldo_r = d; q.ldo_s = d;
  q.offsets = offsets; q.n_routed = n_routed; q.shared_rows = shared_rows;
  ffn_f32_gemm_kernel<0><<<dim3(gx, (d + 63) / 64), 256, 0, st>>>(q);
  count_launch();
  return check_launch();
}

int launch_balance_reduce(const float* pstat, int nblocks, const int32_t* counts, int64_t T,
                          int n, int K, float* f, float* P, cudaStream_t st) {
  balance_reduce_kernel<<<1, 256, 0, st>>>(pstat, nblocks, counts, T, n, K, f, P);
  count_launch();
  return check_launch();
}

int launch_zero(void* p, size_t bytes, cudaStream_t st) {
  return cudaMemsetAsync(p, 0, bytes, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
