/*
 * moe.h -- C ABI of libmoe: the DeepSeekMoE layer forward on NVIDIA B200
 * (sm_100a).
 *
 * The layer (from "DeepSeekMoE: Towards Ultimate Expert Specialization in
 * Mixture-of-Experts Language Models", §3.2 Shared Expert Isolation,
 * eqs. (9)-(11)):
 *
 *   h_t  = u_t + sum_{s < K_s} FFN_s(u_t) + sum_{k < K} g_{t,k} FFN_{idx[t,k]}(u_t)
 *   s_t  = Softmax_i(u_t^T e_i (+ b_i))   over the N_r routed experts
 *   idx  = the K largest s_{t,i} (lower expert index wins ties),
 *   g    = s at those experts, not renormalised
 *   FFN(x) = W2 (SiLU(W1 x) * (W3 x))    (SwiGLU, no biases)
 *
 * with N_r = mN - K_s fine-grained routed experts (§3.1) and K = mK - K_s.
 * Layer normalisation is not part of the layer (the pages omit it, §2).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers are DEVICE pointers owned by the caller unless a parameter says
 *   HOST.  The library never allocates device memory; scratch space comes
 *   from the caller's workspace `ws` (size from moe_workspace_size).
 * - All tensors are dense row-major.  Element types: `dtype` MOE_DTYPE_BF16
 *   means activations and weights are bfloat16 (raw 16-bit); MOE_DTYPE_F32
 *   means float32.  Router bias, gates and fp32 intermediates are float32;
 *   indices are int32.
 * - Base pointers must be 16-byte aligned (MOE_ERR_ALIGN otherwise).
 * - The bf16 path runs the expert GEMMs on tcgen05 tensor cores and needs
 *   d % 64 == 0 and inter % 64 == 0; the fp32 path runs them on CUDA cores.
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *   default stream) and never synchronises the host, except where stated.
 * - Return value: MOE_OK (0) or a negative MOE_ERR_* code.  Nothing is
 *   launched after a validation error.  MOE_ERR_CUDA reports a launch error.
 *   A kernel that gives up on a bounded wait records MOE_ERR_DEVICE_CHECK in
 *   the workspace's status word, read with moe_read_status.
 * - Results are bitwise reproducible from run to run (no atomics decide any
 *   value or order).
 * - Kernels are launched with programmatic dependent launch: one may start
 *   its set-up while the previous kernel on the stream finishes, but it reads
 *   and writes no global memory before that kernel has completed, so the
 *   usual stream order holds for the caller's own work too.
 * - moe_layer_forward only enqueues kernels on `stream` (no allocation, no
 *   host synchronisation), so a caller may capture it into a CUDA graph and
 *   replay it; replays give the eager result bit for bit.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* moe_stream_t; /* a cudaStream_t */

enum {
  MOE_DTYPE_F32 = 0,
  MOE_DTYPE_BF16 = 1,
};

enum {
  MOE_OK = 0,
  MOE_ERR_NULLPTR = -1,      /* a required pointer is NULL */
  MOE_ERR_SHAPE = -2,        /* sizes out of range or inconsistent */
  MOE_ERR_ALIGN = -3,        /* a pointer is not 16-byte aligned */
  MOE_ERR_WORKSPACE = -4,    /* workspace smaller than moe_workspace_size */
  MOE_ERR_DTYPE = -5,        /* unknown dtype */
  MOE_ERR_CUDA = -6,         /* CUDA runtime / launch error */
  MOE_ERR_DEVICE_CHECK = -7, /* a kernel gave up waiting (see moe_read_status) */
  MOE_ERR_UNSUPPORTED = -8,  /* no device of compute capability 10.0 */
  MOE_ERR_SCRATCH_LIMIT = -9, /* shape too large for moe_dispatch_static_scratch */
};

/* Router flags (moe_shape_t.flags). */
enum {
  /* The router bias b_i shifts only the top-K selection; the gates are the
     softmax of the unbiased logits (the per-expert load-balancing bias the
     csdn.net DeepSeekMoE article describes in words, §2.3).  Default (0):
     the bias is part of the logit for both selection and softmax. */
  MOE_FLAG_BIAS_SELECT_ONLY = 1,
  /* Tile shape of the bf16 expert GEMMs (default: chosen from the average
     rows per routed expert).  SINGLE_CTA: 128-row tiles, one SM each.
     CTA_PAIR: 256-row tiles computed by the two SMs of a 2-CTA cluster
     (tcgen05 cta_group::2).  Setting both is MOE_ERR_SHAPE.  Results are the
     same up to fp32 summation order inside the tensor cores. */
  MOE_FLAG_GEMM_SINGLE_CTA = 2,
  MOE_FLAG_GEMM_CTA_PAIR = 4,
  /* bf16 router on the CUDA cores: each logit is two fp32 FMA chains over
     the halves of d in increasing j, added once.  Default (0): the logits
     are one tcgen05 MMA tile per 128 tokens (bf16 products are exact in
     fp32; fp32 accumulation in the tensor cores' own order).  The two agree
     up to fp32 summation order.  The fp32 dtype always uses the CUDA
     cores. */
  MOE_FLAG_ROUTER_SIMT = 8,
  /* Failure injection, for tests of the error path: the TMA producer of each
     bf16 expert GEMM waits, before its first load, for a shared-memory slot
     that nothing releases.  That wait gives up after 1 ms like any bounded
     wait: the kernel records MOE_ERR_DEVICE_CHECK in the workspace status
     word, lets its in-flight work finish, frees its tensor memory and
     returns.  The call's outputs are then not valid; the context stays
     usable.  Never set in production. */
  MOE_FLAG_INJECT_WAIT_TIMEOUT = 16,
  /* CTA-pair tiles at most 256 columns wide.  Default (0): where every
     group's output width is a multiple of 512 (2*inter and 2*inter*n_shared
     for the gate/up GEMM, d for the down GEMM), a CTA pair computes
     256 x 512 tiles (two N = 256 MMAs per k-block, 48 rather than 64 bytes
     of operand tiles per clock of tensor work).  Same results up to fp32
     summation order inside the tensor cores. */
  MOE_FLAG_GEMM_NARROW = 32,
};

/* Layer shape.  Limits: 1 <= n_routed <= 256, 1 <= top_k <= min(n_routed, 32),
   0 <= n_shared <= 64, T >= 0 (T = 0 is a no-op), d >= 1, inter >= 1.  */
typedef struct {
  int64_t T;        /* tokens */
  int32_t d;        /* hidden size */
  int32_t n_routed; /* N_r = mN - K_s routed experts */
  int32_t n_shared; /* K_s shared experts */
  int32_t inter;    /* I, intermediate width of one fine-grained expert */
  int32_t top_k;    /* K = mK - K_s routed experts per token */
  int32_t dtype;    /* MOE_DTYPE_* */
  int32_t flags;    /* MOE_FLAG_* */
} moe_shape_t;

/* Human-readable name of a status code (static string). */
const char* moe_strerror(int status);

/* Bytes of workspace that moe_layer_forward, moe_dispatch and
   moe_expert_ffn need for `shape` (a multiple of 256). */
int moe_workspace_size(const moe_shape_t* shape, size_t* bytes);

/* W13 packing used by the tensor-core gate/up GEMM.
   W1, W3: [n_experts, inter, d]; W13 out: [n_experts, 2*inter, d] where, for
   every block b of 64 intermediate rows, packed rows 128b..128b+63 are W1
   rows 64b..64b+63 and packed rows 128b+64..128b+127 are W3 rows 64b..64b+63.
   (For dtype F32 the packed layout is the same.)  inter % 64 must be 0.
   Weight preparation, done once per model, not per forward. */
int moe_pack_w13(const moe_shape_t* shape, int32_t n_experts, const void* W1,
                 const void* W3, void* W13, moe_stream_t stream);

/* a1-a2, router (eqs. (10)-(11)): logits u_t.e_i (+ b_i) accumulated in fp32
   (tensor cores for bf16, see MOE_FLAG_ROUTER_SIMT), softmax over the
   n_routed experts, top-K.
   u: [T, d]; E: [n_routed, d]; bias: [n_routed] float32 or NULL.
   Outputs idx: [T, top_k] int32 in descending score order (ties: lower
   index first); w: [T, top_k] float32 gates (not renormalised). */
int moe_route(const moe_shape_t* shape, const void* u, const void* E,
              const float* bias, int32_t* idx, float* w, moe_stream_t stream);

/* a3, dispatch ("each token is computed only by its K experts", §2):
   counts[e] = #{(t,k): idx[t,k] = e}; offsets = exclusive scan (n_routed+1);
   perm[p] = slot t*top_k+k of position p, expert e's slots filling
   offsets[e]..offsets[e+1]-1 in increasing t; inv[t*top_k+k] = its position.
   idx must hold distinct experts per token in [0, n_routed).
   All outputs int32; bit-exact.  Uses workspace `ws`. */
int moe_dispatch(const moe_shape_t* shape, const int32_t* idx, int32_t* counts,
                 int32_t* offsets, int32_t* perm, int32_t* inv, void* ws,
                 size_t ws_bytes, moe_stream_t stream);

/* The same dispatch as moe_dispatch, same outputs bit for bit, for callers
   that cannot supply device memory per call: the paper has no counterpart;
   it is an interface for embedders.  Allocation may synchronise the device
   or fail once a caching pool holds the GPU's memory, so a latency-bound
   serving loop, or a host library without an allocator of its own, may not
   be able to provide `ws`.  This call allocates nothing: its scratch is one
   fixed array of MOE_DISPATCH_STATIC_SCRATCH_BYTES inside libmoe.
   Limit: 2 * round_up_256(ceil(T/128) * n_routed * 4) bytes must fit in
   that array (T <= 32768 at 256 routed experts, T <= 131072 at 64);
   larger shapes return MOE_ERR_SCRATCH_LIMIT before any launch.
   Set-up: the first call on each device (current device at the call)
   looks up the array's device address; make that first call before any
   stream capture begins on the device.  If that lookup fails the call
   returns MOE_ERR_CUDA and clears the calling thread's last CUDA error
   (cudaGetLastError), including an earlier one the caller had not read.
   Tracing (moe_profile_enable) brackets its kernels as MOE_KERNEL_DISPATCH.
   Sharing: every call in the process, on any stream, uses the same array.
   Calls whose kernels may overlap on a device race on it and corrupt each
   other's perm/inv/offsets; order them (one stream, or events).  Nothing in
   the array has to start at zero: each call writes every entry it reads. */
#define MOE_DISPATCH_STATIC_SCRATCH_BYTES (512u * 1024u)
int moe_dispatch_static_scratch(const moe_shape_t* shape, const int32_t* idx,
                                int32_t* counts, int32_t* offsets, int32_t* perm,
                                int32_t* inv, moe_stream_t stream);

/* a4-a6, expert FFNs: for every position p of expert e's segment,
   y[p] = FFN_e(u_{perm[p]/top_k}); and ysh[t] = sum_s FFN_s(u_t) over the
   shared experts (computed as one SwiGLU FFN of width n_shared*inter, the
   segmentation identity of §3.1).
   W13: [n_routed, 2*inter, d] packed by moe_pack_w13; W2: [n_routed, d, inter];
   W13_s: [n_shared, 2*inter, d] packed; W2_s: [n_shared, d, inter].
   y: [T*top_k, d] in dtype; ysh: [T, d] float32.  fp32 accumulation; for bf16
   the SwiGLU activation is rounded to bf16 before the down projection.
   perm/offsets as produced by moe_dispatch.  Uses workspace `ws`. */
int moe_expert_ffn(const moe_shape_t* shape, const void* u, const int32_t* perm,
                   const int32_t* offsets, const void* W13, const void* W2,
                   const void* W13_s, const void* W2_s, void* y, float* ysh,
                   void* ws, size_t ws_bytes, moe_stream_t stream);

/* a7, combine + residual (eq. (9)): h_t = u_t + ysh_t + sum_{k<K} w[t,k] *
   y[inv[t*K+k]], accumulated in fp32 in exactly that order, rounded once to
   dtype.  h: [T, d] dtype. */
int moe_combine(const moe_shape_t* shape, const void* u, const float* ysh,
                const void* y, const float* w, const int32_t* inv, void* h,
                moe_stream_t stream);

/* The whole layer: route, dispatch, expert FFNs and combine, on `stream`,
   with every intermediate in `ws`.  Arguments as above; h: [T, d] dtype.
   Decode-sized batches (see moe_forward_path) run as one kernel that
   streams each activated expert's weights once in units of 64 intermediate
   rows, with fp32 partial down projections summed in a fixed order, and
   other batches of up to 128 tokens route, dispatch and gather in one
   kernel (each after a one-warp kernel that zeroes its grid-wide counters
   in ws); their h matches the oracle within the same bars but is not the
   stage-wise result bit for bit.  All other batches give exactly the result
   of moe_route, moe_dispatch, moe_expert_ffn and moe_combine. */
int moe_layer_forward(const moe_shape_t* shape, const void* u, const void* E,
                      const float* bias, const void* W13, const void* W2,
                      const void* W13_s, const void* W2_s, void* h, void* ws,
                      size_t ws_bytes, moe_stream_t stream);

/* moe_layer_forward with the activations in HOST memory: u_host [T, d] is
   copied to the device, the layer runs, and h is copied back into h_host;
   the call returns when h_host is written.  Page-locked host buffers make
   the copies asynchronous DMA.  Weights stay on the device.  Batches of at
   least 4352 tokens run in up to 4 chunks: the uploads and downloads go
   through two streams of the library's own, overlapping the forward of
   other chunks on `stream`, and start after the work already on `stream`.
   h equals moe_layer_forward's bit for bit.  Calls on one device run one
   at a time.  Workspace: moe_workspace_size plus 2*T*d*elem bytes. */
int moe_layer_forward_host(const moe_shape_t* shape, const void* u_host,
                           const void* E, const float* bias, const void* W13,
                           const void* W2, const void* W13_s, const void* W2_s,
                           void* h_host, void* ws, size_t ws_bytes,
                           moe_stream_t stream);

/* How moe_layer_forward runs `shape`:
   MOE_PATH_DECODE_LAYER: one kernel for the whole layer (bf16, 1 <= T <= 8,
     d in {256, 512, 1024, 2048}, inter % 64 == 0, and neither a GEMM tile
     shape nor failure injection forced in flags);
   MOE_PATH_SMALL_BATCH: router, dispatch and gather in one kernel with fp32
     CUDA-core logits, then the grouped GEMMs and the combine (other bf16
     batches of at most 128 tokens with d in {256, 512, 1024, 2048}, without
     MOE_FLAG_ROUTER_SIMT);
   MOE_PATH_STAGES: router, dispatch, grouped GEMMs, combine, each as
     moe_route / moe_dispatch / moe_expert_ffn / moe_combine compute them
     (h is their result bit for bit).
   The first two match the oracle within the same bars; their gates follow
   their own fp32 logits, so h is not the stage-wise result bit for bit. */
enum { MOE_PATH_STAGES = 0, MOE_PATH_DECODE_LAYER = 1, MOE_PATH_SMALL_BATCH = 2 };
int moe_forward_path(const moe_shape_t* shape, int32_t* path);

/* Bytes moe_layer_forward_host needs. */
int moe_workspace_size_host(const moe_shape_t* shape, size_t* bytes);

/* Expert load statistics of §3.3, eqs. (12)-(14), for the routing in idx
   and the scores of the router: f[e] = N'/(K'T) * counts[e] and P[e] =
   (1/T) sum_t s_{t,e}, with s recomputed from u, E, bias as in moe_route.
   f, P: [n_routed] float32.  (Training statistic; not on the forward path.)
   Uses workspace `ws`. */
int moe_expert_balance(const moe_shape_t* shape, const void* u, const void* E,
                       const float* bias, const int32_t* counts, float* f,
                       float* P, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Copies the workspace status word (0 or MOE_ERR_DEVICE_CHECK) to *status
   and clears it; synchronises `stream`. */
int moe_read_status(const void* ws, int32_t* status, moe_stream_t stream);

/* Tracing: device time of each stage.  While enabled, every kernel (the
   dispatch kernels count as one stage) that libmoe launches is
   bracketed by CUDA events recorded on its stream.  moe_profile_read waits
   for those events and returns, oldest first, the stage kind (MOE_KERNEL_*)
   and elapsed milliseconds of each bracketed launch since the last read:
   at most `max` entries are written and *count receives the number
   written; up to 4096 are kept, later ones are dropped.  `on`: 0 = off,
   1 = every stage, otherwise a mask of (1 << MOE_KERNEL_*) bits naming the
   stages to bracket (each bracket adds two event records to the stream, so
   a mask keeps the timing of the other stages undisturbed).  Tracing never
   changes any result. */
enum {
  MOE_KERNEL_ROUTER = 1,
  MOE_KERNEL_DISPATCH = 2,
  MOE_KERNEL_GATHER = 3,
  MOE_KERNEL_GEMM_GATE_UP = 4, /* grouped gate/up GEMM + SwiGLU (tcgen05) */
  MOE_KERNEL_GEMM_DOWN = 5,    /* grouped down GEMM (tcgen05) */
  MOE_KERNEL_COMBINE = 6,
  MOE_KERNEL_FFN_F32 = 7,      /* the fp32 expert FFN (both GEMMs) */
  MOE_KERNEL_MEMSET = 8,
  MOE_KERNEL_PACK = 9,
  MOE_KERNEL_BALANCE = 10,
  MOE_KERNEL_DECODE_LAYER = 11, /* the whole layer for decode-sized batches */
};
int moe_profile_enable(int on);
int moe_profile_read(int32_t* kinds, float* ms, int32_t max, int32_t* count);
const char* moe_kernel_name(int32_t kind);

/* Number of kernels this library has launched since load (all threads). */
uint64_t moe_launch_count(void);

/* Library version string. */
const char* moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
