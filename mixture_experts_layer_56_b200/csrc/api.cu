// C ABI of libmoe (include/moe.h): validation, workspace carving and the
// launch sequence of the DeepSeekMoE layer forward on the caller's stream.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "decode_fused.h"
#include "gemm_sm100.h"
#include "kernels.h"

namespace moe {

static std::atomic<uint64_t> g_launches{0};

void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

int check_launch() { return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// ---------------------------------------------------------------------------
// tracing: CUDA events around each stage, on the stage's stream
// ---------------------------------------------------------------------------
namespace {
struct ProfRec {
  int32_t kind;
  cudaEvent_t beg, end;
};
struct Profiler {
  std::mutex mu;
  std::atomic<bool> on{false};
  std::atomic<uint32_t> mask{~0u};  // bit k: bracket stages of kind k
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};
Profiler& prof() {
  static Profiler p;
  return p;
}
constexpr size_t kMaxProfRecs = 4096;

// Records `e` on `st`; inside a stream capture as an event node of the graph
// (a plain record there is only a dependency within the capture), so that
// every replay records it.
void record_event(cudaEvent_t e, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
  else
    cudaEventRecord(e, st);
}

}  // namespace

// RAII bracket: records the start event now and the end event when it goes
// out of scope (after the stage's launches were enqueued).
StageScope::StageScope(int32_t kind, cudaStream_t st) : st_(st) {
  Profiler& p = prof();
  if (!p.on.load() || kind < 0 || kind > 31 || !((p.mask.load() >> kind) & 1u)) return;
  std::lock_guard<std::mutex> lock(p.mu);
  if (p.recs.size() >= kMaxProfRecs) return;
  ProfRec r{kind, p.get(), p.get()};
  if (!r.beg || !r.end) return;
  record_event(r.beg, st_);
  p.recs.push_back(r);
  idx_ = static_cast<long>(p.recs.size()) - 1;
}

StageScope::~StageScope() {
  if (idx_ < 0) return;
  Profiler& p = prof();
  std::lock_guard<std::mutex> lock(p.mu);
  record_event(p.recs[static_cast<size_t>(idx_)].end, st_);
}

namespace {
using Stage = StageScope;
}  // namespace

namespace {

constexpr size_t kAlign = 256;
inline size_t round_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

struct Layout {
  size_t status, idx, w, counts, offsets, perm, inv, chunk_counts, chunk_base, pstat;
  size_t xperm, act, act_s, y, ysh;
  size_t dec_logits, dec_part, dec_sync;  // the decode kernel's (empty unless eligible)
  size_t total;
  size_t u_host, h_host, total_host;  // extra staging for moe_layer_forward_host
};

size_t elem_bytes(int dtype) { return dtype == MOE_DTYPE_BF16 ? 2 : 4; }

Layout layout_of(const moe_shape_t& s) {
  const size_t T = static_cast<size_t>(s.T), K = s.top_k, n = s.n_routed, d = s.d,
               I = s.inter, ns = s.n_shared, el = elem_bytes(s.dtype);
  const size_t nch = static_cast<size_t>(dispatch_num_chunks(s.T));
  const size_t nrc = static_cast<size_t>(router_num_ctas(s.T));
  Layout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += round_up(bytes);
    return at;
  };
  L.status = take(kAlign);
  L.idx = take(T * K * 4);
  L.w = take(T * K * 4);
  L.counts = take(n * 4);
  L.offsets = take((n + 1) * 4);
  L.perm = take(T * K * 4);
  L.inv = take(T * K * 4);
  L.chunk_counts = take(nch * n * 4);
  L.chunk_base = take(nch * n * 4);
  L.pstat = take(nrc * n * 4);
  L.xperm = take(T * K * d * el);
  L.act = take(T * K * I * el);
  L.act_s = take(T * ns * I * el);
  L.y = take(T * K * d * el);
  L.ysh = take(T * d * 4);
  const bool dec = decode_fused_eligible(s);
  const bool front = !dec && decode_front_eligible(s);
  L.dec_logits = take(dec || front ? T * n * 4 : 0);
  L.dec_part = take(dec ? decode_partial_rows(s) * d * 4 : 0);
  L.dec_sync = take(dec || front ? kAlign : 0);
  L.total = o;
  L.u_host = take(T * d * el);
  L.h_host = take(T * d * el);
  L.total_host = o;
  return L;
}

int validate(const moe_shape_t* s) {
  if (!s) return MOE_ERR_NULLPTR;
  if (s->dtype != MOE_DTYPE_F32 && s->dtype != MOE_DTYPE_BF16) return MOE_ERR_DTYPE;
  if (s->T < 0 || s->d < 1 || s->n_routed < 1 || s->n_routed > 256 || s->top_k < 1 ||
      s->top_k > s->n_routed || s->top_k > 32 || s->n_shared < 0 || s->n_shared > 64 ||
      s->inter < 1)
    return MOE_ERR_SHAPE;
  const int32_t known = MOE_FLAG_BIAS_SELECT_ONLY | MOE_FLAG_GEMM_SINGLE_CTA |
                        MOE_FLAG_GEMM_CTA_PAIR | MOE_FLAG_ROUTER_SIMT |
                        MOE_FLAG_INJECT_WAIT_TIMEOUT | MOE_FLAG_GEMM_NARROW;
  if ((s->flags & ~known) != 0) return MOE_ERR_SHAPE;
  if ((s->flags & MOE_FLAG_GEMM_SINGLE_CTA) && (s->flags & MOE_FLAG_GEMM_CTA_PAIR))
    return MOE_ERR_SHAPE;
  // positions are int32; rows address TMA coordinates (int32)
  if (s->T * static_cast<int64_t>(s->top_k) > 0x7fffffffLL) return MOE_ERR_SHAPE;
  if (s->inter % 64 != 0) return MOE_ERR_SHAPE;
  if (s->dtype == MOE_DTYPE_BF16) {
    if (s->d % 64 != 0) return MOE_ERR_SHAPE;
  } else {
    if (s->d % 4 != 0) return MOE_ERR_SHAPE;
  }
  return MOE_OK;
}

inline bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

struct DeviceInfo {
  int ok = -1;  // -1 unknown, 0 unsupported, 1 sm_100
  int sms = 0;
};

int device_info(DeviceInfo* out) {
  static DeviceInfo cache[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  DeviceInfo& di = cache[dev];
  if (di.ok < 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    di.ok = (major == 10 && minor == 0) ? 1 : 0;
    di.sms = sms;
  }
  *out = di;
  return di.ok == 1 ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// expert FFNs on workspace-resident gathered rows
// y_slot_order: write routed expert outputs at row perm[p] (token slot
// t*K+k) instead of row p, so that the combine reads each token's rows
// contiguously.
int run_expert_ffn(const moe_shape_t& s, const Layout& L, const void* u, const int32_t* perm,
                   const int32_t* offsets, const void* W13, const void* W2, const void* W13_s,
                   const void* W2_s, void* y, float* ysh, void* ws, cudaStream_t st, int sms,
                   bool y_slot_order, bool rows_gathered = false) {
  const int64_t T = s.T, K = s.top_k, rows = T * K;
  const int d = s.d, I = s.inter, n = s.n_routed, ns = s.n_shared;
  void* xperm = at<void>(ws, L.xperm);
  void* act = at<void>(ws, L.act);
  void* act_s = at<void>(ws, L.act_s);
  if (!rows_gathered) {
    // expert-sorted copies of the routed token rows
    Stage sg(MOE_KERNEL_GATHER, st);
    if (int rc = launch_gather(s.dtype, u, perm, rows, d, static_cast<int>(K), xperm, st))
      return rc;
  }
  if (ns == 0) {
    // no shared experts: ysh = 0
    Stage sg(MOE_KERNEL_MEMSET, st);
    if (int rc = launch_zero(ysh, static_cast<size_t>(T) * d * 4, st)) return rc;
  }

  if (s.dtype == MOE_DTYPE_F32) {
    const int max_mt = static_cast<int>((rows + 63) / 64 + (rows < n ? rows : n));
    Stage sg(MOE_KERNEL_FFN_F32, st);
    return launch_ffn_f32(static_cast<const float*>(xperm), static_cast<const float*>(u), offsets,
                          n, T, ns, d, I, static_cast<const float*>(W13),
                          static_cast<const float*>(W2), static_cast<const float*>(W13_s),
                          static_cast<const float*>(W2_s), static_cast<float*>(act),
                          static_cast<float*>(act_s), static_cast<float*>(y), ysh, max_mt, st);
  }

  using namespace sm100;
  const uint64_t d64 = static_cast<uint64_t>(d), I64 = static_cast<uint64_t>(I);
  int32_t* status = at<int32_t>(ws, L.status);
  // 256-row tiles on CTA pairs once experts average at least half such a
  // tile; 128-row tiles on single SMs otherwise (decode-sized batches)
  bool pair = rows >= static_cast<int64_t>(n) * 128;
  if (s.flags & MOE_FLAG_GEMM_SINGLE_CTA) pair = false;
  if (s.flags & MOE_FLAG_GEMM_CTA_PAIR) pair = true;
  const int BM = pair ? 256 : 128;
  // rows of an A box: below 128 tokens no group has more than T rows
  const uint32_t a_rows = pair || T >= 128 ? 128u : static_cast<uint32_t>((T + 7) / 8 * 8);
  const int64_t routed_mt_ub = (rows + BM - 1) / BM + (rows < n ? rows : n);
  const int64_t shared_mt = ns > 0 ? (T + BM - 1) / BM : 0;
  auto launch = [&](int BN, int epi, const GemmMaps& m, const GroupedGemmArgs& a) {
    const int64_t tiles = routed_mt_ub * a.nt_routed + shared_mt * a.nt_shared;
    if (pair) {
      const int64_t cl = tiles < sms / 2 ? tiles : sms / 2;
      return launch_grouped_gemm_pair(BN, epi, m, a, static_cast<int>(cl), st);
    }
    const int64_t grid = tiles < sms ? tiles : sms;
    return launch_grouped_gemm(BN, epi, m, a, static_cast<int>(grid), st);
  };

  // the widest tile whose tile count still covers every SM (single-CTA
  // tiles only: decode-sized batches need the extra parallelism)
  auto pick_bn = [&](int n_cols_r, int n_cols_s, int widest, int narrowest) {
    int bn = widest;
    while (!pair && bn > narrowest && (n_cols_r % bn == 0) &&
           routed_mt_ub * (n_cols_r / bn) + shared_mt * (n_cols_s / bn) < sms)
      bn /= 2;
    return bn;
  };

  // CTA pairs take 512-column tiles where both groups' widths allow them
  const bool narrow = (s.flags & MOE_FLAG_GEMM_NARROW) != 0;
  auto wide_ok = [&](int64_t n_cols_r, int64_t n_cols_s) {
    return pair && !narrow && n_cols_r % 512 == 0 && (ns == 0 || n_cols_s % 512 == 0);
  };
  auto b_box = [&](int BN) { return static_cast<uint32_t>(BN == 512 ? 128 : (pair ? BN / 2 : BN)); };

  // ---- gate/up + SwiGLU ---------------------------------------------------
  {
    const int BN = wide_ok(2 * I64, 2 * I64 * ns)
                       ? 512
                       : pick_bn(2 * I, 2 * I * ns, (2 * I) % 256 == 0 ? 256 : 128, 128);
    const uint32_t bbox = b_box(BN);
    const int bk = BN == 512 ? kWideBK : 64;  // K per k-block
    const uint32_t bk32 = static_cast<uint32_t>(bk);
    GemmMaps m;
    bool ok = make_map_bf16(&m.a_r, 2, xperm, d64, rows, 1, d64 * 2, 0, a_rows, bk32) &&
              make_map_bf16(&m.b_r, 3, W13, d64, 2 * I64, n, d64 * 2, 2 * I64 * d64 * 2, bbox,
                            bk32);
    if (ns > 0) {
      ok = ok && make_map_bf16(&m.a_s, 2, u, d64, T, 1, d64 * 2, 0, a_rows, bk32) &&
           make_map_bf16(&m.b_s, 3, W13_s, d64, 2 * I64 * ns, 1, d64 * 2, 2 * I64 * ns * d64 * 2,
                         bbox, bk32);
    } else {
      m.a_s = m.a_r;
      m.b_s = m.b_r;
    }
    if (!ok) return MOE_ERR_CUDA;
    GroupedGemmArgs a{};
    a.offsets = offsets;
    a.n_routed = n;
    a.shared_rows = ns > 0 ? static_cast<int32_t>(T) : 0;
    a.kb_routed = d / bk;
    a.kb_shared = d / bk;
    a.kb_per_expert = d / bk;
    a.nt_routed = 2 * I / BN;
    a.nt_shared = 2 * I * ns / BN;
    a.out_r = act;
    a.ld_r = I;
    a.out_s = act_s;
    a.ld_s = static_cast<int64_t>(I) * ns;
    a.status = status;
    a.a_rows = static_cast<int32_t>(a_rows);
    a.inject_wait_timeout = (s.flags & MOE_FLAG_INJECT_WAIT_TIMEOUT) ? 1 : 0;
    Stage sg(MOE_KERNEL_GEMM_GATE_UP, st);
    if (int rc = launch(BN, kEpiSwiGLU, m, a)) return rc;
  }
  // ---- down projection ----------------------------------------------------
  {
    const int BN = wide_ok(d64, d64)
                       ? 512
                       : pick_bn(d, d, d % 256 == 0 ? 256 : (d % 128 == 0 ? 128 : 64), 64);
    const uint32_t bbox = b_box(BN);
    const int bk = BN == 512 ? kWideBK : 64;  // K per k-block
    const uint32_t bk32 = static_cast<uint32_t>(bk);
    GemmMaps m;
    bool ok = make_map_bf16(&m.a_r, 2, act, I64, rows, 1, I64 * 2, 0, a_rows, bk32) &&
              make_map_bf16(&m.b_r, 3, W2, I64, d64, n, I64 * 2, d64 * I64 * 2, bbox, bk32);
    if (ns > 0) {
      ok = ok && make_map_bf16(&m.a_s, 2, act_s, I64 * ns, T, 1, I64 * ns * 2, 0, a_rows, bk32) &&
           make_map_bf16(&m.b_s, 3, W2_s, I64, d64, ns, I64 * 2, d64 * I64 * 2, bbox, bk32);
    } else {
      m.a_s = m.a_r;
      m.b_s = m.b_r;
    }
    if (!ok) return MOE_ERR_CUDA;
    GroupedGemmArgs a{};
    a.offsets = offsets;
    a.n_routed = n;
    a.shared_rows = ns > 0 ? static_cast<int32_t>(T) : 0;
    a.kb_routed = I / bk;
    a.kb_shared = I * ns / bk;
    a.kb_per_expert = I / bk;
    a.nt_routed = d / BN;
    a.nt_shared = d / BN;
    a.out_r = y;
    a.ld_r = d;
    a.row_map_r = y_slot_order ? perm : nullptr;
    a.out_s = ysh;
    a.ld_s = d;
    a.status = status;
    a.a_rows = static_cast<int32_t>(a_rows);
    a.inject_wait_timeout = (s.flags & MOE_FLAG_INJECT_WAIT_TIMEOUT) ? 1 : 0;
    Stage sg(MOE_KERNEL_GEMM_DOWN, st);
    if (int rc = launch(BN, kEpiPlain, m, a)) return rc;
  }
  return MOE_OK;
}

int forward_device(const moe_shape_t& s, const Layout& L, const void* u, const void* E,
                   const float* bias, const void* W13, const void* W2, const void* W13_s,
                   const void* W2_s, void* h, void* ws, cudaStream_t st, int sms) {
  if (decode_fused_eligible(s)) {
    // a handful of tokens: the whole layer in one kernel
    Stage sg(MOE_KERNEL_DECODE_LAYER, st);
    return launch_decode_fused(s, u, E, bias, W13, W2, W13_s, W2_s, h, at<int32_t>(ws, L.idx),
                               at<float>(ws, L.w), at<float>(ws, L.dec_logits),
                               at<float>(ws, L.dec_part), at<void>(ws, L.dec_sync),
                               at<int32_t>(ws, L.status), sms, st);
  }
  const int64_t T = s.T;
  const int K = s.top_k, n = s.n_routed;
  int32_t* idx = at<int32_t>(ws, L.idx);
  float* w = at<float>(ws, L.w);
  int32_t* counts = at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv = at<int32_t>(ws, L.inv);
  void* y = at<void>(ws, L.y);
  float* ysh = at<float>(ws, L.ysh);
  if (decode_front_eligible(s)) {
    // a small batch: router, dispatch and gather in one launch, then the
    // grouped GEMMs and the combine as below
    {
      Stage sg(MOE_KERNEL_ROUTER, st);
      if (int rc = launch_decode_front(s, u, E, bias, idx, w, at<float>(ws, L.dec_logits), counts,
                                       offsets, perm, inv, at<void>(ws, L.xperm),
                                       at<void>(ws, L.dec_sync), at<int32_t>(ws, L.status), sms,
                                       st))
        return rc;
    }
    if (int rc = run_expert_ffn(s, L, u, perm, offsets, W13, W2, W13_s, W2_s, y, ysh, ws, st, sms,
                                /*y_slot_order=*/true, /*rows_gathered=*/true))
      return rc;
    Stage sg(MOE_KERNEL_COMBINE, st);
    return launch_combine(s.dtype, u, ysh, y, w, nullptr, T, s.d, K, h, st);
  }
  // batches of more than one dispatch chunk: the router also counts
  int32_t* chunk_counts = at<int32_t>(ws, L.chunk_counts);
  bool counted = false;
  {
    Stage sg(MOE_KERNEL_ROUTER, st);
    if (int rc = launch_router(s.dtype, u, E, bias, T, s.d, n, K, s.flags, idx, w, nullptr,
                               at<int32_t>(ws, L.status), st,
                               T > kDispatchChunk ? chunk_counts : nullptr, &counted))
      return rc;
  }
  // the dispatch of batches above one chunk also gathers the routed rows
  const DispatchGather dg{s.dtype, u, s.d, at<void>(ws, L.xperm)};
  bool gathered = false;
  {
    Stage sg(MOE_KERNEL_DISPATCH, st);
    if (int rc = launch_dispatch(idx, T, K, n, chunk_counts, at<int32_t>(ws, L.chunk_base), counts,
                                 offsets, perm, inv, st, counted, &dg, &gathered))
      return rc;
  }
  // the tensor-core path writes y in token-slot order (the combine then
  // reads each token's rows contiguously); the fp32 path keeps expert order
  const bool slot_order = s.dtype == MOE_DTYPE_BF16;
  if (int rc = run_expert_ffn(s, L, u, perm, offsets, W13, W2, W13_s, W2_s, y, ysh, ws, st, sms,
                              slot_order, gathered))
    return rc;
  Stage sg(MOE_KERNEL_COMBINE, st);
  return launch_combine(s.dtype, u, ysh, y, w, slot_order ? nullptr : inv, T, s.d, K, h, st);
}

bool shared_ptrs_ok(const moe_shape_t& s, const void* W13_s, const void* W2_s) {
  return s.n_shared == 0 || (W13_s && W2_s);
}

// Chunks of moe_layer_forward_host: each above kMinHostChunk tokens, where the
// router runs one CTA per 128-token tile with no cluster split, up to 4.
constexpr int64_t kMinHostChunk = 2176;
int host_chunks(int64_t T) {
  const int64_t n = T / kMinHostChunk;
  return static_cast<int>(n < 1 ? 1 : (n > 4 ? 4 : n));
}

// Per device: an upload and a download stream and the events that order
// them against the caller's stream (created once; no device memory).
struct HostPipe {
  cudaStream_t s_in = nullptr, s_out = nullptr;
  std::vector<cudaEvent_t> ev;  // [0] start, [1..n] uploads, [n+1..2n] forwards
  std::mutex busy;              // one host-buffer call at a time per device
};
int host_pipe(int nc, HostPipe** out) {
  static HostPipe pipes[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  HostPipe& hp = pipes[dev];
  if (!hp.s_in &&
      (cudaStreamCreateWithFlags(&hp.s_in, cudaStreamNonBlocking) != cudaSuccess ||
       cudaStreamCreateWithFlags(&hp.s_out, cudaStreamNonBlocking) != cudaSuccess))
    return MOE_ERR_CUDA;
  while (hp.ev.size() < static_cast<size_t>(1 + 2 * nc)) {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return MOE_ERR_CUDA;
    hp.ev.push_back(e);
  }
  *out = &hp;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_strerror(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_NULLPTR: return "null pointer";
    case MOE_ERR_SHAPE: return "invalid shape";
    case MOE_ERR_ALIGN: return "pointer not 16-byte aligned";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_DTYPE: return "invalid dtype";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_CHECK: return "a kernel gave up waiting (device check)";
    case MOE_ERR_UNSUPPORTED: return "device is not sm_100 (B200)";
    case MOE_ERR_SCRATCH_LIMIT: return "shape exceeds the fixed dispatch scratch";
    default: return "unknown status";
  }
}

const char* moe_version(void) { return "moe-b200 0.1.0 (sm_100a)"; }

uint64_t moe_launch_count(void) { return g_launches.load(); }

int moe_profile_enable(int on) {
  prof().mask.store(on == 1 ? ~0u : static_cast<uint32_t>(on));
  prof().on.store(on != 0);
  return MOE_OK;
}

int moe_profile_read(int32_t* kinds, float* ms, int32_t max, int32_t* count) {
  if (!count || (max > 0 && (!kinds || !ms))) return MOE_ERR_NULLPTR;
  Profiler& p = prof();
  std::lock_guard<std::mutex> lock(p.mu);
  int32_t n = 0;
  int rc = MOE_OK;
  for (const ProfRec& r : p.recs) {
    if (n < max) {
      float t = 0.0f;
      if (cudaEventSynchronize(r.end) != cudaSuccess ||
          cudaEventElapsedTime(&t, r.beg, r.end) != cudaSuccess) {
        rc = MOE_ERR_CUDA;
        cudaGetLastError();  // a failed query must not surface in a later launch check
      }
      kinds[n] = r.kind;
      ms[n] = t;
      ++n;
    }
    p.pool.push_back(r.beg);
    p.pool.push_back(r.end);
  }
  p.recs.clear();
  *count = n;
  return rc;
}

const char* moe_kernel_name(int32_t kind) {
  switch (kind) {
    case MOE_KERNEL_ROUTER: return "router_topk";
    case MOE_KERNEL_DISPATCH: return "dispatch";
    case MOE_KERNEL_GATHER: return "gather_rows";
    case MOE_KERNEL_GEMM_GATE_UP: return "grouped_gemm_gate_up_swiglu";
    case MOE_KERNEL_GEMM_DOWN: return "grouped_gemm_down";
    case MOE_KERNEL_COMBINE: return "combine_residual";
    case MOE_KERNEL_FFN_F32: return "ffn_f32";
    case MOE_KERNEL_MEMSET: return "memset";
    case MOE_KERNEL_PACK: return "pack_w13";
    case MOE_KERNEL_BALANCE: return "expert_balance";
    case MOE_KERNEL_DECODE_LAYER: return "decode_layer";
    default: return "unknown";
  }
}

int moe_workspace_size(const moe_shape_t* shape, size_t* bytes) {
  if (!bytes) return MOE_ERR_NULLPTR;
  if (int rc = validate(shape)) return rc;
  *bytes = layout_of(*shape).total;
  return MOE_OK;
}

int moe_forward_path(const moe_shape_t* shape, int32_t* path) {
  if (!path) return MOE_ERR_NULLPTR;
  if (int rc = validate(shape)) return rc;
  *path = decode_fused_eligible(*shape)   ? MOE_PATH_DECODE_LAYER
          : decode_front_eligible(*shape) ? MOE_PATH_SMALL_BATCH
                                          : MOE_PATH_STAGES;
  return MOE_OK;
}

int moe_workspace_size_host(const moe_shape_t* shape, size_t* bytes) {
  if (!bytes) return MOE_ERR_NULLPTR;
  if (int rc = validate(shape)) return rc;
  *bytes = layout_of(*shape).total_host;
  return MOE_OK;
}

int moe_pack_w13(const moe_shape_t* shape, int32_t n_experts, const void* W1, const void* W3,
                 void* W13, moe_stream_t stream) {
  if (int rc = validate(shape)) return rc;
  if (n_experts < 0) return MOE_ERR_SHAPE;
  if (n_experts == 0) return MOE_OK;
  if (!W1 || !W3 || !W13) return MOE_ERR_NULLPTR;
  if (misaligned(W1) || misaligned(W3) || misaligned(W13)) return MOE_ERR_ALIGN;
  DeviceInfo di;
  if (int rc = device_info(&di)) return rc;
  Stage sg(MOE_KERNEL_PACK, static_cast<cudaStream_t>(stream));
  return launch_pack_w13(shape->dtype, W1, W3, W13, n_experts, shape->inter, shape->d,
                         static_cast<cudaStream_t>(stream));
}

int moe_route(const moe_shape_t* shape, const void* u, const void* E, const float* bias,
              int32_t* idx, float* w, moe_stream_t stream) {
  if (int rc = validate(shape)) return rc;
  if (shape->T == 0) return MOE_OK;
  if (!u || !E || !idx || !w) return MOE_ERR_NULLPTR;
  if (misaligned(u) || misaligned(E) || misaligned(idx) || misaligned(w) ||
      (bias && misaligned(bias)))
    return MOE_ERR_ALIGN;
  DeviceInfo di;
  if (int rc = device_info(&di)) return rc;
  Stage sg(MOE_KERNEL_ROUTER, static_cast<cudaStream_t>(stream));
  return launch_router(shape->dtype, u, E, bias, shape->T, shape->d, shape->n_routed,
                       shape->top_k, shape->flags, idx, w, nullptr, nullptr,
                       static_cast<cudaStream_t>(stream));
}

int moe_dispatch(const moe_shape_t* shape, const int32_t* idx, int32_t* counts, int32_t* offsets,
                 int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (int rc = validate(shape)) return rc;
  if (!counts || !offsets || !ws) return MOE_ERR_NULLPTR;
  if (shape->T > 0 && (!idx || !perm || !inv)) return MOE_ERR_NULLPTR;
  if (misaligned(counts) || misaligned(offsets) || misaligned(ws) ||
      (shape->T > 0 && (misaligned(idx) || misaligned(perm) || misaligned(inv))))
    return MOE_ERR_ALIGN;
  const Layout L = layout_of(*shape);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  DeviceInfo di;
  if (int rc = device_info(&di)) return rc;
  Stage sg(MOE_KERNEL_DISPATCH, static_cast<cudaStream_t>(stream));
  return launch_dispatch(idx, shape->T, shape->top_k, shape->n_routed,
                         at<int32_t>(ws, L.chunk_counts), at<int32_t>(ws, L.chunk_base), counts,
                         offsets, perm, inv, static_cast<cudaStream_t>(stream));
}

int moe_expert_ffn(const moe_shape_t* shape, const void* u, const int32_t* perm,
                   const int32_t* offsets, const void* W13, const void* W2, const void* W13_s,
                   const void* W2_s, void* y, float* ysh, void* ws, size_t ws_bytes,
                   moe_stream_t stream) {
  if (int rc = validate(shape)) return rc;
  if (shape->T == 0) return MOE_OK;
  if (!u || !perm || !offsets || !W13 || !W2 || !y || !ysh || !ws) return MOE_ERR_NULLPTR;
  if (!shared_ptrs_ok(*shape, W13_s, W2_s)) return MOE_ERR_NULLPTR;
  if (misaligned(u) || misaligned(perm) || misaligned(offsets) || misaligned(W13) ||
      misaligned(W2) || misaligned(y) || misaligned(ysh) || misaligned(ws) ||
      (W13_s && misaligned(W13_s)) || (W2_s && misaligned(W2_s)))
    return MOE_ERR_ALIGN;
  const Layout L = layout_of(*shape);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  DeviceInfo di;
  if (int rc = device_info(&di)) return rc;
  return run_expert_ffn(*shape, L, u, perm, offsets, W13, W2, W13_s, W2_s, y, ysh, ws,
                        static_cast<cudaStream_t>(stream), di.sms, /*y_slot_order=*/false);
}

int moe_combine(const moe_shape_t* shape, const void* u, const float* ysh, const void* y,
                const float* w, const int32_t* inv, void* h, moe_stream_t stream) {
  if (int rc = validate(shape)) return rc;
  if (shape->T == 0) return MOE_OK;
  if (!u || !ysh || !y || !w || !inv || !h) return MOE_ERR_NULLPTR;
  if (misaligned(u) || misaligned(ysh) || misaligned(y) || misaligned(w) || misaligned(inv) ||
      misaligned(h))
    return MOE_ERR_ALIGN;
  DeviceInfo di;
  if (int rc = device_info(&di)) return rc;
  Stage sg(MOE_KERNEL_COMBINE, static_cast<cudaStream_t>(stream));
  return launch_combine(shape->dtype, u, ysh, y, w, inv, shape->T, shape->d, shape->top_k, h,
                        static_cast<cudaStream_t>(stream));
}

int moe_layer_forward(const moe_shape_t* shape, const void* u, const void* E, const float* bias,
                      const void* W13, const void* W2, const void* W13_s, const void* W2_s,
                      void* h, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (int rc = validate(shape)) return rc;
  if (shape->T == 0) return MOE_OK;
  if (!u || !E || !W13 || !W2 || !h || !ws) return MOE_ERR_NULLPTR;
  if (!shared_ptrs_ok(*shape, W13_s, W2_s)) return MOE_ERR_NULLPTR;
  if (misaligned(u) || misaligned(E) || misaligned(W13) || misaligned(W2) || misaligned(h) ||
      misaligned(ws) || (bias && misaligned(bias)) || (W13_s && misaligned(W13_s)) ||
      (W2_s && misaligned(W2_s)))
    return MOE_ERR_ALIGN;
  const Layout L = layout_of(*shape);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  DeviceInfo di;
  if (int rc = device_info(&di)) return rc;
  return forward_device(*shape, L, u, E, bias, W13, W2, W13_s, W2_s, h, ws,
                        static_cast<cudaStream_t>(stream), di.sms);
}

int moe_layer_forward_host(const moe_shape_t* shape, const void* u_host, const void* E,
                           const float* bias, const void* W13, const void* W2, const void* W13_s,
                           const void* W2_s, void* h_host, void* ws, size_t ws_bytes,
                           moe_stream_t stream) {
  if (int rc = validate(shape)) return rc;
  if (shape->T == 0) return MOE_OK;
  if (!u_host || !E || !W13 || !W2 || !h_host || !ws) return MOE_ERR_NULLPTR;
  if (!shared_ptrs_ok(*shape, W13_s, W2_s)) return MOE_ERR_NULLPTR;
  if (misaligned(E) || misaligned(W13) || misaligned(W2) || misaligned(ws) ||
      (bias && misaligned(bias)) || (W13_s && misaligned(W13_s)) || (W2_s && misaligned(W2_s)))
    return MOE_ERR_ALIGN;
  const Layout L = layout_of(*shape);
  if (ws_bytes < L.total_host) return MOE_ERR_WORKSPACE;
  DeviceInfo di;
  if (int rc = device_info(&di)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t row_bytes = static_cast<size_t>(shape->d) * elem_bytes(shape->dtype);
  const size_t bytes = static_cast<size_t>(shape->T) * row_bytes;
  uint8_t* u_dev = at<uint8_t>(ws, L.u_host);
  uint8_t* h_dev = at<uint8_t>(ws, L.h_host);
  const int nc = host_chunks(shape->T);
  if (nc == 1) {
    if (cudaMemcpyAsync(u_dev, u_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (int rc = forward_device(*shape, L, u_dev, E, bias, W13, W2, W13_s, W2_s, h_dev, ws, st,
                                di.sms))
      return rc;
    if (cudaMemcpyAsync(h_host, h_dev, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return cudaStreamSynchronize(st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  // Chunks of tokens: chunk i's upload and chunk i-1's download overlap the
  // forward of the chunk between them.  Tokens are independent and every
  // chunk runs with the whole batch's GEMM tile mode (and above the router's
  // cluster-split size), so h is the one-pass result bit for bit.
  HostPipe* hp = nullptr;
  if (int rc = host_pipe(nc, &hp)) return rc;
  std::lock_guard<std::mutex> busy(hp->busy);
  // on an error, nothing may still copy from or to the caller's buffers
  auto fail = [&](int rc) {
    cudaStreamSynchronize(hp->s_in);
    cudaStreamSynchronize(st);
    cudaStreamSynchronize(hp->s_out);
    return rc;
  };
  moe_shape_t sc = *shape;
  if (!(sc.flags & (MOE_FLAG_GEMM_SINGLE_CTA | MOE_FLAG_GEMM_CTA_PAIR))) {
    const bool pair = shape->T * shape->top_k >= static_cast<int64_t>(shape->n_routed) * 128;
    sc.flags |= pair ? MOE_FLAG_GEMM_CTA_PAIR : MOE_FLAG_GEMM_SINGLE_CTA;
  }
  // the copies start after the caller's earlier work on `stream`
  if (cudaEventRecord(hp->ev[0], st) != cudaSuccess ||
      cudaStreamWaitEvent(hp->s_in, hp->ev[0], 0) != cudaSuccess)
    return fail(MOE_ERR_CUDA);
  auto chunk = [&](int i, int64_t* t0, int64_t* tn) {
    *t0 = shape->T * i / nc;
    *tn = shape->T * (i + 1) / nc - *t0;
  };
  for (int i = 0; i < nc; ++i) {
    int64_t t0, tn;
    chunk(i, &t0, &tn);
    if (cudaMemcpyAsync(u_dev + t0 * row_bytes, static_cast<const uint8_t*>(u_host) + t0 * row_bytes,
                        tn * row_bytes, cudaMemcpyHostToDevice, hp->s_in) != cudaSuccess ||
        cudaEventRecord(hp->ev[1 + i], hp->s_in) != cudaSuccess)
      return fail(MOE_ERR_CUDA);
  }
  for (int i = 0; i < nc; ++i) {
    int64_t t0, tn;
    chunk(i, &t0, &tn);
    sc.T = tn;
    const Layout Lc = layout_of(sc);  // intermediates of one chunk (below L's staging)
    if (cudaStreamWaitEvent(st, hp->ev[1 + i], 0) != cudaSuccess) return fail(MOE_ERR_CUDA);
    if (int rc = forward_device(sc, Lc, u_dev + t0 * row_bytes, E, bias, W13, W2, W13_s, W2_s,
                                h_dev + t0 * row_bytes, ws, st, di.sms))
      return fail(rc);
    if (cudaEventRecord(hp->ev[1 + nc + i], st) != cudaSuccess ||
        cudaStreamWaitEvent(hp->s_out, hp->ev[1 + nc + i], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t*>(h_host) + t0 * row_bytes, h_dev + t0 * row_bytes,
                        tn * row_bytes, cudaMemcpyDeviceToHost, hp->s_out) != cudaSuccess)
      return fail(MOE_ERR_CUDA);
  }
  return cudaStreamSynchronize(hp->s_out) == cudaSuccess &&
                 cudaStreamSynchronize(st) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

int moe_expert_balance(const moe_shape_t* shape, const void* u, const void* E, const float* bias,
                       const int32_t* counts, float* f, float* P, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
  if (int rc = validate(shape)) return rc;
  if (shape->T == 0) return MOE_ERR_SHAPE;  // eqs. (12)-(13) divide by T
  if (!u || !E || !counts || !f || !P || !ws) return MOE_ERR_NULLPTR;
  if (misaligned(u) || misaligned(E) || misaligned(ws) || (bias && misaligned(bias)))
    return MOE_ERR_ALIGN;
  const Layout L = layout_of(*shape);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  DeviceInfo di;
  if (int rc = device_info(&di)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Stage sg(MOE_KERNEL_BALANCE, st);
  float* pstat = at<float>(ws, L.pstat);
  // the router pass also rewrites the workspace's idx / w scratch
  if (int rc = launch_router(shape->dtype, u, E, bias, shape->T, shape->d, shape->n_routed,
                             shape->top_k, shape->flags, at<int32_t>(ws, L.idx), at<float>(ws, L.w),
                             pstat, at<int32_t>(ws, L.status), st))
    return rc;
  return launch_balance_reduce(pstat, router_num_ctas(shape->T), counts, shape->T,
                               shape->n_routed, shape->top_k, f, P, st);
}

int moe_read_status(const void* ws, int32_t* status, moe_stream_t stream) {
  if (!ws || !status) return MOE_ERR_NULLPTR;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* dev = reinterpret_cast<int32_t*>(const_cast<void*>(ws));
  if (cudaMemcpyAsync(status, dev, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaMemsetAsync(dev, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
