"""Benchmark of the DeepSeekMoE layer forward on B200 GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config small]
                    [--impl ours|reference]

A step is one whole layer forward (router, dispatch, expert FFNs, combine)
over one batch of T synthetic tokens, through the C ABI (moe_layer_forward)
with the activations resident in HBM, replayed from captured CUDA graphs
(`--eager` launches the kernels directly).  Between timed steps L2 is flushed
(a 256 MB memset, outside the step's events).  Every rank runs its own batch
with replicated weights (tokens are independent, so there is no collective on
the data path: weak scaling); the time is the max over ranks.

One JSON line is printed by rank 0.  Besides the step throughput it holds:
* e2e: the same metric through moe_layer_forward_host (u and h in pinned
  host memory, both copies inside the timed call);
* roofline: the grouped gate/up GEMM (the dominant kernel) against the
  measured dense-bf16 peak (decode-sized batches: the HBM copy peak, for the
  W1/W3 bytes of the activated experts), from CUDA events around that kernel
  inside the timed steps;
* cpu_baseline: the fp64 CPU oracle timed on a bounded sample of tokens;
* clocks: SM clock and throttle reasons sampled during the timed region.
`--impl reference` times the CPU oracle alone (the reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer fwd tokens/s and TFLOP/s (% B200 BF16 peak); decode GB/s (% HBM)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def workload_desc(wl):
    return (f"{wl.name}: T={wl.T} d={wl.d} routed={wl.n_routed} shared={wl.n_shared} "
            f"I={wl.inter} top-{wl.top_k} {wl.dtype}"
            + (f" router-bias N(0,{wl.bias_var})" if wl.bias_var else "")
            + (f" Zipf({wl.zipf_s}) router norms" if wl.zipf_s else ""))


def weight_bytes_streamed(wl, counts, gate_up_only=False):
    """Bytes of expert weights a forward must read: every expert hit plus the
    shared ones (decode roofline).  gate_up_only: the W1/W3 share that the
    gate/up GEMM reads (2 d I per expert); else all three matrices and the
    router centroids."""
    el = 2 if wl.dtype == "bf16" else 4
    hit = int((counts > 0).sum())
    if gate_up_only:
        return (hit + wl.n_shared) * 2 * wl.d * wl.inter * el
    return (hit + wl.n_shared) * 3 * wl.d * wl.inter * el + wl.n_routed * wl.d * el


def max_over_ranks(x: float, device=None) -> float:
    """The largest value of x over all ranks (x itself without a process
    group): the job's time is its slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Polls the SM clock and the clock-event reasons (read only) during the
    timed region, through NVML, every few milliseconds."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass
        self.period = period_s
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- the oracle
def oracle_tokens_per_s(x, budget_s: float, max_tokens: int | None = None):
    """The CPU oracle (as it stands) on the first S tokens of the workload,
    S grown until one run takes about budget_s; returns (tokens/s, S, threads)."""
    import numpy as np
    from oracle import moe_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        threads = 1
    wl = x.wl
    f = {k: x.as_f64(k) for k in ("E", "bias", "W1", "W3", "W2", "W1_s", "W3_s", "W2_s")}
    u = x.as_f64("u")
    cap = wl.T if max_tokens is None else min(wl.T, max_tokens)

    def run(S):
        t0 = time.perf_counter()
        O.layer_forward(u[:S], f["E"], f["bias"], f["W1"], f["W3"], f["W2"], f["W1_s"],
                        f["W3_s"], f["W2_s"], wl.top_k)
        return time.perf_counter() - t0

    S = min(16, cap)
    dt = run(S)
    while dt < budget_s / 4 and S < cap:
        S = min(cap, S * 4)
        dt = run(S)
    return S / dt, S, threads, dt


# --------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from mixture_experts_layer_56_b200 import synthetic as S
    wl = S.WORKLOADS[args.config]
    x = S.make_inputs(wl)
    # size the per-step sample so that the whole run stays within a few minutes
    rate, S_cal, threads, _ = oracle_tokens_per_s(x, budget_s=2.0)
    steps_total = args.steps + args.warmup
    per_step_s = max(0.05, min(10.0, 120.0 / max(1, steps_total)))
    sample = int(max(1, min(wl.T, rate * per_step_s)))
    import numpy as np
    from oracle import moe_oracle as O
    f = {k: x.as_f64(k) for k in ("E", "bias", "W1", "W3", "W2", "W1_s", "W3_s", "W2_s")}
    u = x.as_f64("u")

    def step():
        O.layer_forward(u[:sample], f["E"], f["bias"], f["W1"], f["W3"], f["W2"], f["W1_s"],
                        f["W3_s"], f["W2_s"], wl.top_k)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = sample * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(wl), "tokens_per_step": sample,
                   "note": "fp64 CPU oracle on the first tokens of the batch"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"first {sample} of {wl.T} tokens per step, full weights"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------- our arm
def kernel_source_hash():
    p = os.path.join(ROOT, "mixture_experts_layer_56_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(p)):
        if f.startswith("gemm_sm100") or f.startswith("sm100_ptx"):
            h.update(open(os.path.join(p, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(config_name):
    """DRAM bytes per launch of the gate/up GEMM from a committed ncu summary,
    if it was taken on the current kernel source and this workload."""
    p = os.path.join(ROOT, "profiles", "gemm_gate_up_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        if d.get("source_hash") == kernel_source_hash() and d.get("workload") == config_name:
            return d.get("dram_bytes_per_launch")
    except Exception:
        return None
    return None


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from mixture_experts_layer_56_b200 import _lib as L
    from mixture_experts_layer_56_b200 import synthetic as S
    from mixture_experts_layer_56_b200.layer import MoELayer, to_device

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device(f"cuda:{local}"))
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    if not os.path.exists(L.LIB_PATH):
        import __graft_entry__
        __graft_entry__.build()

    wl = S.WORKLOADS[args.config]
    x = S.make_inputs(wl)
    flags = {"auto": 0, "single": L.MOE_FLAG_GEMM_SINGLE_CTA, "pair": L.MOE_FLAG_GEMM_CTA_PAIR}[args.gemm]
    layer = MoELayer(x, dev, flags=flags, host_io=True)
    u = to_device(x.u, dev)
    h = torch.empty_like(u)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def forward():
        # the stream current at call time (a graph capture switches it)
        L.moe_layer_forward(layer.shape, u, layer.E, layer.bias, layer.W13, layer.W2,
                            layer.W13_s, layer.W2_s, h, layer.ws,
                            stream=torch.cuda.current_stream(dev))

    # CUDA events around the dominant kernel, on the stream it runs on,
    # inside the timed steps; the other stages are bracketed in a separate
    # pass so that their events do not stretch the timed steps
    dominant = L.MOE_KERNEL_GEMM_GATE_UP if wl.dtype == "bf16" else L.MOE_KERNEL_FFN_F32
    timed_kinds = (dominant,)

    graphs = []
    if not args.eager:
        # the forward captured into a few CUDA graphs, replayed in turn, one
        # per step (the C ABI only enqueues work on the caller's stream, so it
        # captures as is).  Half of them also capture event records around
        # the dominant kernel: after the timed loop those events hold the
        # kernel's last runs inside the timed steps (the other graphs carry
        # no events, which would stretch the steps a little).
        forward()
        torch.cuda.synchronize(dev)
        L.moe_profile_read()
        n_graphs = min(8, max(1, args.steps))
        for i in range(n_graphs):
            L.moe_profile_enable(i % 2 == 0, kinds=timed_kinds)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                forward()
            graphs.append(g)
        L.moe_profile_enable(False)
        torch.cuda.synchronize(dev)
    step_no = [0]

    def step():
        if graphs:
            graphs[step_no[0] % len(graphs)].replay()
            step_no[0] += 1
        else:
            forward()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    assert layer.status() == 0
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    launches0 = L.moe_launch_count()
    if not graphs:
        L.moe_profile_read()
        L.moe_profile_enable(True, kinds=timed_kinds)
    step_no[0] = 0
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        barrier()
    launches = L.moe_launch_count() - launches0
    recs = L.moe_profile_read()  # eager: every timed step; graphs: each one's last replay
    L.moe_profile_enable(False)
    if graphs:
        # replays bypass the library's launch counter: count one eager step
        c0 = L.moe_launch_count()
        forward()
        torch.cuda.synchronize(dev)
        launches = (L.moe_launch_count() - c0) * args.steps
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), dev)
    assert layer.status() == 0
    tokens = wl.T * world * args.steps
    value = tokens / (total_ms / 1e3)
    ms_per_step = total_ms / args.steps
    tflops = wl.expert_flops() * world * args.steps / (total_ms / 1e3) / 1e12

    timed_recs = recs
    graphs.clear()
    # ---- every stage's device time: a separate, untimed pass ---------------
    L.moe_profile_enable(True)
    for _ in range(20):
        flush.zero_()
        forward()
    torch.cuda.synchronize(dev)
    stage_recs = L.moe_profile_read()
    L.moe_profile_enable(False)

    def mean_ms(rs):
        acc = {}
        for name, ms in rs:
            acc.setdefault(name, []).append(ms)
        return {k: sum(v) / len(v) for k, v in acc.items()}
    stage_ms = mean_ms(stage_recs)
    # the roofline kernels' time: from the timed steps
    kernel_ms = dict(stage_ms)
    kernel_ms.update(mean_ms(timed_recs))

    # ---- e2e through the host-buffer entry point ---------------------------
    u_h = u.cpu().pin_memory()
    h_h = torch.empty_like(u_h).pin_memory()
    e2e_steps = max(3, min(args.steps, 50))
    layer.forward_host(u_h, h_h, stream=stream)
    barrier()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(e2e_steps):
        layer.forward_host(u_h, h_h, stream=stream)
    e_end.record(stream)
    barrier()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), dev)
    e2e_value = wl.T * world * e2e_steps / (e2e_ms / 1e3)
    io_bytes = wl.T * wl.d * (2 if wl.dtype == "bf16" else 4)

    # ---- roofline of the dominant kernel -----------------------------------
    peaks, peak_src = load_peaks()
    clocks = clk.summary()
    if wl.dtype == "bf16" and "grouped_gemm_gate_up_swiglu" in kernel_ms and wl.T >= 1024:
        gate_up_flops = 4.0 * wl.T * (wl.top_k + wl.n_shared) * wl.d * wl.inter
        ms = kernel_ms["grouped_gemm_gate_up_swiglu"]
        achieved = gate_up_flops / (ms / 1e3) / 1e12
        # the sustained GEMM peak when the power cap held the clocks down
        # during the timed steps, else the burst one
        capped = "sw_power_cap" in (clocks.get("reasons") or [])
        peak = float(peaks["bf16_tflops_sustained" if capped else "bf16_tflops"])
        roofline = {"bound": "tensor", "kernel": "grouped_gemm_gate_up_swiglu",
                    "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": ncu_traffic(wl.name),
                    "frac_of_burst": achieved / float(peaks["bf16_tflops"]),
                    "frac_of_sustained": achieved / float(peaks["bf16_tflops_sustained"]),
                    "peak_source": f"{peak_src} bf16 {'sustained' if capped else 'burst'} "
                                   f"(MEASURED_PEAKS.json)",
                    "flops_per_launch": gate_up_flops, "ms_per_launch": ms}
    else:
        # decode-sized batches: the gate/up GEMM streams the activated experts'
        # W1/W3 (the fp32 layer's single FFN kernel streams all three)
        counts = routed_counts(layer, u, L, torch)
        bf16 = wl.dtype == "bf16"
        byts = weight_bytes_streamed(wl, counts, gate_up_only=bf16)
        name = "grouped_gemm_gate_up_swiglu" if bf16 else "ffn_f32"
        ms = kernel_ms.get(name, 0.0)
        achieved = byts / (ms / 1e3) / 1e9 if ms > 0 else None
        peak = float(peaks["hbm_gbs"])
        roofline = {"bound": "hbm", "kernel": name,
                    "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": (achieved / peak) if achieved else None, "traffic": None,
                    "peak_source": f"{peak_src} HBM copy (MEASURED_PEAKS.json)",
                    "bytes_per_launch": byts, "ms_per_launch": ms}

    # ---- CPU baseline (rank 0, N = 1 only) -----------------------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, S_tok, threads, dt = oracle_tokens_per_s(x, budget_s=args.cpu_budget)
        cpu = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"fp64 oracle layer forward on the first {S_tok} of {wl.T} tokens "
                         f"({dt:.1f} s)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": workload_desc(wl), "tokens_per_gpu_step": wl.T,
                       "gemm_tiles": args.gemm, "cuda_graph": not args.eager,
                       "parallelism": f"replicas x{world} (token batches, no collective)",
                       "l2": "flushed between steps (256 MB memset outside the step events)",
                       "init": "seeded splitmix64/Box-Muller normals, bf16"},
            "tflops": tflops,
            "tflops_frac_of_bf16_peak": tflops / float(peaks["bf16_tflops"]),
            "stage_ms": {k: round(v, 4) for k, v in stage_ms.items()},
            "stage_ms_source": "CUDA events around every stage, 20 untimed steps; the "
                               "roofline kernel's time comes from events inside the timed steps",
            "gpu_launches": int(launches),
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": io_bytes,
                    "d2h_bytes_per_step": io_bytes},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def routed_counts(layer, u, L, torch):
    """Per-expert token counts of this batch, through moe_route + moe_dispatch."""
    wl = layer.wl
    T, K, n = wl.T, wl.top_k, wl.n_routed
    i32 = dict(dtype=torch.int32, device=layer.device)
    idx = torch.empty((T, K), **i32)
    w = torch.empty((T, K), dtype=torch.float32, device=layer.device)
    L.moe_route(layer.shape, u, layer.E, layer.bias, idx, w)
    counts = torch.empty(n, **i32)
    offsets = torch.empty(n + 1, **i32)
    perm = torch.empty(T * K, **i32)
    inv = torch.empty(T * K, **i32)
    L.moe_dispatch(layer.shape, idx, counts, offsets, perm, inv, layer.ws)
    return counts.cpu().numpy()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="small")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch every step's kernels directly instead of replaying a captured "
                         "CUDA graph")
    ap.add_argument("--gemm", default="auto", choices=["auto", "single", "pair"],
                    help="tile shape of the expert GEMMs (default: chosen by the library)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
