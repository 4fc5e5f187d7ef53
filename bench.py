"""Benchmark of the DeepSeekMoE layer forward on B200 GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config large]
                    [--impl ours|reference] [--no-per-config]

A step is one whole layer forward (router, dispatch, expert FFNs, combine)
over one batch of T synthetic tokens, through the C ABI (moe_layer_forward)
with the activations resident in HBM, replayed from captured CUDA graphs
(`--eager` launches the kernels directly).  Between timed steps L2 is flushed
(a 256 MB memset, outside the step's events).  Every rank runs its own batch
with replicated weights (tokens are independent, so there is no collective on
the data path: weak scaling); the time is the max over ranks.

The headline workload is the largest layer (T=32768, d=4096, 128 routed + 4
shared experts, I=1536, top-12).  One JSON line is printed by rank 0.  Besides
the step throughput it holds:
* e2e: the same metric through moe_layer_forward_host (u and h in pinned
  host memory, both copies inside the timed call);
* roofline: the grouped gate/up GEMM (the dominant kernel) against the
  measured dense-bf16 peak, from CUDA events around that kernel inside the
  timed steps; `expert_gemms` adds the down GEMM;
* per_config (one GPU): the small layer, the 16B-shaped prefill layer and the
  16B-shaped decode steps T = 1, 8, 32, 128, each timed on its own with CUDA
  events and its own clock samples.  Decode entries report the whole layer's
  streamed weight bytes (activated experts + router) per step against the HBM
  copy peak;
* cpu_baseline: the fp64 CPU oracle, single-threaded, timed on a bounded
  sample of tokens;
* clocks: SM clock and throttle reasons sampled during the timed region.
`--impl reference` times the CPU oracle alone (the reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
import re
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
# B200 datasheet figures (context): dense bf16 tensor-core peak, HBM3e bandwidth
DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_HBM_GBS = 7700.0
HEADLINE = "large"
PER_CONFIG = ("small", "16b", "decode1", "decode8", "decode32", "decode128")


def load_peaks():
    """The roofline denominators: MEASURED_PEAKS.json where present (any key
    it lacks from the fallback figures), else the fallback figures."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        peaks = {k: float(d.get(k, v)) for k, v in FALLBACK_PEAKS.items()}
        return peaks, "measured (MEASURED_PEAKS.json)"
    return dict(FALLBACK_PEAKS), "fallback (no MEASURED_PEAKS.json)"


def workload_desc(wl):
    return (f"{wl.name}: T={wl.T} d={wl.d} routed={wl.n_routed} shared={wl.n_shared} "
            f"I={wl.inter} top-{wl.top_k} {wl.dtype}"
            + (f" router-bias N(0,{wl.bias_var})" if wl.bias_var else "")
            + (f" Zipf({wl.zipf_s}) router norms" if wl.zipf_s else ""))


def weight_bytes_streamed(wl, counts, gate_up_only=False):
    """Bytes of weights a forward must read: the W1/W3/W2 rows of every
    routed expert the batch hits plus the shared ones, and the router
    centroids (decode roofline).  gate_up_only: the W1/W3 share that the
    gate/up GEMM reads (2 d I per expert)."""
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

    def __init__(self, device_index: int, period_s: float = 0.002):
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

    def _sample(self):
        nv = self._nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
            mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            for bit, name in self.REASONS.items():
                if mask & bit and name != "gpu_idle":
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self._t.join()
            if not self.samples:
                self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- the oracle
def _single_thread():
    """Context that limits the BLAS under numpy to one thread (the oracle is
    a single-threaded baseline); returns (context, thread count)."""
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1), 1
    except Exception:  # pragma: no cover - threadpoolctl ships with the image
        import contextlib
        return contextlib.nullcontext(), None


def oracle_inputs(x):
    f = {k: x.as_f64(k) for k in ("E", "bias", "W1", "W3", "W2", "W1_s", "W3_s", "W2_s")}
    return x.as_f64("u"), f


def oracle_tokens_per_s(x, budget_s: float, max_tokens: int | None = None):
    """The CPU oracle (as it stands, BLAS on one thread) on the first S
    tokens of the workload, S grown until one run takes about budget_s / 4
    or more; returns (tokens/s, S, threads, seconds of the last run)."""
    from oracle import moe_oracle as O
    wl = x.wl
    u, f = oracle_inputs(x)
    cap = wl.T if max_tokens is None else min(wl.T, max_tokens)
    ctx, threads = _single_thread()

    def run(S):
        t0 = time.perf_counter()
        O.layer_forward(u[:S], f["E"], f["bias"], f["W1"], f["W3"], f["W2"], f["W1_s"],
                        f["W3_s"], f["W2_s"], wl.top_k)
        return time.perf_counter() - t0

    with ctx:
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
    from oracle import moe_oracle as O
    wl = S.WORKLOADS[args.config]
    x = S.make_inputs(wl)
    # size the per-step sample so that the whole run stays within a few minutes
    rate, _, threads, _ = oracle_tokens_per_s(x, budget_s=2.0)
    steps_total = args.steps + args.warmup
    per_step_s = max(0.05, min(10.0, 120.0 / max(1, steps_total)))
    sample = int(max(1, min(wl.T, rate * per_step_s)))
    u, f = oracle_inputs(x)

    def step():
        O.layer_forward(u[:sample], f["E"], f["bias"], f["W1"], f["W3"], f["W2"], f["W1_s"],
                        f["W3_s"], f["W2_s"], wl.top_k)

    ctx, _ = _single_thread()
    with ctx:
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
        "config": {"workload": workload_desc(wl), "tokens_per_gpu_step": sample,
                   "note": "fp64 CPU oracle, BLAS on one thread, on the first tokens of "
                           "the batch"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"first {sample} of {wl.T} tokens per step, full weights, "
                                   f"one BLAS thread"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------- our arm
# the source files each roofline kernel is built from: a traffic record counts
# only while they are unchanged
KERNEL_SOURCES = {
    # the prefill layers' gate/up GEMM: the CTA-pair kernels
    "gate_up": ("gemm_sm100_pair", "gemm_sm100.h", "sm100_ptx", "common.cuh"),
    "decode_layer": ("decode_fused", "sm100_ptx", "common.cuh"),
}


def _code_only(text):
    """Source text without its comments and blank lines: a record stays valid
    across comment edits, not across code changes."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*", "", line).rstrip() for line in text.splitlines())
    return "\n".join(line for line in lines if line)


def kernel_source_hash(kind="gate_up"):
    p = os.path.join(ROOT, "mixture_experts_layer_56_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(p)):
        if f.startswith(KERNEL_SOURCES[kind]):
            h.update(_code_only(open(os.path.join(p, f), encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(config_name, kind="gate_up"):
    """DRAM bytes per launch of the roofline kernel (`kind`) from the committed
    ncu record, if it was taken on this workload and the current source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        for d in json.load(open(p))["records"]:
            if (d.get("kind") == kind and d.get("workload") == config_name
                    and d.get("source_hash") == kernel_source_hash(kind)):
                return d.get("dram_bytes_per_launch")
    except Exception:
        return None
    return None


class Bench:
    """Per-process state of our arm: device, process group, peaks."""

    def __init__(self, args):
        import torch
        import torch.distributed as dist
        from mixture_experts_layer_56_b200 import _lib as L
        self.torch, self.dist, self.L = torch, dist, L
        self.args = args
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        local = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world > 1:
            from datetime import timedelta
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                    device_id=torch.device(f"cuda:{local}"))
        self.dev = torch.device(f"cuda:{local}")
        torch.cuda.set_device(self.dev)
        if not os.path.exists(L.LIB_PATH):
            import __graft_entry__
            __graft_entry__.build()
        self.flags = {"auto": 0, "single": L.MOE_FLAG_GEMM_SINGLE_CTA,
                      "pair": L.MOE_FLAG_GEMM_CTA_PAIR}[args.gemm]
        self.peaks, self.peak_src = load_peaks()
        self.flush = torch.empty(256 << 20, dtype=torch.uint8, device=self.dev)

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()
        self.torch.cuda.synchronize(self.dev)

    # ------------------------------------------------------------------ timing
    def time_forward(self, layer, u, h, steps, warmup):
        """Times `steps` forwards (graph replays unless --eager) with CUDA
        events on the launching stream, L2 flushed before each.  Returns the
        per-step times (max over ranks), the clock record, the gate/up
        kernel's event times from inside the timed steps, and the number of
        library kernels a forward launches."""
        torch, L = self.torch, self.L
        dev = self.dev
        T = u.shape[0]
        shape = layer.shape_for(T)
        stream = torch.cuda.current_stream(dev)

        def forward():
            # the stream current at call time (a graph capture switches it)
            L.moe_layer_forward(shape, u, layer.E, layer.bias, layer.W13, layer.W2,
                                layer.W13_s, layer.W2_s, h, layer.ws,
                                stream=torch.cuda.current_stream(dev))

        dominant = (L.MOE_KERNEL_GEMM_GATE_UP if layer.wl.dtype == "bf16"
                    else L.MOE_KERNEL_FFN_F32)
        timed_kinds = (dominant,)
        graphs = []
        forward()
        torch.cuda.synchronize(dev)
        c0 = L.moe_launch_count()
        forward()
        torch.cuda.synchronize(dev)
        per_forward = L.moe_launch_count() - c0
        if not self.args.eager:
            # the forward captured into a few CUDA graphs, replayed in turn, one
            # per step (the C ABI only enqueues work on the caller's stream, so
            # it captures as is).  Half of them also capture event records
            # around the dominant kernel: after the timed loop those events hold
            # the kernel's last runs inside the timed steps.
            L.moe_profile_read()
            n_graphs = min(8, max(1, steps))
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

        for _ in range(max(3, warmup)):
            self.flush.zero_()
            step()
        assert layer.status() == 0
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        self.barrier()
        if not graphs:
            L.moe_profile_read()
            L.moe_profile_enable(True, kinds=timed_kinds)
        step_no[0] = 0
        with ClockSampler(dev.index if dev.index is not None else 0) as clk:
            for i in range(steps):
                self.flush.zero_()
                starts[i].record(stream)
                step()
                ends[i].record(stream)
            self.barrier()
        recs = L.moe_profile_read()  # eager: every timed step; graphs: each one's last replay
        L.moe_profile_enable(False)
        graphs.clear()
        step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
        total_ms = max_over_ranks(sum(step_ms), dev)
        assert layer.status() == 0
        return dict(total_ms=total_ms, ms_per_step=total_ms / steps, clocks=clk.summary(),
                    timed_recs=recs, per_forward=int(per_forward), forward=forward)

    def stage_times(self, forward, n=20):
        """Every stage's device time: a separate, untimed pass."""
        torch, L = self.torch, self.L
        L.moe_profile_enable(True)
        for _ in range(n):
            self.flush.zero_()
            forward()
        torch.cuda.synchronize(self.dev)
        recs = L.moe_profile_read()
        L.moe_profile_enable(False)
        return mean_ms(recs)

    # ----------------------------------------------------------------- one config
    def measure(self, layer, u, steps, warmup):
        """One workload: throughput, roofline, stage times, clocks."""
        wl = layer.wl
        T = u.shape[0]
        h = self.torch.empty_like(u)
        r = self.time_forward(layer, u, h, steps, warmup)
        stage_ms = self.stage_times(r["forward"])
        kernel_ms = dict(stage_ms)
        kernel_ms.update(mean_ms(r["timed_recs"]))  # the roofline kernel: timed steps
        ms = r["ms_per_step"]
        world = self.world
        out = {
            "workload": workload_desc(wl),
            "tokens_per_gpu_step": T,
            "steps": steps,
            "ms_per_step": ms,
            "value": T * world / (ms / 1e3),
            "unit": "tokens/s",
            "expert_tflops": wl.expert_flops() / (ms / 1e3) / 1e12,
            "stage_ms": {k: round(v, 4) for k, v in stage_ms.items()},
            "gpu_launches_per_step": r["per_forward"],
            "clocks": r["clocks"],
        }
        out["expert_tflops_frac_of_datasheet"] = out["expert_tflops"] / DATASHEET_BF16_TFLOPS
        capped = "sw_power_cap" in (r["clocks"].get("reasons") or [])
        peak_tf = float(self.peaks["bf16_tflops_sustained" if capped else "bf16_tflops"])
        if wl.dtype == "bf16" and T >= 1024:
            gu = "grouped_gemm_gate_up_swiglu"
            gate_up_flops = 4.0 * T * (wl.top_k + wl.n_shared) * wl.d * wl.inter
            gu_ms = kernel_ms[gu]
            achieved = gate_up_flops / (gu_ms / 1e3) / 1e12
            out["roofline"] = {
                "bound": "tensor", "kernel": gu, "achieved": achieved, "peak": peak_tf,
                "unit": "TFLOP/s", "frac": achieved / peak_tf, "traffic": ncu_traffic(wl.name),
                "frac_of_burst": achieved / float(self.peaks["bf16_tflops"]),
                "frac_of_sustained": achieved / float(self.peaks["bf16_tflops_sustained"]),
                "frac_of_datasheet": achieved / DATASHEET_BF16_TFLOPS,
                "peak_source": f"{self.peak_src} bf16 {'sustained' if capped else 'burst'}; "
                               f"datasheet dense bf16 "
                               f"{DATASHEET_BF16_TFLOPS:.0f} TFLOP/s for frac_of_datasheet",
                "flops_per_launch": gate_up_flops, "ms_per_launch": gu_ms}
            down_ms = stage_ms.get("grouped_gemm_down")
            if down_ms:
                # both expert GEMMs (per-stage events of the untimed pass)
                both_ms = stage_ms[gu] + down_ms
                tf = wl.expert_flops() / (both_ms / 1e3) / 1e12
                out["expert_gemms"] = {
                    "ms": both_ms, "tflops": tf, "frac_of_peak": tf / peak_tf,
                    "frac_of_datasheet": tf / DATASHEET_BF16_TFLOPS,
                    "down_tflops": 2.0 * T * (wl.top_k + wl.n_shared) * wl.d * wl.inter
                                   / (down_ms / 1e3) / 1e12,
                    "source": "CUDA events around each GEMM, untimed eager pass"}
        else:
            # decode-sized batches: the layer streams the activated experts'
            # W1/W3/W2 and the router centroids once per step
            counts = routed_counts(layer, u, self.L, self.torch)
            bf16 = wl.dtype == "bf16"
            layer_bytes = weight_bytes_streamed(wl, counts)
            act_bytes = 2 * T * wl.d * (2 if bf16 else 4)
            hbm = float(self.peaks["hbm_gbs"])
            achieved = (layer_bytes + act_bytes) / (ms / 1e3) / 1e9
            out["experts_hit"] = int((counts > 0).sum()) + wl.n_shared
            one_kernel = (self.L.moe_forward_path(layer.shape_for(T))
                          == self.L.MOE_PATH_DECODE_LAYER)  # the decode layer kernel
            out["roofline"] = {
                "bound": "hbm", "kernel": "whole layer forward (all kernels of one step)",
                "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "frac_of_datasheet": achieved / DATASHEET_HBM_GBS,
                "traffic": ncu_traffic(wl.name, "decode_layer") if one_kernel else None,
                "peak_source": f"{self.peak_src} HBM copy",
                "bytes_per_step": layer_bytes + act_bytes, "ms_per_step": ms,
                "bytes": "W1/W3/W2 of the hit routed + shared experts, E, u in, h out"}
            name = "grouped_gemm_gate_up_swiglu" if bf16 else "ffn_f32"
            k_ms = kernel_ms.get(name, 0.0)
            if k_ms > 0:
                kb = weight_bytes_streamed(wl, counts, gate_up_only=bf16)
                out["gate_up_kernel"] = {
                    "ms": k_ms, "bytes": kb, "gbs": kb / (k_ms / 1e3) / 1e9,
                    "frac": kb / (k_ms / 1e3) / 1e9 / hbm,
                    "source": "CUDA events around the kernel inside the timed graph "
                              "replays (the bracket also covers its launch)"}
        return out

    def e2e(self, layer, u, steps):
        """The headline metric through moe_layer_forward_host: pinned host
        u and h, both copies inside every timed call."""
        torch = self.torch
        stream = torch.cuda.current_stream(self.dev)
        u_h = u.cpu().pin_memory()
        h_h = torch.empty_like(u_h).pin_memory()
        layer.forward_host(u_h, h_h, stream=stream)
        self.barrier()
        e_start = torch.cuda.Event(enable_timing=True)
        e_end = torch.cuda.Event(enable_timing=True)
        e_start.record(stream)
        for _ in range(steps):
            layer.forward_host(u_h, h_h, stream=stream)
        e_end.record(stream)
        self.barrier()
        ms = max_over_ranks(e_start.elapsed_time(e_end), self.dev)
        T = u.shape[0]
        io = T * layer.wl.d * (2 if layer.wl.dtype == "bf16" else 4)
        return {"value": T * self.world * steps / (ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": io, "d2h_bytes_per_step": io, "steps": steps}


def mean_ms(rs):
    acc = {}
    for name, ms in rs:
        acc.setdefault(name, []).append(ms)
    return {k: sum(v) / len(v) for k, v in acc.items()}


def run_ours(args):
    import gc

    from mixture_experts_layer_56_b200 import synthetic as S
    from mixture_experts_layer_56_b200.layer import MoELayer, to_device

    b = Bench(args)
    torch = b.torch
    wl = S.WORKLOADS[args.config]
    x = S.make_inputs(wl)
    layer = MoELayer(x, b.dev, flags=b.flags, host_io=True)
    u = to_device(x.u, b.dev)
    main = b.measure(layer, u, args.steps, args.warmup)
    e2e = b.e2e(layer, u, max(3, min(args.steps, 50)))
    del layer, u
    gc.collect()
    torch.cuda.empty_cache()

    # ---- the other workloads (one GPU): each timed on its own ---------------
    per_config = {}
    if b.world == 1 and not args.no_per_config:
        names = [n for n in PER_CONFIG if n != args.config]
        x16 = None
        for name in names:
            wl_c = S.WORKLOADS[name]
            steps_c = max(10, min(args.steps, 200))
            if name.startswith("decode") or name == "16b":
                # the decode steps run on the 16B-shaped layer's weights, with
                # the first T tokens of its batch
                if x16 is None:
                    x16 = S.make_inputs(S.WORKLOADS["16b"])
                    layer16 = MoELayer(x16, b.dev, flags=b.flags)
                    u16 = to_device(x16.u, b.dev)
                layer_c = layer16
                if name == "16b":
                    u_c = u16
                else:
                    u_c = u16[: wl_c.T].contiguous()
                    layer_c = _LayerView(layer16, wl_c)
            else:
                xc = S.make_inputs(wl_c)
                layer_c = MoELayer(xc, b.dev, flags=b.flags)
                u_c = to_device(xc.u, b.dev)
            per_config[name] = b.measure(layer_c, u_c, steps_c, args.warmup)
            if not (name.startswith("decode") or name == "16b"):
                del layer_c, u_c
                gc.collect()
                torch.cuda.empty_cache()

    # ---- CPU baseline (rank 0, N = 1 only) ----------------------------------
    cpu = None
    if b.rank == 0 and b.world == 1 and not args.no_cpu_baseline:
        rate, S_tok, threads, dt = oracle_tokens_per_s(x, budget_s=args.cpu_budget)
        cpu = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"fp64 oracle layer forward (BLAS on one thread) on the first "
                         f"{S_tok} of {wl.T} tokens, full weights ({dt:.1f} s)"}

    if b.rank == 0:
        line = {
            "metric": METRIC, "value": main["value"], "unit": "tokens/s", "n_gpus": b.world,
            "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": main["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": main["workload"], "tokens_per_gpu_step": wl.T,
                       "gemm_tiles": args.gemm, "cuda_graph": not args.eager,
                       "parallelism": f"replicas x{b.world} (token batches, no collective)",
                       "l2": "flushed between steps (256 MB memset outside the step events)",
                       "init": "seeded splitmix64/Box-Muller normals, bf16"},
            "tflops": main["expert_tflops"],
            "tflops_frac_of_bf16_peak": main["expert_tflops"] / float(b.peaks["bf16_tflops"]),
            "tflops_frac_of_datasheet": main["expert_tflops_frac_of_datasheet"],
            "stage_ms": main["stage_ms"],
            "stage_ms_source": "CUDA events around every stage, 20 untimed steps; the "
                               "roofline kernel's time comes from events inside the timed steps",
            "gpu_launches": main["gpu_launches_per_step"] * args.steps,
            "e2e": e2e,
            "roofline": main["roofline"],
            "expert_gemms": main.get("expert_gemms"),
            "cpu_baseline": cpu,
            "clocks": main["clocks"],
            "per_config": per_config,
        }
        print(json.dumps(line), flush=True)
    if b.world > 1:
        b.dist.barrier()
        b.dist.destroy_process_group()
    return 0


class _LayerView:
    """The 16B-shaped layer's device weights and workspace under another
    workload's name (the decode steps use its first T tokens)."""

    def __init__(self, layer, wl):
        self._layer = layer
        self.wl = wl

    def __getattr__(self, k):
        return getattr(self._layer, k)


def routed_counts(layer, u, L, torch):
    """Per-expert token counts of this batch, through moe_route + moe_dispatch."""
    wl = layer.wl
    T, K, n = u.shape[0], wl.top_k, wl.n_routed
    shape = layer.shape_for(T)
    i32 = dict(dtype=torch.int32, device=layer.device)
    idx = torch.empty((T, K), **i32)
    w = torch.empty((T, K), dtype=torch.float32, device=layer.device)
    L.moe_route(shape, u, layer.E, layer.bias, idx, w)
    counts = torch.empty(n, **i32)
    offsets = torch.empty(n + 1, **i32)
    perm = torch.empty(T * K, **i32)
    inv = torch.empty(T * K, **i32)
    L.moe_dispatch(shape, idx, counts, offsets, perm, inv, layer.ws)
    return counts.cpu().numpy()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=HEADLINE)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the --config workload")
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
