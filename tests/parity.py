"""Helpers of the GPU parity tests: run every stage of the layer through the C
ABI and compare it with the CPU oracle on the same seeded inputs.

Bars (the layer's floating-point results are bf16 with fp32 accumulation):
* routing indices, per-expert counts, offsets, the permutation and its
  inverse: bit-exact.  A token whose oracle scores have two of their K+1
  largest values closer than TIE_GAP is a near tie: it is counted and its
  selection only has to be a valid top-K of the oracle's scores within
  TIE_GAP.  Dispatch outputs are compared with the oracle's dispatch of the
  GPU's own routing, so they stay bit-exact on near ties too.
* gates: |w - s| <= 1e-6 + s (1e-5 + 10 * 2^-24 * sqrt(d) * L_t), L_t the
  token's largest |logit|: an fp32 sum of d products carries a rounding error
  of about 2^-24 * L * sqrt(d) (random-walk growth), and the gate's relative
  error is about twice the logits' absolute error.
* bf16 tensors: |x - x_ref| <= 2e-2 + 2^-8 |x_ref| elementwise (the second
  term is the bf16 output rounding, which alone exceeds 2e-2 once |x| > 5.12)
  and ||x - x_ref||_F / ||x_ref||_F <= 1e-2.
* fp32 layer: |x - x_ref| <= 1e-4 + 1e-5 |x_ref|, relative Frobenius <= 1e-5.

Every parity run also records the literal figures beside those bars
(error_stats, gate_stats): the plain max |err| against the fp64 oracle and
against the oracle rounded to bf16, how many elements exceed 2e-2 (and so
pass only through the 2^-8 |ref| term) and the largest |ref| among them, the
relative Frobenius error, and the worst gate error divided by the fp32 model
2^-24 sqrt(d) L_t s.  With MOE_PARITY_REPORT_DIR set, each report is written
there as parity_<workload>.json.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

from mixture_experts_layer_56_b200 import _lib as L
from mixture_experts_layer_56_b200 import synthetic as S
from mixture_experts_layer_56_b200.layer import MoELayer, to_device, to_numpy
from oracle import moe_oracle as O

TIE_GAP = 1e-5
PATH_NAMES = {L.MOE_PATH_STAGES: "stages (bit-equal to the stage-wise calls)",
              L.MOE_PATH_DECODE_LAYER: "decode layer kernel",
              L.MOE_PATH_SMALL_BATCH: "small-batch front kernel + grouped GEMMs + combine"}
NAMES = ("u", "E", "bias", "W1", "W3", "W2", "W1_s", "W3_s", "W2_s")


def f64_inputs(x: S.LayerInputs) -> dict:
    return {k: x.as_f64(k) for k in NAMES}


def as_f64(t: torch.Tensor) -> np.ndarray:
    a = to_numpy(t)
    if a.dtype == np.uint16:
        return S.bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def gpu_stages(x: S.LayerInputs, device="cuda:0", flags=0, layer=None):
    """Every stage through the C ABI, plus the fused moe_layer_forward."""
    wl = x.wl
    T, K, n, d = wl.T, wl.top_k, wl.n_routed, wl.d
    layer = layer or MoELayer(x, device, flags=flags)
    sh = layer.shape
    dev = layer.device
    u = to_device(x.u, dev)
    i32 = dict(dtype=torch.int32, device=dev)
    idx = torch.full((T, K), -1, **i32)
    w = torch.full((T, K), -1.0, dtype=torch.float32, device=dev)
    L.moe_route(sh, u, layer.E, layer.bias, idx, w)
    counts = torch.full((n,), -1, **i32)
    offsets = torch.full((n + 1,), -1, **i32)
    perm = torch.full((T * K,), -1, **i32)
    inv = torch.full((T * K,), -1, **i32)
    L.moe_dispatch(sh, idx, counts, offsets, perm, inv, layer.ws)
    y = torch.full((T * K, d), float("nan"), dtype=layer.elem_dtype, device=dev)
    ysh = torch.full((T, d), float("nan"), dtype=torch.float32, device=dev)
    L.moe_expert_ffn(sh, u, perm, offsets, layer.W13, layer.W2, layer.W13_s, layer.W2_s, y, ysh,
                     layer.ws)
    h = torch.full_like(u, float("nan"))
    L.moe_combine(sh, u, ysh, y, w, inv, h)
    h_fwd = layer.forward(u)
    torch.cuda.synchronize()
    status = layer.status()
    return dict(idx=to_numpy(idx), w=to_numpy(w), counts=to_numpy(counts),
                offsets=to_numpy(offsets), perm=to_numpy(perm), inv=to_numpy(inv),
                y=as_f64(y), ysh=as_f64(ysh), h=as_f64(h), h_raw=to_numpy(h),
                h_fwd_raw=to_numpy(h_fwd), h_fwd=as_f64(h_fwd), status=status, layer=layer,
                path=L.moe_forward_path(sh))


def check_forward(gpu: dict, ref_h: np.ndarray, near: np.ndarray, bf16: bool, tokens=None):
    """moe_layer_forward's h: the stage-wise result bit for bit, or (the
    one-kernel decode path) the oracle within the bars on every token whose
    K-th and (K+1)-th scores are not a near tie (``near``; its router may
    choose the other expert there).  Returns the error figures of the
    forward's h."""
    h_fwd = gpu["h_fwd"] if tokens is None else gpu["h_fwd"][tokens]
    if gpu["path"] == L.MOE_PATH_STAGES:
        assert np.array_equal(gpu["h_raw"], gpu["h_fwd_raw"]), "layer_forward != stage-wise result"
        return None
    keep = ~near if tokens is None else ~near[tokens]
    assert keep.any(), "every token is a near tie: the case checks nothing"
    assert_close(h_fwd[keep], ref_h[keep], f"h (forward path {gpu['path']})", bf16)
    return error_stats(h_fwd[keep], ref_h[keep], bf16)


def near_tie_tokens(s: np.ndarray, K: int) -> np.ndarray:
    """Tokens whose K+1 largest scores hold two values closer than TIE_GAP."""
    m = min(K + 1, s.shape[1])
    top = -np.sort(-s, axis=1)[:, :m]
    if m < 2:
        return np.zeros(s.shape[0], dtype=bool)
    return np.min(top[:, :-1] - top[:, 1:], axis=1) < TIE_GAP


def check_routing(idx: np.ndarray, w: np.ndarray, s: np.ndarray, K: int,
                  ref_idx: np.ndarray | None = None, gate_s: np.ndarray | None = None,
                  logits: np.ndarray | None = None, d: int = 1):
    """Returns (near-tie count, mismatch count); asserts the bars above.
    ``s`` ranks the experts (the selection key), ``gate_s`` gives the gates
    (defaults to s), ``logits`` / ``d`` set the fp32 gate tolerance."""
    gate_s = s if gate_s is None else gate_s
    if ref_idx is None:
        ref_idx, _ = O.topk_gates(s, K)
    near = near_tie_tokens(s, K)
    mism = np.any(idx != ref_idx, axis=1)
    bad = np.where(mism & ~near)[0]
    assert bad.size == 0, f"{bad.size} tokens differ outside near ties, e.g. t={bad[:5]}"
    n = s.shape[1]
    assert np.all((idx >= 0) & (idx < n))
    for t in np.where(mism)[0]:
        sel = idx[t]
        assert len(set(sel.tolist())) == K
        kth = np.sort(s[t])[::-1][K - 1]
        assert np.all(s[t, sel] >= kth - TIE_GAP)
        assert np.all(np.diff(s[t, sel]) <= TIE_GAP)
    g = np.take_along_axis(gate_s, idx.astype(np.int64), axis=1)
    err = np.abs(w.astype(np.float64) - g)
    L_t = np.abs(logits).max(axis=1, keepdims=True) if logits is not None else 1.0
    rel = 1e-5 + 10.0 * 2.0 ** -24 * np.sqrt(d) * L_t
    assert np.all(err <= 1e-6 + rel * g), float(err.max())
    return int(near.sum()), int(mism.sum())


def check_dispatch(gpu: dict, n: int):
    counts, offsets, perm, inv = O.dispatch(gpu["idx"], n)
    np.testing.assert_array_equal(gpu["counts"], counts)
    np.testing.assert_array_equal(gpu["offsets"], offsets)
    np.testing.assert_array_equal(gpu["perm"], perm)
    np.testing.assert_array_equal(gpu["inv"], inv)


def assert_close(got: np.ndarray, ref: np.ndarray, what: str, bf16: bool = True):
    if bf16:
        atol, rtol_el, rel_fro = 2e-2, 2.0 ** -8, 1e-2
    else:
        atol, rtol_el, rel_fro = 1e-4, 1e-5, 1e-5
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    bound = atol + rtol_el * np.abs(ref)
    worst = int(np.argmax(err - bound))
    assert np.all(err <= bound), (f"{what}: max |err| {err.max():.3e} (at {worst}: got "
                                  f"{got.flat[worst]:.6f}, ref {ref.flat[worst]:.6f})")
    nref = np.linalg.norm(ref)
    if nref > 0:
        rel = np.linalg.norm(got - ref) / nref
        assert rel <= rel_fro, f"{what}: relative Frobenius error {rel:.3e}"
    return float(err.max())


def bf16_round(x: np.ndarray) -> np.ndarray:
    """x rounded to float32 and then to bf16 (nearest even), as float64."""
    return S.bf16_bits_to_f32(S.f32_to_bf16_bits(x.astype(np.float32))).astype(np.float64)


def error_stats(got: np.ndarray, ref: np.ndarray, bf16: bool = True) -> dict:
    """The literal error figures of one output against the fp64 oracle."""
    err = np.abs(got - ref)
    atol = 2e-2 if bf16 else 1e-4
    over = err > atol
    nref = np.linalg.norm(ref)
    out = {
        "elements": int(err.size),
        "max_abs_err": float(err.max()) if err.size else 0.0,
        "atol": atol,
        "n_over_atol": int(over.sum()),
        "max_abs_ref_where_over_atol": float(np.abs(ref[over]).max()) if over.any() else None,
        "max_err_minus_atol_over_abs_ref": (float(((err - atol)[over] / np.abs(ref[over])).max())
                                            if over.any() else None),
        "rel_fro": float(np.linalg.norm(got - ref) / nref) if nref > 0 else 0.0,
        "max_abs_ref": float(np.abs(ref).max()) if ref.size else 0.0,
    }
    if bf16:
        out["max_abs_err_vs_bf16_rounded_ref"] = (float(np.abs(got - bf16_round(ref)).max())
                                                  if err.size else 0.0)
    return out


def gate_stats(w: np.ndarray, idx: np.ndarray, gate_s: np.ndarray, logits: np.ndarray,
               d: int, mism: np.ndarray) -> dict:
    """Gate errors (tokens whose selection matches the oracle's) against the
    bar |w - s| <= 1e-6 + s (1e-5 + F * 2^-24 sqrt(d) L_t), F = 10: the
    factor each gate needs, (|w - s| - 1e-6 - 1e-5 s) / (2^-24 sqrt(d) L_t s),
    at worst and at the 99th percentile (0 where the fixed terms cover it),
    and the same for the gates of at least 1e-3."""
    ok = ~mism
    g = np.take_along_axis(gate_s, idx.astype(np.int64), axis=1)[ok]
    err = np.abs(w.astype(np.float64)[ok] - g)
    L_t = np.abs(logits).max(axis=1, keepdims=True)[ok]
    model = 2.0 ** -24 * np.sqrt(d) * L_t * g
    need = np.maximum(err - 1e-6 - 1e-5 * g, 0.0) / np.maximum(model, 1e-300)
    big = g >= 1e-3
    return {"max_abs_err": float(err.max()) if err.size else 0.0,
            "max_rel_err_gates_ge_1e-3": float((err[big] / g[big]).max()) if big.any() else 0.0,
            "factor_needed_max": float(need.max()) if err.size else 0.0,
            "factor_needed_p99": float(np.quantile(need, 0.99)) if err.size else 0.0,
            "factor_needed_max_gates_ge_1e-3": float(need[big].max()) if big.any() else 0.0,
            "factor_allowed": 10.0}


def write_report(name: str, rep: dict) -> None:
    """parity_<name>.json under MOE_PARITY_REPORT_DIR (if set)."""
    out = os.environ.get("MOE_PARITY_REPORT_DIR")
    if not out:
        return
    os.makedirs(out, exist_ok=True)
    with open(os.path.join(out, f"parity_{name}.json"), "w") as f:
        json.dump({k: v for k, v in rep.items() if k != "gpu"}, f, indent=1, sort_keys=True)


def full_parity(x: S.LayerInputs, flags: int = 0, device="cuda:0"):
    """Every stage against the oracle, every token.  Returns a report."""
    wl = x.wl
    f = f64_inputs(x)
    gpu = gpu_stages(x, device, flags)
    assert gpu["status"] == 0
    bf16 = wl.dtype == S.DTYPE_BF16
    l = O.router_logits(f["u"], f["E"], None)
    if flags & L.MOE_FLAG_BIAS_SELECT_ONLY and f["bias"] is not None:
        key = O.softmax(l + f["bias"][None, :])
        gate_s = O.softmax(l)
        ref_idx, _ = O.topk_gates_select_only_bias(l, f["bias"], wl.top_k)
    else:
        key = O.softmax(l if f["bias"] is None else l + f["bias"][None, :])
        gate_s = key
        ref_idx = None
    lb = l if f["bias"] is None else l + f["bias"][None, :]
    near, mism = check_routing(gpu["idx"], gpu["w"], key, wl.top_k, ref_idx, gate_s, lb, wl.d)
    ref_sel = ref_idx if ref_idx is not None else O.topk_gates(key, wl.top_k)[0]
    mism_rows = np.any(gpu["idx"] != ref_sel, axis=1)
    check_dispatch(gpu, wl.n_routed)
    # FFN + combine evaluated by the oracle on the GPU's routing
    ref = O.layer_forward(f["u"], f["E"], f["bias"], f["W1"], f["W3"], f["W2"], f["W1_s"],
                          f["W3_s"], f["W2_s"], wl.top_k, idx=gpu["idx"])
    g = np.take_along_axis(gate_s, gpu["idx"].astype(np.int64), axis=1)
    ref_h = O.combine(f["u"], ref["y_shared"], ref["y"], g, ref["inv"], wl.top_k)
    ey = assert_close(gpu["y"], ref["y"], "y", bf16)
    esh = assert_close(gpu["ysh"], ref["y_shared"], "ysh", bf16)
    eh = assert_close(gpu["h"], ref_h, "h", bf16)
    fwd = check_forward(gpu, ref_h, O.topk_gap(key, wl.top_k) < TIE_GAP, bf16)
    rep = dict(workload=wl.name, tokens=int(wl.T), tokens_checked=int(wl.T), flags=int(flags),
               forward_path=PATH_NAMES[gpu["path"]],
               h_forward=fwd,
               near_ties=near, mismatches=mism, err_y=ey, err_ysh=esh, err_h=eh,
               h=error_stats(gpu["h"], ref_h, bf16), y=error_stats(gpu["y"], ref["y"], bf16),
               ysh=error_stats(gpu["ysh"], ref["y_shared"], bf16),
               gates=gate_stats(gpu["w"], gpu["idx"], gate_s, lb, wl.d, mism_rows),
               routing="idx/counts/offsets/perm/inv bit-exact on every token (near ties "
                       "counted)", gpu=gpu)
    if flags == 0:
        write_report(wl.name, rep)
    return rep


def sample_tokens(gpu: dict, K: int, n_random: int = 512, seed: int = 0) -> np.ndarray:
    """Random tokens plus every token of the most-loaded expert's first tile
    and of each expert's last partial 128-row tile."""
    T = gpu["idx"].shape[0]
    rng = np.random.default_rng(seed)
    picks = set(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    counts, offsets, perm = gpu["counts"], gpu["offsets"], gpu["perm"]
    e_max = int(np.argmax(counts))
    for p in range(offsets[e_max], min(offsets[e_max] + 128, offsets[e_max + 1])):
        picks.add(int(perm[p]) // K)
    for e in range(counts.size):
        c = int(counts[e])
        if c % 128:
            for p in range(offsets[e] + (c // 128) * 128, offsets[e + 1]):
                picks.add(int(perm[p]) // K)
    return np.array(sorted(picks), dtype=np.int64)


def sampled_parity(x: S.LayerInputs, device="cuda:0", n_random: int = 512):
    """Full-size check: routing and dispatch for every token, y and h on a
    sample of tokens (see sample_tokens)."""
    wl = x.wl
    f = f64_inputs(x)
    gpu = gpu_stages(x, device)
    assert gpu["status"] == 0
    l = O.router_logits(f["u"], f["E"], f["bias"])
    s = O.softmax(l)
    near, mism = check_routing(gpu["idx"], gpu["w"], s, wl.top_k, logits=l, d=wl.d)
    mism_rows = np.any(gpu["idx"] != O.topk_gates(s, wl.top_k)[0], axis=1)
    check_dispatch(gpu, wl.n_routed)
    toks = sample_tokens(gpu, wl.top_k, n_random)
    g = np.take_along_axis(s, gpu["idx"].astype(np.int64), axis=1)
    ref_h = O.layer_forward_tokens(f["u"], gpu["idx"], g, toks, f["W1"], f["W3"], f["W2"],
                                   f["W1_s"], f["W3_s"], f["W2_s"])
    eh = assert_close(gpu["h"][toks], ref_h, "h (sampled)")
    # shared output on the sample
    ref_sh = O.shared_experts(f["u"][toks], f["W1_s"], f["W3_s"], f["W2_s"])
    esh = assert_close(gpu["ysh"][toks], ref_sh, "ysh (sampled)")
    fwd = check_forward(gpu, ref_h, O.topk_gap(s, wl.top_k) < TIE_GAP, True, tokens=toks)
    rep = dict(workload=wl.name, tokens=int(wl.T), tokens_checked=int(toks.size), flags=0,
               forward_path=PATH_NAMES[gpu["path"]],
               h_forward=fwd,
               near_ties=near, mismatches=mism, err_h=eh, err_ysh=esh, sampled=int(toks.size),
               h=error_stats(gpu["h"][toks], ref_h), ysh=error_stats(gpu["ysh"][toks], ref_sh),
               gates=gate_stats(gpu["w"], gpu["idx"], s, l, wl.d, mism_rows),
               routing="idx/counts/offsets/perm/inv bit-exact on every token (near ties "
                       "counted); h and ysh on the sampled tokens",
               sample=f"{n_random} random tokens plus every token of the most-loaded expert's "
                      f"first 128 rows and of each expert's last partial 128-row tile",
               gpu=gpu)
    write_report(wl.name, rep)
    return rep
