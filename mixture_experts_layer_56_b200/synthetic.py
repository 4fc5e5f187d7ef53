"""Seeded synthetic inputs for the DeepSeekMoE layer forward.

This module is the one piece shared by the CUDA path, its tests and the CPU
oracle.  It draws numbers and encodes them; it holds none of the layer's
arithmetic (no logits, softmax, selection, FFN or combine).

Generator (counter based, so any element can be drawn on its own):

* splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): ``z = x + 0x9E3779B97F4A7C15``, then two
  xor-shift-multiply rounds and a final xor-shift.
* Element ``i`` of stream ``s`` under seed ``seed`` hashes the counter
  ``key(seed, s) + i`` where ``key = splitmix64((seed << 32) | s)``.
* Box-Muller (1958) on the two 32-bit halves of that hash:
  ``u1 = (hi + 1) / 2^32`` in (0, 1], ``u2 = lo / 2^32`` in [0, 1),
  ``z = sqrt(-2 ln u1) * cos(2 pi u2)``: one standard normal per counter.
* A value is ``float32(std * z)``; bf16 tensors are that float32 rounded to
  bfloat16 with round-to-nearest-even, kept as raw ``uint16`` bits.

Workloads are the layer shapes the DeepSeekMoE pages discuss (fine-grained
routed experts plus shared experts, every expert a SwiGLU FFN), with the
initialisations stated in each ``Workload``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# stream ids, one per tensor, so that a tensor's values do not depend on the
# sizes of the tensors drawn before it
STREAM = {"u": 1, "E": 2, "bias": 3, "W1": 4, "W3": 5, "W2": 6,
          "W1_s": 7, "W3_s": 8, "W2_s": 9}

DTYPE_F32 = "f32"
DTYPE_BF16 = "bf16"


def splitmix64(x: np.ndarray) -> np.ndarray:
    """splitmix64 output function applied elementwise to uint64 counters."""
    with np.errstate(over="ignore"):
        z = x + _GOLDEN_GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _stream_key(seed: int, stream: int) -> np.uint64:
    base = np.array([(np.uint64(seed) << np.uint64(32)) | np.uint64(stream)],
                    dtype=np.uint64)
    return splitmix64(base)[0]


def _normal_chunk(key: np.uint64, start: int, n: int) -> np.ndarray:
    ctr = np.arange(start, start + n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        h = splitmix64(ctr + key)
    hi = (h >> np.uint64(32)).astype(np.float64)
    lo = (h & np.uint64(0xFFFFFFFF)).astype(np.float64)
    u1 = (hi + 1.0) * (1.0 / 4294967296.0)
    u2 = lo * (1.0 / 4294967296.0)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def standard_normal(seed: int, stream: int, n: int, start: int = 0,
                    threads: int = 8) -> np.ndarray:
    """``n`` standard normals (float64) for counters ``start .. start+n-1``."""
    key = _stream_key(seed, stream)
    chunk = 1 << 22
    if n <= chunk:
        return _normal_chunk(key, start, n)
    out = np.empty(n, dtype=np.float64)

    def work(off):
        m = min(chunk, n - off)
        out[off:off + m] = _normal_chunk(key, start + off, m)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(work, range(0, n, chunk)))
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    nan = (b & np.uint32(0x7FFFFFFF)) > np.uint32(0x7F800000)
    rounded = np.where(nan, (b >> np.uint32(16)) | np.uint32(0x40), rounded)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float32."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


@dataclass(frozen=True)
class Workload:
    """One layer shape plus its initialisation recipe.

    ``n_routed`` is mN - K_s, ``top_k`` is mK - K_s, ``n_shared`` is K_s and
    ``inter`` is the intermediate width of one fine-grained expert.
    Standard deviations are square roots of the stated variances.
    """
    name: str
    T: int
    d: int
    n_routed: int
    n_shared: int
    inter: int
    top_k: int
    dtype: str = DTYPE_BF16
    bias_var: float = 0.0          # router bias b_i ~ N(0, bias_var); 0 = no bias
    zipf_s: float = 0.0            # router row norms scaled by Zipf(s); 0 = off
    w2_var: float | None = None    # W2 variance; None = 1/fan_in = 1/inter
    seed: int = 0
    note: str = ""

    @property
    def has_bias(self) -> bool:
        return self.bias_var > 0.0

    def expert_flops(self) -> float:
        """Algorithmic FLOPs of the expert FFNs: T*(K+K_s)*6*d*I."""
        return float(self.T) * (self.top_k + self.n_shared) * 6.0 * self.d * self.inter

    def router_flops(self) -> float:
        return 2.0 * self.T * self.d * self.n_routed


WORKLOADS = {
    "tiny": Workload("tiny", T=64, d=128, n_routed=16, n_shared=1, inter=64,
                     top_k=4, dtype=DTYPE_F32, w2_var=1.0 / 64,
                     note="fp32 correctness layer"),
    "small": Workload("small", T=8192, d=1280, n_routed=63, n_shared=1,
                      inter=896, top_k=7,
                      note="small-model-shaped layer, uniform-ish routing"),
    "16b": Workload("16b", T=16384, d=2048, n_routed=64, n_shared=2,
                    inter=1408, top_k=6, bias_var=0.5,
                    note="16B-shaped prefill, router bias skews loads"),
    "large": Workload("large", T=32768, d=4096, n_routed=128, n_shared=4,
                      inter=1536, top_k=12, zipf_s=1.1,
                      note="large-shaped layer, Zipf(1.1) router norms"),
}
for _t in (1, 8, 32, 128):
    WORKLOADS[f"decode{_t}"] = Workload(
        f"decode{_t}", T=_t, d=2048, n_routed=64, n_shared=2, inter=1408,
        top_k=6, bias_var=0.5, note="16B-shaped decode step")


def custom_workload(name, T, d, n_routed, n_shared, inter, top_k,
                  dtype=DTYPE_BF16, bias_var=0.0, zipf_s=0.0, seed=0):
    return Workload(name, T=T, d=d, n_routed=n_routed, n_shared=n_shared,
                    inter=inter, top_k=top_k, dtype=dtype, bias_var=bias_var,
                    zipf_s=zipf_s, seed=seed)


@dataclass
class LayerInputs:
    """Raw inputs of one layer.  bf16 tensors are uint16 bit arrays, fp32
    tensors float32 arrays.  Weight layouts follow the method's notation:
    W1/W3 are [n, I, d] (x -> W x), W2 is [n, d, I]."""
    wl: Workload
    u: np.ndarray
    E: np.ndarray
    bias: np.ndarray | None
    W1: np.ndarray
    W3: np.ndarray
    W2: np.ndarray
    W1_s: np.ndarray
    W3_s: np.ndarray
    W2_s: np.ndarray
    extras: dict = field(default_factory=dict)

    def as_f64(self, name: str) -> np.ndarray:
        """The exact input values widened to float64."""
        a = getattr(self, name)
        if a is None:
            return None
        if a.dtype == np.uint16:
            return bf16_bits_to_f32(a).astype(np.float64)
        return a.astype(np.float64)


def _encode(x64: np.ndarray, dtype: str) -> np.ndarray:
    x32 = x64.astype(np.float32)
    return x32 if dtype == DTYPE_F32 else f32_to_bf16_bits(x32)


def _draw(wl: Workload, name: str, shape, std: float) -> np.ndarray:
    n = int(np.prod(shape)) if len(shape) else 1
    z = standard_normal(wl.seed, STREAM[name], n)
    return _encode(std * z, wl.dtype).reshape(shape)


def zipf_row_scale(n: int, s: float) -> np.ndarray:
    """c_i = (i+1)^-s / mean_j (j+1)^-s: Zipf-shaped norms with mean 1."""
    r = np.arange(1, n + 1, dtype=np.float64) ** (-s)
    return r / r.mean()


def make_inputs(wl: Workload) -> LayerInputs:
    """Draw every input of ``wl`` in the fixed order u, E, bias, W1, W3, W2,
    W1_s, W3_s, W2_s (each from its own stream)."""
    T, d, n, ns, I = wl.T, wl.d, wl.n_routed, wl.n_shared, wl.inter
    u = _draw(wl, "u", (T, d), 1.0)
    zE = standard_normal(wl.seed, STREAM["E"], n * d).reshape(n, d) / math.sqrt(d)
    if wl.zipf_s > 0:
        zE = zE * zipf_row_scale(n, wl.zipf_s)[:, None]
    E = _encode(zE, wl.dtype)
    bias = None
    if wl.has_bias:
        # the router bias is float32 for every dtype
        bias = (math.sqrt(wl.bias_var)
                * standard_normal(wl.seed, STREAM["bias"], n)).astype(np.float32)
    w13_std = 1.0 / math.sqrt(d)
    w2_std = math.sqrt(wl.w2_var) if wl.w2_var is not None else 1.0 / math.sqrt(I)
    W1 = _draw(wl, "W1", (n, I, d), w13_std)
    W3 = _draw(wl, "W3", (n, I, d), w13_std)
    W2 = _draw(wl, "W2", (n, d, I), w2_std)
    W1_s = _draw(wl, "W1_s", (ns, I, d), w13_std)
    W3_s = _draw(wl, "W3_s", (ns, I, d), w13_std)
    W2_s = _draw(wl, "W2_s", (ns, d, I), w2_std)
    return LayerInputs(wl, u, E, bias, W1, W3, W2, W1_s, W3_s, W2_s)
