"""A DeepSeekMoE layer held on one GPU, calling libmoe through its C ABI.

``MoELayer`` owns the device copies of the router centroids, the optional
router bias and the expert weights (W13 packed once by ``moe_pack_w13``) plus
the workspace, and runs ``moe_layer_forward`` on torch's current stream.
torch provides device memory and streams only; every step of the layer runs
in libmoe's kernels.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as L
from .synthetic import DTYPE_BF16, LayerInputs, Workload


def to_device(a: np.ndarray | None, device) -> torch.Tensor | None:
    """numpy array (uint16 = bf16 bits, float32, int32) -> device tensor."""
    if a is None:
        return None
    if a.dtype == np.uint16:
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device, non_blocking=False)


def to_numpy(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def shape_of(wl: Workload, T: int | None = None, flags: int = 0) -> L.MoeShape:
    return L.make_shape(wl.T if T is None else T, wl.d, wl.n_routed, wl.n_shared, wl.inter,
                        wl.top_k, L.MOE_DTYPE_BF16 if wl.dtype == DTYPE_BF16 else L.MOE_DTYPE_F32,
                        flags)


class MoELayer:
    """Device-resident weights of one layer plus its workspace."""

    def __init__(self, inputs: LayerInputs, device="cuda:0", flags: int = 0,
                 max_tokens: int | None = None, host_io: bool = False):
        wl = inputs.wl
        self.wl = wl
        self.device = torch.device(device)
        self.flags = flags
        self.max_tokens = wl.T if max_tokens is None else max_tokens
        self.shape = shape_of(wl, self.max_tokens, flags)
        dev = self.device
        self.E = to_device(inputs.E, dev)
        self.bias = to_device(inputs.bias, dev)
        self.W2 = to_device(inputs.W2, dev)
        self.W2_s = to_device(inputs.W2_s, dev) if wl.n_shared > 0 else None
        self.W13 = self._pack(inputs.W1, inputs.W3, wl.n_routed)
        self.W13_s = self._pack(inputs.W1_s, inputs.W3_s, wl.n_shared) if wl.n_shared > 0 else None
        nbytes = (L.moe_workspace_size_host(self.shape) if host_io
                  else L.moe_workspace_size(self.shape))
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)

    @property
    def elem_dtype(self):
        return torch.bfloat16 if self.wl.dtype == DTYPE_BF16 else torch.float32

    def _pack(self, W1: np.ndarray, W3: np.ndarray, n: int) -> torch.Tensor:
        w1 = to_device(W1, self.device)
        w3 = to_device(W3, self.device)
        out = torch.empty((n, 2 * self.wl.inter, self.wl.d), dtype=w1.dtype, device=self.device)
        L.moe_pack_w13(self.shape, n, w1, w3, out)
        return out

    def shape_for(self, T: int) -> L.MoeShape:
        return shape_of(self.wl, T, self.flags)

    def forward(self, u: torch.Tensor, h: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        T = u.shape[0]
        assert T <= self.max_tokens
        if h is None:
            h = torch.empty_like(u)
        L.moe_layer_forward(self.shape_for(T), u, self.E, self.bias, self.W13, self.W2,
                            self.W13_s, self.W2_s, h, self.ws, stream=stream)
        return h

    def forward_host(self, u_host: torch.Tensor, h_host: torch.Tensor, stream=None) -> torch.Tensor:
        """u and h in (pinned) host memory; copies run inside the call."""
        T = u_host.shape[0]
        L.moe_layer_forward_host(self.shape_for(T), u_host, self.E, self.bias, self.W13,
                                 self.W2, self.W13_s, self.W2_s, h_host, self.ws, stream=stream)
        return h_host

    def status(self) -> int:
        return L.moe_read_status(self.ws)
