"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (moe_layer_forward on one GPU): the small-model layer in full,
the 16B-shaped prefill and decode layers and the large layer with routing and
dispatch checked for every token and the outputs on sampled tokens."""
import dataclasses

import numpy as np
import pytest
import torch

from mixture_experts_layer_56_b200 import synthetic as S
from tests import parity as P

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    yield


@pytest.fixture(scope="module")
def inputs_16b():
    return S.make_inputs(S.WORKLOADS["16b"])


def test_small_layer_every_token():
    rep = P.full_parity(S.make_inputs(S.WORKLOADS["small"]))
    print("small", {k: v for k, v in rep.items() if k != "gpu"})


def test_16b_prefill_sampled(inputs_16b):
    rep = P.sampled_parity(inputs_16b)
    counts = rep["gpu"]["counts"]
    # the router bias skews the loads
    assert counts.max() > 2 * counts.mean()
    print("16b", {k: v for k, v in rep.items() if k != "gpu"})


@pytest.mark.parametrize("T", [1, 8, 32, 128])
def test_16b_decode_every_token(inputs_16b, T):
    wl = S.WORKLOADS[f"decode{T}"]
    x = dataclasses.replace(inputs_16b, wl=wl, u=inputs_16b.u[:T])
    rep = P.full_parity(x)
    print(f"decode{T}", {k: v for k, v in rep.items() if k != "gpu"})


def test_large_layer_sampled():
    x = S.make_inputs(S.WORKLOADS["large"])
    rep = P.sampled_parity(x, n_random=256)
    counts = rep["gpu"]["counts"]
    assert counts.max() > 4 * counts.mean()  # Zipf router norms: heavy imbalance
    print("large", {k: v for k, v in rep.items() if k != "gpu"})
