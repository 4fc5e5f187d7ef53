"""Failure detection on the GPU without a fault: every wait of the tensor-core
kernels is bounded.  MOE_FLAG_INJECT_WAIT_TIMEOUT plants one wait that nothing
satisfies (the GEMMs' TMA producer waits for a shared-memory slot that is
never released, with a 1 ms limit).  The kernels must give up, record
MOE_ERR_DEVICE_CHECK in the workspace status word and return; the context
must stay usable, so that the next normal forward matches the oracle."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_56_b200 import _lib as L
from mixture_experts_layer_56_b200 import synthetic as S
from mixture_experts_layer_56_b200.layer import MoELayer, to_device
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    yield


MODES = {"single_cta": L.MOE_FLAG_GEMM_SINGLE_CTA, "cta_pair": L.MOE_FLAG_GEMM_CTA_PAIR}


@pytest.mark.parametrize("mode", sorted(MODES))
def test_expired_wait_sets_status_and_context_survives(mode):
    wl = S.custom_workload("stall", T=300, d=256, n_routed=16, n_shared=2, inter=128, top_k=4)
    x = S.make_inputs(wl)
    layer = MoELayer(x, "cuda:0", flags=MODES[mode] | L.MOE_FLAG_INJECT_WAIT_TIMEOUT)
    u = to_device(x.u, "cuda:0")
    assert layer.status() == L.MOE_OK
    layer.forward(u)                      # launches return; the kernels give up
    torch.cuda.synchronize()              # and finish: no hang, no fault
    assert layer.status() == L.MOE_ERR_DEVICE_CHECK
    assert layer.status() == L.MOE_OK     # reading the word cleared it
    # the same context, the same workspace: a normal forward is correct
    rep = P.full_parity(x, flags=MODES[mode])
    assert rep["gpu"]["status"] == L.MOE_OK
    good = MoELayer(x, "cuda:0", flags=MODES[mode])
    good.ws.copy_(layer.ws)               # the workspace the failed call left behind
    h = good.forward(u)
    torch.cuda.synchronize()
    assert good.status() == L.MOE_OK
    h_ref = rep["gpu"]["h_fwd_raw"]
    assert np.array_equal(P.to_numpy(h), h_ref)
