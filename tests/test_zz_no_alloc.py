"""moe_dispatch_static_scratch (fixed in-library scratch, no allocation)
against moe_dispatch (caller workspace) through the C ABI: integer outputs,
so the bar is bit-exact.  Collected last so that it also runs after every
other GPU test in the same process; it passes alone as well."""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_layer_56_b200 import _lib as L

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    yield


def _routing(T, n, K, seed):
    """Seeded routing indices: K distinct experts per token, a skewed
    preference so that counts differ across experts and some stay empty."""
    rng = np.random.default_rng(seed)
    pref = rng.standard_normal(n) * 1.5
    keys = rng.standard_normal((T, n)) + pref[None, :]
    return np.argsort(-keys, axis=1, kind="stable")[:, :K].astype(np.int32)


def _outputs(T, n, K):
    z = lambda m: torch.full((m,), -7, dtype=torch.int32, device=DEV)  # noqa: E731
    return dict(counts=z(n), offsets=z(n + 1), perm=z(max(T * K, 1)), inv=z(max(T * K, 1)))


def _with_workspace(shape, idx, T, n, K):
    o = _outputs(T, n, K)
    ws = torch.empty(L.moe_workspace_size(shape), dtype=torch.uint8, device=DEV)
    L.moe_dispatch(shape, idx, o["counts"], o["offsets"], o["perm"], o["inv"], ws)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in o.items()}


def _static(shape, idx, o):
    for v in o.values():
        v.fill_(-7)
    torch.cuda.synchronize()
    rc = L.lib().moe_dispatch_static_scratch(
        ctypes.byref(shape), idx.data_ptr(), o["counts"].data_ptr(), o["offsets"].data_ptr(),
        o["perm"].data_ptr(), o["inv"].data_ptr(), None)
    assert rc == L.MOE_OK, L.strerror(rc)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in o.items()}


# (T, n_routed, K): one block, several chunks with a ragged tail, the
# 16B-expert shape, and the largest T the fixed scratch takes at 256 experts
SHAPES = [(100, 64, 6), (5000, 64, 6), (8192, 63, 7), (32768, 256, 8)]


@pytest.mark.parametrize("T,n,K", SHAPES)
def test_static_scratch_dispatch_matches_workspace_dispatch_twice(T, n, K):
    shape = L.make_shape(T, 256, n, 1, 128, K)
    idx = torch.from_numpy(_routing(T, n, K, seed=T + n)).to(DEV)
    ref = _with_workspace(shape, idx, T, n, K)
    o = _outputs(T, n, K)
    for _ in range(2):  # two calls in a row on the same shared scratch
        got = _static(shape, idx, o)
        for k in ref:
            assert np.array_equal(got[k], ref[k]), k


def test_static_scratch_reused_across_shapes_without_allocating():
    """A large call leaves the scratch full of its values; a smaller call
    after it must not depend on them.  Device free memory stays unchanged
    across the calls once set up."""
    big = (20000, 128, 8)
    small = (3000, 32, 3)
    cases = []
    for T, n, K in (big, small, big):
        shape = L.make_shape(T, 256, n, 1, 128, K)
        idx = torch.from_numpy(_routing(T, n, K, seed=7 * T + n)).to(DEV)
        cases.append((shape, idx, _with_workspace(shape, idx, T, n, K), _outputs(T, n, K)))
    torch.cuda.synchronize()
    _static(cases[0][0], cases[0][1], cases[0][3])  # set-up on this device
    free_before, _ = torch.cuda.mem_get_info()
    for shape, idx, ref, o in cases:
        got = _static(shape, idx, o)
        for k in ref:
            assert np.array_equal(got[k], ref[k]), k
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before


def test_static_scratch_rejects_shapes_beyond_its_size():
    T, n, K = 32769, 256, 8  # one chunk more than fits at 256 experts
    shape = L.make_shape(T, 256, n, 1, 128, K)
    idx = torch.zeros(T * K, dtype=torch.int32, device=DEV)
    o = _outputs(T, n, K)
    before = L.moe_launch_count()
    rc = L.lib().moe_dispatch_static_scratch(
        ctypes.byref(shape), idx.data_ptr(), o["counts"].data_ptr(), o["offsets"].data_ptr(),
        o["perm"].data_ptr(), o["inv"].data_ptr(), None)
    assert rc == L.MOE_ERR_SCRATCH_LIMIT
    assert L.moe_launch_count() == before
    assert "scratch" in L.strerror(rc)
