"""GPU parity: every stage of the layer through the C ABI against the CPU
oracle on the same seeded inputs (bars in tests/parity.py)."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_56_b200 import _lib as L
from mixture_experts_layer_56_b200 import synthetic as S
from mixture_experts_layer_56_b200.layer import MoELayer, to_device, to_numpy
from tests import parity as P

pytestmark = pytest.mark.gpu

W = S.custom_workload


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    yield


# (name, workload) -- each spans several 128-row tiles plus a ragged tail and
# exercises one tile width of the tensor-core path
CASES = [
    W("tiles_bn256", T=300, d=256, n_routed=16, n_shared=2, inter=128, top_k=4),
    W("ragged_bn128_bias", T=1000, d=384, n_routed=20, n_shared=1, inter=192, top_k=6,
      bias_var=0.5),
    W("noshared_bn64", T=517, d=320, n_routed=63, n_shared=0, inter=64, top_k=7),
    W("zipf_router", T=777, d=512, n_routed=40, n_shared=3, inter=128, top_k=5, zipf_s=1.1),
    # every width a multiple of 512: CTA pairs take 256 x 512 tiles
    W("wide_tiles", T=1100, d=512, n_routed=12, n_shared=2, inter=256, top_k=3),
    W("wide_ragged", T=333, d=1024, n_routed=5, n_shared=1, inter=512, top_k=2, bias_var=0.5),
    # widths 512 j + 256 (d = 768, 1280): CTA pairs take 256-column tiles; in
    # pair_mixed the shared gate/up group alone is a multiple of 512 wide
    W("pair_odd256", T=700, d=768, n_routed=6, n_shared=1, inter=384, top_k=2),
    W("pair_mixed", T=600, d=1280, n_routed=10, n_shared=2, inter=640, top_k=3, bias_var=0.5),
]


def test_tiny_fp32_config_full():
    rep = P.full_parity(S.make_inputs(S.WORKLOADS["tiny"]))
    print(rep["near_ties"], rep["err_h"])


GEMM_MODES = {"single_cta": L.MOE_FLAG_GEMM_SINGLE_CTA, "cta_pair": L.MOE_FLAG_GEMM_CTA_PAIR,
              "cta_pair_narrow": L.MOE_FLAG_GEMM_CTA_PAIR | L.MOE_FLAG_GEMM_NARROW}


@pytest.mark.parametrize("mode", sorted(GEMM_MODES))
@pytest.mark.parametrize("wl", CASES, ids=[c.name for c in CASES])
def test_bf16_cases_full(wl, mode):
    rep = P.full_parity(S.make_inputs(wl), flags=GEMM_MODES[mode])
    print(wl.name, mode, {k: v for k, v in rep.items() if k != "gpu"})


@pytest.mark.parametrize("d,inter", [(512, 256), (768, 384)], ids=["w512", "w768"])
@pytest.mark.parametrize("mode", sorted(GEMM_MODES))
def test_gemm_tile_modes_agree(mode, d, inter):
    """Both tile shapes give results within the bf16 bar of each other and
    the same routing (the routing does not depend on the GEMM)."""
    wl = W("modes", T=900, d=d, n_routed=8, n_shared=1, inter=inter, top_k=2)
    x = S.make_inputs(wl)
    a = P.gpu_stages(x, flags=GEMM_MODES[mode])
    b = P.gpu_stages(x, flags=0)
    assert np.array_equal(a["idx"], b["idx"])
    P.assert_close(a["h"], b["h"], "h across tile modes")


def test_every_expert_selected_sums_gates_to_one():
    """K = N_r: every token uses every routed expert; gates sum to 1."""
    wl = W("k_equals_n", T=130, d=128, n_routed=8, n_shared=1, inter=64, top_k=8)
    rep = P.full_parity(S.make_inputs(wl))
    w = rep["gpu"]["w"].astype(np.float64)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-5)
    assert np.all(rep["gpu"]["counts"] == 130)


def test_empty_experts_from_skewed_bias():
    """A strong router bias leaves most experts without tokens."""
    wl = W("skewed", T=400, d=128, n_routed=32, n_shared=1, inter=64, top_k=2, bias_var=100.0)
    rep = P.full_parity(S.make_inputs(wl))
    assert np.sum(rep["gpu"]["counts"] == 0) >= 8


@pytest.mark.parametrize("mode", sorted(GEMM_MODES))
@pytest.mark.parametrize("T", [1, 2, 127, 128, 129, 255, 256, 257])
def test_token_counts_around_one_tile(T, mode):
    wl = W(f"t{T}", T=T, d=256, n_routed=4, n_shared=1, inter=128, top_k=2)
    P.full_parity(S.make_inputs(wl), flags=GEMM_MODES[mode])


def test_duplicate_centroids_lower_index_wins():
    wl = W("dups", T=512, d=256, n_routed=16, n_shared=1, inter=64, top_k=4)
    x = S.make_inputs(wl)
    x.E[9] = x.E[2]
    x.E[13] = x.E[2]
    rep = P.full_parity(x)
    idx = rep["gpu"]["idx"]
    for t in range(wl.T):
        row = idx[t].tolist()
        for dup in (9, 13):
            if dup in row:
                assert 2 in row and row.index(2) < row.index(dup)
    # logits of duplicates are equal, so 9 can only appear when 2 did
    assert any(2 in r for r in idx.tolist())


def test_select_only_bias_flag():
    wl = W("selbias", T=600, d=256, n_routed=24, n_shared=1, inter=128, top_k=4, bias_var=1.0)
    P.full_parity(S.make_inputs(wl), flags=L.MOE_FLAG_BIAS_SELECT_ONLY)


def test_zero_tokens_launch_nothing():
    wl = W("t0", T=0, d=256, n_routed=16, n_shared=1, inter=128, top_k=4)
    sh = L.make_shape(0, 256, 16, 1, 128, 4)
    before = L.moe_launch_count()
    assert L.lib().moe_layer_forward(sh, *([None] * 9), 0, None) == 0
    assert L.moe_launch_count() == before


def test_forward_is_bitwise_deterministic():
    wl = W("det", T=700, d=256, n_routed=32, n_shared=2, inter=128, top_k=6)
    x = S.make_inputs(wl)
    layer = MoELayer(x)
    u = to_device(x.u, "cuda:0")
    a = to_numpy(layer.forward(u))
    b = to_numpy(layer.forward(u))
    assert np.array_equal(a, b)


def test_host_io_entry_point_matches_device_path():
    wl = W("hostio", T=333, d=256, n_routed=16, n_shared=1, inter=128, top_k=4)
    x = S.make_inputs(wl)
    layer = MoELayer(x, host_io=True)
    u = to_device(x.u, "cuda:0")
    ref = to_numpy(layer.forward(u))
    u_h = u.cpu().pin_memory()
    h_h = torch.empty_like(u_h).pin_memory()
    layer.forward_host(u_h, h_h)
    assert np.array_equal(to_numpy(h_h), ref)


def test_expert_balance_statistics():
    """§3.3 eqs. (12)-(13) from the router's scores and the dispatch counts."""
    from oracle import moe_oracle as O
    wl = W("bal", T=1000, d=256, n_routed=24, n_shared=1, inter=64, top_k=4, bias_var=0.3)
    x = S.make_inputs(wl)
    rep = P.full_parity(x)
    layer = rep["gpu"]["layer"]
    dev = layer.device
    counts = to_device(rep["gpu"]["counts"], dev)
    f = torch.empty(24, dtype=torch.float32, device=dev)
    Pm = torch.empty(24, dtype=torch.float32, device=dev)
    L.moe_expert_balance(layer.shape, to_device(x.u, dev), layer.E, layer.bias, counts, f, Pm,
                         layer.ws)
    torch.cuda.synchronize()
    fx = P.f64_inputs(x)
    s = O.softmax(O.router_logits(fx["u"], fx["E"], fx["bias"]))
    f_ref, P_ref, _ = O.expert_balance(s, rep["gpu"]["idx"])
    np.testing.assert_allclose(to_numpy(f), f_ref, rtol=1e-6)
    np.testing.assert_allclose(to_numpy(Pm), P_ref, rtol=1e-4, atol=1e-7)
    np.testing.assert_allclose(to_numpy(f).sum(), 24.0, rtol=1e-5)


@pytest.mark.parametrize("wl", CASES[:3], ids=[c.name for c in CASES[:3]])
def test_simt_router_full(wl):
    """The CUDA-core router (MOE_FLAG_ROUTER_SIMT) meets the same bars."""
    P.full_parity(S.make_inputs(wl), flags=L.MOE_FLAG_ROUTER_SIMT)


# expert counts that reach every epilogue variant of the tensor-core router:
# 1, 2, 3 and 4 register chunks, and the chunked path (256 experts, or
# select-only bias beyond 64 experts), with and without the cluster split
ROUTER_CASES = CASES + [
    W("router_90", T=300, d=256, n_routed=90, n_shared=1, inter=64, top_k=6, bias_var=0.5),
    W("router_128", T=300, d=256, n_routed=128, n_shared=1, inter=64, top_k=12),
    W("router_256", T=300, d=256, n_routed=256, n_shared=1, inter=64, top_k=8),
    # more than 16 tiles of 128 tokens: one CTA per tile (no cluster split)
    W("router_t2200_n40", T=2200, d=256, n_routed=40, n_shared=1, inter=64, top_k=5),
    W("router_t2200_n256", T=2200, d=256, n_routed=256, n_shared=1, inter=64, top_k=8),
]
ROUTER_FLAGS = {"bias_in_softmax": 0, "bias_select_only": L.MOE_FLAG_BIAS_SELECT_ONLY}


@pytest.mark.parametrize("bias_mode", sorted(ROUTER_FLAGS))
@pytest.mark.parametrize("wl", ROUTER_CASES, ids=[c.name for c in ROUTER_CASES])
def test_tensor_core_and_simt_routers_agree(wl, bias_mode):
    """Both routers compute the same logits up to fp32 summation order: the
    same experts for every token without a near tie in the oracle's scores,
    gates within the fp32 gate bar."""
    from oracle import moe_oracle as O
    if bias_mode == "bias_select_only" and wl.bias_var == 0:
        wl = S.custom_workload(wl.name + "_b", T=wl.T, d=wl.d, n_routed=wl.n_routed,
                               n_shared=wl.n_shared, inter=wl.inter, top_k=wl.top_k, bias_var=0.5)
    x = S.make_inputs(wl)
    layer = MoELayer(x, "cuda:0")
    u = to_device(x.u, "cuda:0")
    bf = ROUTER_FLAGS[bias_mode]
    out = {}
    for name, fl in (("tc", bf), ("simt", bf | L.MOE_FLAG_ROUTER_SIMT)):
        sh = L.make_shape(wl.T, wl.d, wl.n_routed, wl.n_shared, wl.inter, wl.top_k, flags=fl)
        idx = torch.full((wl.T, wl.top_k), -1, dtype=torch.int32, device="cuda:0")
        w = torch.full((wl.T, wl.top_k), -1.0, dtype=torch.float32, device="cuda:0")
        L.moe_route(sh, u, layer.E, layer.bias, idx, w)
        torch.cuda.synchronize()
        out[name] = (to_numpy(idx), to_numpy(w))
    fx = P.f64_inputs(x)
    s = O.softmax(O.router_logits(fx["u"], fx["E"], fx["bias"]))
    near = P.near_tie_tokens(s, wl.top_k)
    if bias_mode == "bias_select_only":
        ref_idx, _ = O.topk_gates_select_only_bias(O.router_logits(fx["u"], fx["E"], None),
                                                   fx["bias"], wl.top_k)
        assert np.all((out["tc"][0] == ref_idx).all(axis=1) | near)
    same = np.all(out["tc"][0] == out["simt"][0], axis=1)
    assert np.all(same | near)
    ok = same & ~near
    np.testing.assert_allclose(out["tc"][1][ok], out["simt"][1][ok], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("n", [24, 90, 200])
def test_balance_statistics_every_router_variant(n):
    """Eqs. (12)-(13) through the statistics variants of the router
    (register-resident up to 64 experts, chunked beyond)."""
    from oracle import moe_oracle as O
    wl = W(f"bal{n}", T=700, d=256, n_routed=n, n_shared=1, inter=64, top_k=4, bias_var=0.3)
    x = S.make_inputs(wl)
    rep = P.full_parity(x)
    layer = rep["gpu"]["layer"]
    dev = layer.device
    counts = to_device(rep["gpu"]["counts"], dev)
    f = torch.empty(n, dtype=torch.float32, device=dev)
    Pm = torch.empty(n, dtype=torch.float32, device=dev)
    L.moe_expert_balance(layer.shape, to_device(x.u, dev), layer.E, layer.bias, counts, f, Pm,
                         layer.ws)
    torch.cuda.synchronize()
    fx = P.f64_inputs(x)
    s = O.softmax(O.router_logits(fx["u"], fx["E"], fx["bias"]))
    f_ref, P_ref, _ = O.expert_balance(s, rep["gpu"]["idx"])
    np.testing.assert_allclose(to_numpy(f), f_ref, rtol=1e-6)
    np.testing.assert_allclose(to_numpy(Pm), P_ref, rtol=1e-4, atol=1e-7)


def test_forward_replays_from_a_cuda_graph_bitwise():
    """moe_layer_forward only enqueues work on the caller's stream: captured
    into a CUDA graph (its kernels keep programmatic dependent launch), each
    replay gives the eager result bit for bit, also after the input changes."""
    wl = W("graph", T=600, d=256, n_routed=24, n_shared=1, inter=128, top_k=4)
    x = S.make_inputs(wl)
    layer = MoELayer(x)
    u = to_device(x.u, "cuda:0")
    h = torch.empty_like(u)

    def fwd():
        L.moe_layer_forward(layer.shape, u, layer.E, layer.bias, layer.W13, layer.W2,
                            layer.W13_s, layer.W2_s, h, layer.ws,
                            stream=torch.cuda.current_stream())

    fwd()
    torch.cuda.synchronize()
    ref = to_numpy(h).copy()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    for _ in range(3):
        h.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(to_numpy(h), ref)
    u.copy_(torch.flip(u, dims=[0]))  # new tokens in the same buffer
    g.replay()
    torch.cuda.synchronize()
    ref2 = to_numpy(h).copy()
    fwd()
    torch.cuda.synchronize()
    assert np.array_equal(to_numpy(h), ref2)
    assert not np.array_equal(ref, ref2)
    assert layer.status() == 0


def test_half_activated_small_shapes():
    """Half-activated variant (§4.5, Figs. 5-6): the small layer's shapes with about half
    the routed experts per token (K = 3 instead of 7), same kernels."""
    wl = W("half_activated", T=1500, d=1280, n_routed=63, n_shared=1, inter=896, top_k=3)
    rep = P.full_parity(S.make_inputs(wl))
    assert rep["gpu"]["counts"].sum() == 1500 * 3


def test_host_io_chunked_pipeline_matches_device_path():
    """Above 4352 tokens the host-buffer call runs in chunks whose copies
    overlap the forward; h still equals the one-pass device forward bit for
    bit (same GEMM tile mode for every chunk, no router cluster split)."""
    for T in (4400, 9000):
        wl = W(f"hostio{T}", T=T, d=256, n_routed=16, n_shared=1, inter=128, top_k=4)
        x = S.make_inputs(wl)
        layer = MoELayer(x, host_io=True)
        u = to_device(x.u, "cuda:0")
        ref = to_numpy(layer.forward(u))
        u_h = u.cpu().pin_memory()
        h_h = torch.empty_like(u_h).pin_memory()
        for _ in range(2):
            h_h.zero_()
            layer.forward_host(u_h, h_h)
            assert np.array_equal(to_numpy(h_h), ref)
        assert layer.status() == 0


# Decode-sized batches run the whole layer as one kernel (moe_forward_path):
# every hidden size it takes, with and without shared experts, a router
# bias, the selection-only bias, K up to 16 and up to 256 routed experts.
DECODE_CASES = [
    W("dec_d256", T=1, d=256, n_routed=16, n_shared=1, inter=128, top_k=4),
    W("dec_d512_t8", T=8, d=512, n_routed=64, n_shared=2, inter=192, top_k=6, bias_var=0.5),
    W("dec_d1024_noshared", T=5, d=1024, n_routed=32, n_shared=0, inter=256, top_k=3),
    W("dec_d2048_k16", T=3, d=2048, n_routed=256, n_shared=1, inter=64, top_k=16, bias_var=4.0),
    W("dec_d256_t7", T=7, d=256, n_routed=8, n_shared=4, inter=320, top_k=8),
    W("dec_d1024_t16", T=16, d=1024, n_routed=40, n_shared=2, inter=128, top_k=6),
    W("dec_d2048_t13", T=13, d=2048, n_routed=64, n_shared=2, inter=192, top_k=6, bias_var=0.5),
]


@pytest.mark.parametrize("wl", DECODE_CASES, ids=[c.name for c in DECODE_CASES])
def test_decode_layer_kernel(wl):
    x = S.make_inputs(wl)
    layer = MoELayer(x)
    assert L.moe_forward_path(layer.shape) == L.MOE_PATH_DECODE_LAYER
    rep = P.full_parity(x)
    assert rep["h_forward"] is not None
    print(wl.name, rep["h_forward"])


def test_decode_layer_kernel_select_only_bias_and_repeat():
    wl = W("dec_sel", T=6, d=512, n_routed=24, n_shared=1, inter=128, top_k=4, bias_var=1.0)
    x = S.make_inputs(wl)
    rep = P.full_parity(x, flags=L.MOE_FLAG_BIAS_SELECT_ONLY)
    assert rep["gpu"]["path"] == L.MOE_PATH_DECODE_LAYER
    # the same call again on the same workspace: bitwise the same h
    layer = rep["gpu"]["layer"]
    u = to_device(x.u, "cuda:0")
    h1 = to_numpy(layer.forward(u))
    h2 = to_numpy(layer.forward(u))
    torch.cuda.synchronize()
    assert layer.status() == 0
    assert np.array_equal(h1, h2)
    assert np.array_equal(h1, rep["gpu"]["h_fwd_raw"])


# Batches of 17 to 128 tokens route, dispatch and gather in one kernel before
# the grouped GEMMs (moe_forward_path MOE_PATH_SMALL_BATCH).
SMALL_BATCH_CASES = [
    W("sb_t17", T=17, d=512, n_routed=64, n_shared=2, inter=128, top_k=6, bias_var=0.5),
    W("sb_t100_n256", T=100, d=1024, n_routed=256, n_shared=1, inter=64, top_k=8),
    W("sb_t128_noshared", T=128, d=256, n_routed=20, n_shared=0, inter=192, top_k=3),
]


@pytest.mark.parametrize("wl", SMALL_BATCH_CASES, ids=[c.name for c in SMALL_BATCH_CASES])
def test_small_batch_front_kernel(wl):
    x = S.make_inputs(wl)
    rep = P.full_parity(x)
    assert rep["gpu"]["path"] == L.MOE_PATH_SMALL_BATCH
    assert rep["h_forward"] is not None


@pytest.mark.parametrize("T", [4, 64])
def test_small_paths_replay_from_a_cuda_graph_bitwise(T):
    """The one-kernel decode layer (T = 4) and the small-batch front kernel
    (T = 64) zero their sync words with a one-warp kernel before them:
    captured into a CUDA graph, every replay gives the eager result."""
    wl = W(f"graph{T}", T=T, d=512, n_routed=32, n_shared=1, inter=128, top_k=4)
    x = S.make_inputs(wl)
    layer = MoELayer(x)
    assert L.moe_forward_path(layer.shape) == (L.MOE_PATH_DECODE_LAYER if T <= 16
                                               else L.MOE_PATH_SMALL_BATCH)
    u = to_device(x.u, "cuda:0")
    h = torch.empty_like(u)

    def fwd():
        L.moe_layer_forward(layer.shape, u, layer.E, layer.bias, layer.W13, layer.W2,
                            layer.W13_s, layer.W2_s, h, layer.ws,
                            stream=torch.cuda.current_stream())

    fwd()
    torch.cuda.synchronize()
    ref = to_numpy(h).copy()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    for _ in range(3):
        h.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(to_numpy(h), ref)
    assert layer.status() == 0
