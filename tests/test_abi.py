"""libmoe.so loads, exports every entry point include/moe.h declares, and its
host-side validation returns the documented codes.  No GPU: every call here
returns before touching a device."""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_56_b200 import _lib as L
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(L.LIB_PATH):
        import __graft_entry__
        __graft_entry__.build()
    return L.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    # and the binding covers the same set
    assert set(names) == set(L.SIGNATURES), set(names) ^ set(L.SIGNATURES)


def test_version_and_strerror(lib):
    assert "sm_100a" in L.moe_version()
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8):
        assert L.strerror(code) and L.strerror(code) != "unknown status"
    assert L.strerror(-99) == "unknown status"


def _shape(**kw):
    base = dict(T=64, d=128, n_routed=16, n_shared=1, inter=64, top_k=4,
                dtype=L.MOE_DTYPE_BF16, flags=0)
    base.update(kw)
    return L.make_shape(**base)


def _ws_rc(shape):
    n = ctypes.c_size_t(0)
    return L.lib().moe_workspace_size(ctypes.byref(shape), ctypes.byref(n)), n.value


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=7), L.MOE_ERR_DTYPE),
    (dict(T=-1), L.MOE_ERR_SHAPE),
    (dict(n_routed=0), L.MOE_ERR_SHAPE),
    (dict(n_routed=257), L.MOE_ERR_SHAPE),
    (dict(top_k=0), L.MOE_ERR_SHAPE),
    (dict(top_k=17), L.MOE_ERR_SHAPE),          # K > n_routed
    (dict(n_routed=64, top_k=33), L.MOE_ERR_SHAPE),
    (dict(n_shared=-1), L.MOE_ERR_SHAPE),
    (dict(inter=96), L.MOE_ERR_SHAPE),          # not a multiple of 64
    (dict(d=96), L.MOE_ERR_SHAPE),              # bf16 tensor-core path needs d % 64 == 0
    (dict(flags=64), L.MOE_ERR_SHAPE),          # unknown flag
    (dict(flags=6), L.MOE_ERR_SHAPE),           # both GEMM tile shapes forced
    (dict(T=2**31, top_k=2), L.MOE_ERR_SHAPE),  # T*K positions overflow int32
])
def test_workspace_size_rejects_bad_shapes(lib, kw, code):
    rc, _ = _ws_rc(_shape(**kw))
    assert rc == code


def test_workspace_size_grows_with_tokens(lib):
    rc0, n0 = _ws_rc(_shape(T=0))
    rc1, n1 = _ws_rc(_shape(T=64))
    rc2, n2 = _ws_rc(_shape(T=4096))
    assert rc0 == rc1 == rc2 == 0
    assert 0 < n0 < n1 < n2 and n2 % 256 == 0
    # fp32 accepts d % 4 == 0
    assert _ws_rc(_shape(d=100, dtype=L.MOE_DTYPE_F32))[0] == 0
    assert L.moe_workspace_size_host(_shape()) > L.moe_workspace_size(_shape())


def test_null_and_alignment_errors_return_before_any_launch(lib):
    s = _shape()
    null = ctypes.c_void_p(0)
    assert lib.moe_workspace_size(None, ctypes.byref(ctypes.c_size_t())) == L.MOE_ERR_NULLPTR
    assert lib.moe_workspace_size(ctypes.byref(s), None) == L.MOE_ERR_NULLPTR
    assert lib.moe_route(ctypes.byref(s), null, null, null, null, null, null) == L.MOE_ERR_NULLPTR
    assert lib.moe_layer_forward(ctypes.byref(s), *([null] * 9), 0, null) == L.MOE_ERR_NULLPTR
    odd = ctypes.c_void_p(0x1008)
    assert lib.moe_route(ctypes.byref(s), odd, odd, null, odd, odd, null) == L.MOE_ERR_ALIGN
    assert lib.moe_combine(ctypes.byref(s), odd, odd, odd, odd, odd, odd, null) == L.MOE_ERR_ALIGN
    # a workspace that is too small is refused (checked before the device)
    p = ctypes.c_void_p(0x10000)
    assert lib.moe_dispatch(ctypes.byref(s), p, p, p, p, p, p, 16, null) == L.MOE_ERR_WORKSPACE
    assert lib.moe_expert_ffn(ctypes.byref(s), p, p, p, p, p, p, p, p, p, p, 16, null) == \
        L.MOE_ERR_WORKSPACE
    # shared experts declared but no shared weights
    assert lib.moe_expert_ffn(ctypes.byref(s), p, p, p, p, p, null, null, p, p, p, 1 << 40,
                              null) == L.MOE_ERR_NULLPTR


def test_zero_tokens_is_a_no_op(lib):
    s = _shape(T=0)
    null = ctypes.c_void_p(0)
    assert lib.moe_route(ctypes.byref(s), null, null, null, null, null, null) == L.MOE_OK
    assert lib.moe_layer_forward(ctypes.byref(s), *([null] * 9), 0, null) == L.MOE_OK
    assert lib.moe_combine(ctypes.byref(s), *([null] * 6), null) == L.MOE_OK


def test_launch_counter_starts_at_zero_without_gpu(lib):
    assert L.moe_launch_count() == 0


@pytest.mark.parametrize("T", [1, 100, 4400, 9000])
@pytest.mark.parametrize("dtype", [L.MOE_DTYPE_BF16, L.MOE_DTYPE_F32])
def test_host_workspace_holds_the_activation_staging(lib, T, dtype):
    """moe_workspace_size_host = moe_workspace_size + room for u and h
    (2 T d elements, each region rounded to 256 bytes)."""
    s = _shape(T=T, dtype=dtype, d=256)
    el = 2 if dtype == L.MOE_DTYPE_BF16 else 4
    stage = -(-T * 256 * el // 256) * 256
    assert L.moe_workspace_size_host(s) == L.moe_workspace_size(s) + 2 * stage


@pytest.mark.parametrize("lang,std", [("c", "c99"), ("c++", "c++11")])
def test_header_compiles_standalone(lang, std, tmp_path):
    """include/moe.h is a plain C header: it compiles on its own as C99 and
    as C++11, with warnings as errors."""
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    r = subprocess.run([cc, "-x", lang, f"-std={std}", "-Wall", "-Wextra", "-Werror",
                        "-fsyntax-only", HEADER], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
