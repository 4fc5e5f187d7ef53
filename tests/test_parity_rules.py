"""The host-side rules the GPU parity tests apply, checked on the CPU: the
near-tie rule for routing and the binding's constants against the header."""
import os
import re

import numpy as np
import pytest

from mixture_experts_layer_56_b200 import _lib as L
from oracle import moe_oracle as O
from tests import parity as P
from tests.conftest import ROOT


def _scores():
    # token 0: clear gaps; token 1: experts 1 and 2 tie within 1e-5 at the K boundary
    s = np.array([[0.50, 0.30, 0.15, 0.05],
                  [0.40, 0.2999995, 0.3000000, 0.0000005]])
    return s / s.sum(axis=1, keepdims=True)


def test_near_tie_swap_is_counted_not_failed():
    s = _scores()
    ref, g = O.topk_gates(s, 2)
    idx = ref.copy()
    idx[1] = [0, 1]  # the other expert of the tied pair
    w = np.take_along_axis(s, idx.astype(np.int64), axis=1).astype(np.float32)
    near, mism = P.check_routing(idx, w, s, 2)
    assert near >= 1 and mism == 1


def test_mismatch_outside_near_ties_fails():
    s = _scores()
    ref, _ = O.topk_gates(s, 2)
    idx = ref.copy()
    idx[0] = [0, 2]  # expert 2 is 0.15 below expert 1: not a near tie
    w = np.take_along_axis(s, idx.astype(np.int64), axis=1).astype(np.float32)
    with pytest.raises(AssertionError):
        P.check_routing(idx, w, s, 2)


def test_gate_error_beyond_the_fp32_bar_fails():
    s = _scores()
    idx, g = O.topk_gates(s, 2)
    w = g.astype(np.float32) + 1e-4
    with pytest.raises(AssertionError):
        P.check_routing(idx, w, s, 2)


def _header_constants():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    consts = {k: int(v) for k, v in re.findall(r"\b(MOE_[A-Z0-9_]+)\s*=\s*(-?\d+)", text)}
    m = re.search(r"#define\s+MOE_DISPATCH_STATIC_SCRATCH_BYTES\s+\((\d+)u\s*\*\s*(\d+)u\)", text)
    consts["MOE_DISPATCH_STATIC_SCRATCH_BYTES"] = int(m.group(1)) * int(m.group(2))
    return consts


def test_binding_constants_match_the_header():
    consts = _header_constants()
    assert len(consts) >= 20
    for name, value in consts.items():
        assert hasattr(L, name), name
        assert getattr(L, name) == value, name
