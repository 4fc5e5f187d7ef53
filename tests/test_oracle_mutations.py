"""Plant plausible mistakes in (copies of) the oracle's steps on the CPU and
check that the pins notice each one: a pin that passes a wrong oracle pins
nothing."""
import json
import os

import numpy as np
import pytest

from oracle import moe_oracle as O
from tests.test_oracle_pins import _arr

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _worked(golden_dir):
    ex = json.load(open(os.path.join(golden_dir, "worked_example.json")))
    args = [_arr(ex[k]) for k in ("u", "E")] + [None] + \
           [_arr(ex[k]) for k in ("W1", "W3", "W2", "W1_s", "W3_s", "W2_s")]
    return args, ex["shape"]["top_k"], ex["expected"]


def _worked_example_passes(golden_dir):
    args, K, exp = _worked(golden_dir)
    try:
        out = O.layer_forward(*args, K)
    except Exception:
        return False
    return (np.array_equal(out["idx"], np.array(exp["idx"]))
            and np.allclose(out["g"], exp["g"], atol=1e-14)
            and np.allclose(out["h"], exp["h"], atol=1e-13))


MUTANTS = {
    "silu sign": ("silu", lambda x: x / (1.0 + np.exp(x))),
    "plain sigmoid": ("silu", lambda x: 1.0 / (1.0 + np.exp(-x))),
    "renormalised gates": ("topk_gates", lambda s, K: (
        np.argsort(-s, axis=1, kind="stable")[:, :K].astype(np.int32),
        np.take_along_axis(s, np.argsort(-s, axis=1, kind="stable")[:, :K], 1)
        / np.take_along_axis(s, np.argsort(-s, axis=1, kind="stable")[:, :K], 1).sum(1, keepdims=True))),
    "higher index wins ties": ("topk_gates", lambda s, K: (
        (s.shape[1] - 1 - np.argsort(-s[:, ::-1], axis=1, kind="stable")[:, :K]).astype(np.int32),
        np.take_along_axis(s, s.shape[1] - 1 - np.argsort(-s[:, ::-1], axis=1, kind="stable")[:, :K], 1))),
    "dropped shared experts": ("shared_experts", lambda u, a, b, c: np.zeros_like(u)),
    "dropped residual": ("combine", lambda u, ysh, y, g, inv, K: O.__dict__["_orig_combine"](
        np.zeros_like(u), ysh, y, g, inv, K)),
    "gate/up swapped": ("swiglu_ffn", lambda x, W1, W3, W2: (O.silu(x @ W3.T) * (x @ W1.T)) @ W2.T),
    "softmax without max shift but squared": ("softmax", lambda l: np.exp(2 * l) / np.exp(2 * l).sum(1, keepdims=True)),
    "ascending top-k": ("topk_gates", lambda s, K: (
        np.argsort(s, axis=1, kind="stable")[:, :K].astype(np.int32),
        np.take_along_axis(s, np.argsort(s, axis=1, kind="stable")[:, :K], 1))),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistake(name, golden_dir, monkeypatch):
    assert _worked_example_passes(golden_dir)
    attr, fn = MUTANTS[name]
    monkeypatch.setitem(O.__dict__, "_orig_combine", O.combine)
    monkeypatch.setattr(O, attr, fn)
    assert not _worked_example_passes(golden_dir), name


def test_routed_rows_pin_rejects_a_wrong_token_of_a_slot(monkeypatch):
    """Planted mistake: a position's token taken as slot % K instead of
    slot // K (the slot is t*K + k)."""
    from tests.test_oracle_pins import test_routed_expert_outputs_against_torch as pin

    def wrong(u, perm, offsets, K, W1, W3, W2):
        y = np.zeros((perm.size, u.shape[1]))
        for e in range(W1.shape[0]):
            lo, hi = int(offsets[e]), int(offsets[e + 1])
            if hi > lo:
                y[lo:hi] = O.swiglu_ffn(u[perm[lo:hi] % K], W1[e], W3[e], W2[e])
        return y

    pin()  # the pin holds for the oracle as it is
    monkeypatch.setattr(O, "routed_expert_outputs", wrong)
    with pytest.raises(AssertionError):
        pin()


def test_logit_pin_rejects_a_dropped_router_bias(monkeypatch):
    """Planted mistake: eq. (11)'s logits without the per-expert bias."""
    from tests.test_oracle_pins import test_router_logits_match_matmul_and_bias as pin
    orig = O.router_logits
    pin()
    monkeypatch.setattr(O, "router_logits", lambda u, E, bias=None, block=None: orig(u, E, None))
    with pytest.raises(AssertionError):
        pin()


def test_dispatch_pin_rejects_unstable_token_order(monkeypatch):
    """Planted mistake: each expert's tokens listed in decreasing t."""
    from tests.test_oracle_pins import test_dispatch_brute_force as pin
    orig = O.dispatch

    def reversed_segments(idx, n):
        counts, offsets, perm, inv = orig(idx, n)
        perm = perm.copy()
        for e in range(n):
            perm[offsets[e]:offsets[e + 1]] = perm[offsets[e]:offsets[e + 1]][::-1]
        inv = np.empty_like(inv)
        inv[perm] = np.arange(perm.size, dtype=inv.dtype)
        return counts, offsets, perm, inv

    pin(37, 8, 3)
    monkeypatch.setattr(O, "dispatch", reversed_segments)
    with pytest.raises(AssertionError):
        pin(37, 8, 3)
