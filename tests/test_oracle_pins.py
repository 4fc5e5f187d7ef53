"""Pins of the CPU oracle against what the DeepSeekMoE pages and mathematics
fix: hand-worked closed forms, the pages' printed combination counts,
brute force on tiny inputs, library routines for textbook special cases, and
the method's invariants (segmentation identity, dense sum, shared-expert
independence).  No GPU."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

from oracle import moe_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _num(v):
    if isinstance(v, str):
        neg = v.startswith("-")
        x = math.log(float(v.lstrip("-")[2:]))
        return -x if neg else x
    return float(v)


def _arr(nested):
    return np.vectorize(_num, otypes=[np.float64])(np.array(nested, dtype=object))


def _rand(rng, *shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def _torch_ffn(x, W1, W3, W2):
    """SwiGLU through torch's own linear / silu (library routines)."""
    xt = torch.from_numpy(x)
    a = F.silu(F.linear(xt, torch.from_numpy(W1))) * F.linear(xt, torch.from_numpy(W3))
    return F.linear(a, torch.from_numpy(W2)).numpy()


# ---------------------------------------------------------------- golden ---
def test_worked_example_closed_forms(golden_dir):
    ex = json.load(open(os.path.join(golden_dir, "worked_example.json")))
    sh = ex["shape"]
    u, E = _arr(ex["u"]), _arr(ex["E"])
    W1, W3, W2 = _arr(ex["W1"]), _arr(ex["W3"]), _arr(ex["W2"])
    W1s, W3s, W2s = _arr(ex["W1_s"]), _arr(ex["W3_s"]), _arr(ex["W2_s"])
    out = O.layer_forward(u, E, None, W1, W3, W2, W1s, W3s, W2s, sh["top_k"])
    exp = ex["expected"]
    np.testing.assert_allclose(out["s"], exp["s"], rtol=0, atol=1e-15)
    np.testing.assert_array_equal(out["idx"], np.array(exp["idx"]))
    np.testing.assert_allclose(out["g"], exp["g"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(out["h"], exp["h"], rtol=0, atol=1e-14)


def test_pages_combination_counts(golden_dir):
    """§3.1 prints C(16,2)=120 and C(64,8)=4,426,165,368; the subset
    enumeration used by the brute-force top-K test reproduces the first."""
    cases = json.load(open(os.path.join(golden_dir, "combinations.json")))["cases"]
    for c in cases:
        assert math.comb(c["n_experts"], c["top_k"]) == c["combinations"]
    small = cases[0]
    n = sum(1 for _ in itertools.combinations(range(small["n_experts"]), small["top_k"]))
    assert n == small["combinations"]


# ---------------------------------------------------------------- router ---
def test_softmax_matches_library():
    rng = np.random.default_rng(1)
    l = _rand(rng, 50, 17, scale=3.0)
    np.testing.assert_allclose(O.softmax(l), scipy.special.softmax(l, axis=1),
                               rtol=1e-14, atol=1e-16)


def test_router_logits_match_matmul_and_bias():
    rng = np.random.default_rng(2)
    u, E, b = _rand(rng, 300, 40), _rand(rng, 9, 40), _rand(rng, 9)
    ref = torch.from_numpy(u) @ torch.from_numpy(E).T + torch.from_numpy(b)
    np.testing.assert_allclose(O.router_logits(u, E, b, block=128), ref.numpy(),
                               rtol=1e-12, atol=1e-12)


def test_duplicate_centroids_give_equal_logits():
    rng = np.random.default_rng(3)
    u, E = _rand(rng, 100, 64), _rand(rng, 6, 64)
    E[4] = E[1]
    l = O.router_logits(u, E)
    assert np.array_equal(l[:, 1], l[:, 4])
    idx, _ = O.topk_gates(O.softmax(l), 6)
    # expert 1 precedes its duplicate 4 in every token's order
    pos = np.argsort(idx, axis=1)
    assert np.all(pos[:, 1] < pos[:, 4])


@pytest.mark.parametrize("n,K", [(4, 1), (5, 2), (6, 3), (8, 4), (7, 7)])
def test_topk_brute_force(n, K):
    """Top-K = the K-subset with the largest score sum; among equal sums the
    lexicographically smallest index set (lower index wins ties).  Integer
    logits make sums exact and create many ties."""
    rng = np.random.default_rng(10 * n + K)
    l = rng.integers(-2, 3, size=(200, n)).astype(np.float64)
    idx, g = O.topk_gates(O.softmax(l), K)
    for t in range(l.shape[0]):
        best = None
        for sub in itertools.combinations(range(n), K):
            key = (-sum(l[t, list(sub)]), sub)
            if best is None or key < best:
                best = key
        assert tuple(sorted(idx[t])) == best[1]
        # descending score order within the selection
        assert np.all(np.diff(O.softmax(l)[t, idx[t]]) <= 0)


def test_topk_matches_torch_topk_on_distinct_scores():
    rng = np.random.default_rng(4)
    s = O.softmax(_rand(rng, 500, 63, scale=2.0))
    idx, g = O.topk_gates(s, 7)
    tv, ti = torch.topk(torch.from_numpy(s), 7, dim=1)
    np.testing.assert_array_equal(idx, ti.numpy())
    np.testing.assert_array_equal(g, tv.numpy())


def test_gates_not_renormalised():
    rng = np.random.default_rng(5)
    s = O.softmax(_rand(rng, 64, 16))
    _, g = O.topk_gates(s, 4)
    assert np.all(g > 0) and np.all(g < 1)
    assert np.all(g.sum(axis=1) < 1.0)
    _, gall = O.topk_gates(s, 16)
    np.testing.assert_allclose(gall.sum(axis=1), 1.0, rtol=0, atol=1e-14)


def test_topk_gap():
    s = np.array([[0.5, 0.3, 0.2], [0.4, 0.4, 0.2]])
    np.testing.assert_allclose(O.topk_gap(s, 1), [0.2, 0.0])
    assert np.all(np.isinf(O.topk_gap(s, 3)))


# -------------------------------------------------------------- dispatch ---
def _dispatch_bruteforce(idx, n):
    T, K = len(idx), len(idx[0])
    counts = [0] * n
    for t in range(T):
        for k in range(K):
            counts[idx[t][k]] += 1
    offsets = [0]
    for c in counts:
        offsets.append(offsets[-1] + c)
    perm, fill = [None] * (T * K), list(offsets[:-1])
    for t in range(T):          # tokens in increasing order
        for k in range(K):
            e = idx[t][k]
            perm[fill[e]] = t * K + k
            fill[e] += 1
    inv = [None] * (T * K)
    for p, slot in enumerate(perm):
        inv[slot] = p
    return counts, offsets, perm, inv


@pytest.mark.parametrize("T,n,K", [(1, 4, 2), (37, 8, 3), (100, 16, 4), (5, 3, 3)])
def test_dispatch_brute_force(T, n, K):
    rng = np.random.default_rng(T + n + K)
    idx = np.stack([rng.permutation(n)[:K] for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = O.dispatch(idx, n)
    bc, bo, bp, bi = _dispatch_bruteforce(idx.tolist(), n)
    assert counts.tolist() == bc and offsets.tolist() == bo
    assert perm.tolist() == bp and inv.tolist() == bi
    # invariants
    assert counts.sum() == T * K and offsets[-1] == T * K
    assert np.array_equal(np.sort(perm), np.arange(T * K))
    assert np.array_equal(perm[inv], np.arange(T * K))
    for e in range(n):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(idx.reshape(-1)[seg] == e)
        assert np.all(np.diff(seg // K) > 0)


# ----------------------------------------------------------------- experts --
def test_swiglu_matches_torch_functional():
    rng = np.random.default_rng(6)
    x = _rand(rng, 33, 24)
    W1, W3, W2 = _rand(rng, 16, 24), _rand(rng, 16, 24), _rand(rng, 24, 16)
    np.testing.assert_allclose(O.swiglu_ffn(x, W1, W3, W2), _torch_ffn(x, W1, W3, W2),
                               rtol=1e-12, atol=1e-12)


def test_silu_matches_torch():
    x = np.linspace(-40, 40, 1001)
    np.testing.assert_allclose(O.silu(x), F.silu(torch.from_numpy(x)).numpy(),
                               rtol=1e-14, atol=1e-300)


def _layer_inputs(rng, T, d, n, ns, I):
    return dict(u=_rand(rng, T, d), E=_rand(rng, n, d, scale=d ** -0.5),
                W1=_rand(rng, n, I, d, scale=d ** -0.5), W3=_rand(rng, n, I, d, scale=d ** -0.5),
                W2=_rand(rng, n, d, I, scale=I ** -0.5),
                W1_s=_rand(rng, ns, I, d, scale=d ** -0.5), W3_s=_rand(rng, ns, I, d, scale=d ** -0.5),
                W2_s=_rand(rng, ns, d, I, scale=I ** -0.5))


def test_all_experts_with_unit_gates_is_dense_sum():
    """K = N_r with every gate forced to 1: h = u + sum of all FFNs, evaluated
    directly with torch (no dispatch, no combine)."""
    rng = np.random.default_rng(7)
    p = _layer_inputs(rng, 29, 16, 5, 2, 8)
    out = O.layer_forward(p["u"], p["E"], None, p["W1"], p["W3"], p["W2"],
                          p["W1_s"], p["W3_s"], p["W2_s"], K=5, gates=1.0)
    ref = p["u"].copy()
    for e in range(5):
        ref += _torch_ffn(p["u"], p["W1"][e], p["W3"][e], p["W2"][e])
    for s in range(2):
        ref += _torch_ffn(p["u"], p["W1_s"][s], p["W3_s"][s], p["W2_s"][s])
    np.testing.assert_allclose(out["h"], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("m", [2, 4, 8])
def test_fine_grained_segmentation_identity(m):
    """§3.1: one FFN of width I equals m experts of width I/m (slices of the
    W1/W3 rows and W2 columns) all active with gate 1."""
    rng = np.random.default_rng(8 + m)
    T, d, I = 21, 12, 16
    u = _rand(rng, T, d)
    W1, W3, W2 = _rand(rng, I, d), _rand(rng, I, d), _rand(rng, d, I)
    whole = O.swiglu_ffn(u, W1, W3, W2)
    w = I // m
    seg1 = np.stack([W1[j * w:(j + 1) * w] for j in range(m)])
    seg3 = np.stack([W3[j * w:(j + 1) * w] for j in range(m)])
    seg2 = np.stack([W2[:, j * w:(j + 1) * w] for j in range(m)])
    E = _rand(rng, m, d)
    zero_s = np.zeros((0, w, d)), np.zeros((0, w, d)), np.zeros((0, d, w))
    out = O.layer_forward(u, E, None, seg1, seg3, seg2, *zero_s, K=m, gates=1.0)
    np.testing.assert_allclose(out["h"] - u, whole, rtol=1e-12, atol=1e-12)
    # the same identity read as K_s shared experts = one FFN of width K_s*w
    np.testing.assert_allclose(O.shared_experts(u, seg1, seg3, seg2), whole,
                               rtol=1e-12, atol=1e-12)


def test_shared_experts_independent_of_routing():
    rng = np.random.default_rng(9)
    p = _layer_inputs(rng, 40, 16, 6, 2, 8)
    a = O.layer_forward(p["u"], p["E"], None, p["W1"], p["W3"], p["W2"],
                        p["W1_s"], p["W3_s"], p["W2_s"], K=2)
    E2 = _rand(rng, 6, 16)
    b2 = _rand(rng, 6)
    b = O.layer_forward(p["u"], E2, b2, p["W1"], p["W3"], p["W2"],
                        p["W1_s"], p["W3_s"], p["W2_s"], K=2)
    assert not np.array_equal(a["idx"], b["idx"])

    def shared_part(o):
        routed = O.combine(np.zeros_like(p["u"]), np.zeros_like(p["u"]),
                           o["y"], o["g"], o["inv"], 2)
        return o["h"] - p["u"] - routed

    np.testing.assert_allclose(shared_part(a), shared_part(b), rtol=1e-12, atol=1e-12)
    ref = sum(_torch_ffn(p["u"], p["W1_s"][s], p["W3_s"][s], p["W2_s"][s]) for s in range(2))
    np.testing.assert_allclose(shared_part(a), ref, rtol=1e-12, atol=1e-12)


def test_switch_top1_special_case():
    """§2: K = 1, no shared experts (Switch-style top-1): h = u + s_max FFN_argmax(u)."""
    rng = np.random.default_rng(11)
    p = _layer_inputs(rng, 25, 8, 4, 0, 6)
    out = O.layer_forward(p["u"], p["E"], None, p["W1"], p["W3"], p["W2"],
                          p["W1_s"], p["W3_s"], p["W2_s"], K=1)
    s = scipy.special.softmax(p["u"] @ p["E"].T, axis=1)
    top = np.argmax(s, axis=1)
    ref = p["u"].copy()
    for t in range(25):
        ref[t] += s[t, top[t]] * _torch_ffn(p["u"][t:t + 1], p["W1"][top[t]],
                                            p["W3"][top[t]], p["W2"][top[t]])[0]
    np.testing.assert_allclose(out["h"], ref, rtol=1e-12, atol=1e-12)


def test_gshard_top2_special_case():
    """§2, eqs. (3)-(5): GShard-style top-2 over N experts, no shared ones,
    evaluated with torch.topk and torch.softmax."""
    rng = np.random.default_rng(12)
    p = _layer_inputs(rng, 31, 8, 6, 0, 4)
    out = O.layer_forward(p["u"], p["E"], None, p["W1"], p["W3"], p["W2"],
                          p["W1_s"], p["W3_s"], p["W2_s"], K=2)
    s = torch.softmax(torch.from_numpy(p["u"] @ p["E"].T), dim=1)
    gv, gi = torch.topk(s, 2, dim=1)
    ref = p["u"].copy()
    for t in range(31):
        for k in range(2):
            e = int(gi[t, k])
            ref[t] += float(gv[t, k]) * _torch_ffn(p["u"][t:t + 1], p["W1"][e],
                                                   p["W3"][e], p["W2"][e])[0]
    np.testing.assert_allclose(out["h"], ref, rtol=1e-12, atol=1e-12)


def test_combine_special_cases():
    rng = np.random.default_rng(13)
    T, d, K = 10, 6, 3
    u, ysh = _rand(rng, T, d), _rand(rng, T, d)
    g = rng.random((T, K))
    inv = rng.permutation(T * K).astype(np.int32)
    np.testing.assert_array_equal(O.combine(u, ysh, np.zeros((T * K, d)), g, inv, K), u + ysh)
    y = _rand(rng, T * K, d)
    h = O.combine(u, ysh, y, g, inv, K)
    for t in range(T):
        ref = u[t] + ysh[t] + sum(g[t, k] * y[inv[t * K + k]] for k in range(K))
        np.testing.assert_allclose(h[t], ref, rtol=1e-14, atol=1e-14)


def test_layer_forward_tokens_matches_full():
    rng = np.random.default_rng(14)
    p = _layer_inputs(rng, 50, 16, 8, 1, 8)
    full = O.layer_forward(p["u"], p["E"], None, p["W1"], p["W3"], p["W2"],
                           p["W1_s"], p["W3_s"], p["W2_s"], K=3)
    toks = [0, 7, 49, 23]
    part = O.layer_forward_tokens(p["u"], full["idx"], full["g"], toks, p["W1"], p["W3"],
                                  p["W2"], p["W1_s"], p["W3_s"], p["W2_s"])
    np.testing.assert_allclose(part, full["h"][toks], rtol=1e-12, atol=1e-12)


def test_override_routing_reproduces_own_routing():
    rng = np.random.default_rng(15)
    p = _layer_inputs(rng, 20, 8, 6, 1, 4)
    a = O.layer_forward(p["u"], p["E"], None, p["W1"], p["W3"], p["W2"],
                        p["W1_s"], p["W3_s"], p["W2_s"], K=2)
    b = O.layer_forward(p["u"], p["E"], None, p["W1"], p["W3"], p["W2"],
                        p["W1_s"], p["W3_s"], p["W2_s"], K=2, idx=a["idx"])
    np.testing.assert_array_equal(a["h"], b["h"])


# --------------------------------------------------------------- balance ---
def test_expert_balance_statistics():
    """eqs. (12)-(14): sum_i f_i = N'; uniform routing gives f_i = 1 and,
    with uniform scores, L_ExpBal = alpha1."""
    rng = np.random.default_rng(16)
    s = O.softmax(_rand(rng, 120, 12))
    idx, _ = O.topk_gates(s, 3)
    f, P, L = O.expert_balance(s, idx, alpha1=0.01)
    np.testing.assert_allclose(f.sum(), 12.0, rtol=1e-14)
    np.testing.assert_allclose(P.sum(), 1.0, rtol=1e-14)
    # uniform: each of 4 experts chosen by exactly half of 8 tokens, K=2
    idx_u = np.array([[0, 1], [2, 3]] * 4, dtype=np.int32)
    s_u = np.full((8, 4), 0.25)
    f_u, P_u, L_u = O.expert_balance(s_u, idx_u, alpha1=0.3)
    np.testing.assert_allclose(f_u, 1.0)
    np.testing.assert_allclose(L_u, 0.3)
    # device level, eqs. (15)-(17): two devices of two experts each
    fd, Pd, Ld = O.device_balance(f_u, P_u, [(0, 1), (2, 3)], alpha2=2.0)
    np.testing.assert_allclose(fd, [1.0, 1.0])
    np.testing.assert_allclose(Pd, [0.5, 0.5])
    np.testing.assert_allclose(Ld, 2.0)


def test_select_only_bias_variant():
    """Bias that steers only the selection: with b = 0 it is the plain top-K;
    with a large bias on one expert that expert is always chosen while its
    gate stays its unbiased softmax score."""
    rng = np.random.default_rng(17)
    l = _rand(rng, 40, 8)
    i0, g0 = O.topk_gates_select_only_bias(l, np.zeros(8), 3)
    i1, g1 = O.topk_gates(O.softmax(l), 3)
    np.testing.assert_array_equal(i0, i1)
    np.testing.assert_array_equal(g0, g1)
    b = np.zeros(8)
    b[5] = 1e3
    i2, g2 = O.topk_gates_select_only_bias(l, b, 3)
    assert np.all(i2[:, 0] == 5)
    np.testing.assert_allclose(g2[:, 0], scipy.special.softmax(l, axis=1)[:, 5], rtol=1e-14)


def test_routed_expert_outputs_against_torch():
    """Every routed slot's row: y[inv[t*K+k]] = FFN_{idx[t,k]}(u_t) (eq. (9)'s
    routed terms before the gate), against torch's float64 linear / silu
    evaluated token by token."""
    rng = np.random.default_rng(11)
    T, d, I, n, K = 9, 12, 8, 5, 3
    u = rng.standard_normal((T, d))
    W1 = rng.standard_normal((n, I, d)) / math.sqrt(d)
    W3 = rng.standard_normal((n, I, d)) / math.sqrt(d)
    W2 = rng.standard_normal((n, d, I)) / math.sqrt(I)
    idx = np.argsort(rng.standard_normal((T, n)), axis=1)[:, :K].astype(np.int32)
    counts, offsets, perm, inv = O.dispatch(idx, n)
    y = O.routed_expert_outputs(u, perm, offsets, K, W1, W3, W2)
    tu = torch.from_numpy(u)
    for t in range(T):
        for k in range(K):
            e = int(idx[t, k])
            a = F.silu(F.linear(tu[t], torch.from_numpy(W1[e]))) * \
                F.linear(tu[t], torch.from_numpy(W3[e]))
            ref = F.linear(a, torch.from_numpy(W2[e])).numpy()
            np.testing.assert_allclose(y[inv[t * K + k]], ref, rtol=0, atol=1e-12)
