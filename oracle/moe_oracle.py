"""CPU oracle for the DeepSeekMoE layer forward -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package entry's smoke check and the bench's CPU-baseline
leg may import this module.  The product path never calls it and shares no
code with it: it is plain numpy in float64, written from the equations of
"DeepSeekMoE: Towards Ultimate Expert Specialization in Mixture-of-Experts
Language Models" (papercache.org summary of arXiv 2401.06066):

* §2 (background), eqs. (3)-(5): conventional top-K MoE, h = sum_i g_i FFN_i(u) + u,
  g_i = s_i if s_i is among the K largest else 0, s_i = Softmax_i(u^T e_i).
* §3.1, eqs. (6)-(8): fine-grained segmentation -- mN experts, mK active.
* §3.2, eqs. (9)-(11): K_s shared experts always active and ungated, top
  (mK - K_s) of the (mN - K_s) routed experts, gates not renormalised.
* §3.3, eqs. (12)-(14) and (15)-(17): expert- and device-level balance
  statistics.

The expert FFN is SwiGLU, W2 (SiLU(W1 x) * W3 x), as in DeepSeek LLM (the
dtcms.com overview, "DeepSeek LLM / model structure").

Readings where the pages are silent (each also listed in the design notes):
* the softmax runs over the routed experts only (shared experts have no
  centroid e_i);
* an optional router bias b_i is added to the logit before both the softmax
  and the selection (the pages name a per-expert bias but print no formula);
* ties in the top-K are broken towards the lower expert index;
* layer normalisation is omitted, as on the pages (§2).

Parity pins: every function here is checked by ``tests/test_oracle_pins.py``
against closed forms, brute force, invariants and the values the pages print
(C(16,2) = 120 and C(64,8) = 4,426,165,368 in §3.1).
"""
from __future__ import annotations

import numpy as np


# --------------------------------------------------------------------------
# router: eqs. (10)-(11)
# --------------------------------------------------------------------------
def router_logits(u: np.ndarray, E: np.ndarray, bias: np.ndarray | None = None,
                  block: int | None = None) -> np.ndarray:
    """l[t, i] = u_t^T e_i (+ b_i), eq. (11) before the softmax.

    One matrix-vector product per expert i (over blocks of tokens), so that
    two identical centroids e_i = e_j give bitwise identical logits.
    """
    T = u.shape[0]
    n = E.shape[0]
    if block is None:
        block = max(1, (1 << 21) // max(1, u.shape[1]))
    l = np.empty((T, n), dtype=np.float64)
    for t0 in range(0, T, block):
        ub = u[t0:t0 + block]
        for i in range(n):
            l[t0:t0 + block, i] = ub @ E[i]
    if bias is not None:
        l += np.asarray(bias, dtype=np.float64)[None, :]
    return l


def softmax(l: np.ndarray) -> np.ndarray:
    """s_{i,t} = Softmax_i(l_{i,t}) over the routed experts, eq. (11)."""
    m = l.max(axis=1, keepdims=True)
    e = np.exp(l - m)
    return e / e.sum(axis=1, keepdims=True)


def topk_gates(s: np.ndarray, K: int) -> tuple[np.ndarray, np.ndarray]:
    """eq. (10): keep the K largest scores of each token, gate = score.

    Returns idx[T, K] (int32, in descending score order; equal scores keep
    the lower expert index first) and g[T, K] = s at those experts, not
    renormalised.
    """
    order = np.argsort(-s, axis=1, kind="stable")[:, :K]
    g = np.take_along_axis(s, order, axis=1)
    return order.astype(np.int32), g


def topk_gap(s: np.ndarray, K: int) -> np.ndarray:
    """Score gap between the K-th and (K+1)-th largest score of each token
    (inf when K equals the number of experts): the margin of the selection."""
    if K >= s.shape[1]:
        return np.full(s.shape[0], np.inf)
    srt = -np.sort(-s, axis=1)
    return srt[:, K - 1] - srt[:, K]


# --------------------------------------------------------------------------
# dispatch: "each token is computed only by its K experts" (§2, after eq. 5)
# --------------------------------------------------------------------------
def dispatch(idx: np.ndarray, n_routed: int):
    """Group the T*K routed slots by expert.

    counts[e]  = number of slots (t, k) with idx[t, k] = e
    offsets    = exclusive prefix sum of counts (length n_routed + 1)
    perm[p]    = slot t*K + k at position p; slots of expert e fill
                 offsets[e] .. offsets[e+1]-1 in increasing token order
    inv[slot]  = position of that slot, so perm[inv[s]] = s
    """
    flat = idx.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=n_routed).astype(np.int32)
    offsets = np.zeros(n_routed + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return counts, offsets, perm, inv


# --------------------------------------------------------------------------
# experts: SwiGLU FFN
# --------------------------------------------------------------------------
def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x / (1 + e^-x)."""
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def swiglu_ffn(x: np.ndarray, W1: np.ndarray, W3: np.ndarray,
               W2: np.ndarray) -> np.ndarray:
    """FFN(x) = W2 (SiLU(W1 x) * (W3 x)) for rows x[n, d];
    W1, W3 are [I, d] and W2 is [d, I]."""
    a = silu(x @ W1.T) * (x @ W3.T)
    return a @ W2.T


def shared_experts(u: np.ndarray, W1_s, W3_s, W2_s) -> np.ndarray:
    """First sum of eq. (9): sum over the K_s shared experts, each ungated."""
    out = np.zeros_like(u)
    for s in range(W1_s.shape[0]):
        out += swiglu_ffn(u, W1_s[s], W3_s[s], W2_s[s])
    return out


def routed_expert_outputs(u, perm, offsets, K, W1, W3, W2) -> np.ndarray:
    """y[p] = FFN_e(u_t) for each position p of expert e's segment, where
    slot perm[p] = t*K + k (rows in dispatch order)."""
    y = np.zeros((perm.size, u.shape[1]), dtype=np.float64)
    for e in range(W1.shape[0]):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            tok = perm[lo:hi] // K
            y[lo:hi] = swiglu_ffn(u[tok], W1[e], W3[e], W2[e])
    return y


def combine(u, y_shared, y, g, inv, K) -> np.ndarray:
    """eq. (9): h_t = u_t + shared_t + sum_k g_{t,k} y[inv[t*K+k]]."""
    T = u.shape[0]
    h = u + y_shared
    for k in range(K):
        rows = inv[np.arange(T) * K + k]
        h = h + g[:, k:k + 1] * y[rows]
    return h


# --------------------------------------------------------------------------
# whole layer, eqs. (9)-(11)
# --------------------------------------------------------------------------
def layer_forward(u, E, bias, W1, W3, W2, W1_s, W3_s, W2_s, K,
                  idx=None, gates=None):
    """The DeepSeekMoE layer.  All arrays float64; returns a dict with the
    output h and every intermediate (logits, s, idx, g, counts, offsets,
    perm, inv, y, y_shared).

    ``idx`` replaces the router's selection (e.g. to evaluate the FFN and
    combine on another implementation's routing); ``gates`` replaces the
    gate values (e.g. all ones).
    """
    n = E.shape[0]
    l = router_logits(u, E, bias)
    s = softmax(l)
    if idx is None:
        idx, g = topk_gates(s, K)
    else:
        idx = np.asarray(idx, dtype=np.int32)
        g = np.take_along_axis(s, idx.astype(np.int64), axis=1)
    if gates is not None:
        g = np.broadcast_to(np.asarray(gates, dtype=np.float64), idx.shape).copy()
    counts, offsets, perm, inv = dispatch(idx, n)
    y_sh = shared_experts(u, W1_s, W3_s, W2_s)
    y = routed_expert_outputs(u, perm, offsets, K, W1, W3, W2)
    h = combine(u, y_sh, y, g, inv, K)
    return dict(h=h, logits=l, s=s, idx=idx, g=g, counts=counts,
                offsets=offsets, perm=perm, inv=inv, y=y, y_shared=y_sh)


def layer_forward_tokens(u, idx, g, tokens, W1, W3, W2, W1_s, W3_s, W2_s):
    """h for the listed tokens only, given each token's routing (idx, g):
    eq. (9) for those tokens (for sampled checks at full size).  The routed
    sum is taken expert by expert over the sampled tokens that chose it."""
    tokens = np.asarray(tokens, dtype=np.int64)
    x = u[tokens]
    h = x + shared_experts(x, W1_s, W3_s, W2_s)
    sel = np.asarray(idx)[tokens]
    gs = np.asarray(g)[tokens]
    for e in np.unique(sel):
        rows, ks = np.nonzero(sel == e)
        h[rows] += gs[rows, ks][:, None] * swiglu_ffn(x[rows], W1[e], W3[e], W2[e])
    return h


def topk_gates_select_only_bias(l: np.ndarray, bias: np.ndarray, K: int):
    """Bias that steers only the selection: the K largest l + b are chosen
    (lower index first on ties) and the gates are the softmax of the
    unbiased logits l at those experts, not renormalised."""
    order = np.argsort(-(l + np.asarray(bias, dtype=np.float64)[None, :]), axis=1,
                       kind="stable")[:, :K]
    s = softmax(l)
    return order.astype(np.int32), np.take_along_axis(s, order, axis=1)


# --------------------------------------------------------------------------
# balance statistics, eqs. (12)-(17)
# --------------------------------------------------------------------------
def expert_balance(s: np.ndarray, idx: np.ndarray, alpha1: float = 1.0):
    """eqs. (12)-(14): f_i = N'/(K'T) * #tokens selecting i,
    P_i = mean_t s_{i,t}, L_ExpBal = alpha1 * sum_i f_i P_i."""
    T, n = s.shape
    K = idx.shape[1]
    sel = np.zeros((T, n), dtype=np.float64)
    np.put_along_axis(sel, idx.astype(np.int64), 1.0, axis=1)
    f = n / (K * T) * sel.sum(axis=0)
    P = s.mean(axis=0)
    return f, P, alpha1 * float(np.sum(f * P))


def device_balance(f: np.ndarray, P: np.ndarray, groups, alpha2: float = 1.0):
    """eqs. (15)-(17): f'_i = mean of f over group i, P'_i = sum of P over
    group i, L_DevBal = alpha2 * sum_i f'_i P'_i."""
    fd = np.array([f[list(gr)].mean() for gr in groups])
    Pd = np.array([P[list(gr)].sum() for gr in groups])
    return fd, Pd, alpha2 * float(np.sum(fd * Pd))
