"""Pins of the oracle to facts fixed by the SP-KV page and by mathematics.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with a
closed form, a library special case, a hand-derived fixture or a brute-force
enumeration.  ``test_oracle_pins.py`` runs them all; ``test_oracle_mutations.py``
plants plausible mistakes in the oracle and checks that some pin catches each.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
from scipy.special import expit

from oracle import spkv_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    assert err <= tol, f"{what}: max abs error {err:.3e} > {tol:.1e}"


def _sdpa(Q, K, V, mask):
    """torch scaled_dot_product_attention in fp64 on CPU.  Q [n][Hq][d] queries at
    positions 0..n-1, K/V [T][Hkv][d]; key heads are repeated for GQA (query head
    h uses key head h // G).  ``mask``: None for plain causal, else a bool [n][T]."""
    Hq, Hkv = Q.shape[1], K.shape[1]
    G = Hq // Hkv
    q = torch.from_numpy(np.ascontiguousarray(Q.transpose(1, 0, 2))).double()
    k = torch.from_numpy(np.ascontiguousarray(K.transpose(1, 0, 2))).double().repeat_interleave(G, 0)
    v = torch.from_numpy(np.ascontiguousarray(V.transpose(1, 0, 2))).double().repeat_interleave(G, 0)
    if mask is None:
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    else:
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(mask))
    return o.numpy().transpose(1, 0, 2)


def _rand_qkv(rng, T, Hq, Hkv, d):
    Q = rng.standard_normal((T, Hq, d))
    K = rng.standard_normal((T, Hkv, d))
    V = rng.standard_normal((T, Hkv, d))
    return Q, K, V


def _mlp(rng, N, D, hid, Hkv, scale=0.3):
    h = rng.standard_normal((N, D))
    W1 = rng.standard_normal((hid, D)) * scale
    b1 = rng.standard_normal(hid) * scale
    W2 = rng.standard_normal((Hkv, hid)) * scale
    b2 = rng.standard_normal(Hkv) * scale
    return h, W1, b1, W2, b2


# ---------------------------------------------------------------- Eq. (1) ----

def pin_gelu_textbook():
    g = _golden("gelu_sigmoid_values.json")
    for a, want in g["gelu"]:
        _close(O.gelu(np.array([a])), [want], 1e-15, f"GELU({a})")
    for x, want in g["sigmoid"]:
        _close(O.sigmoid(np.array([x])), [want], 1e-15, f"sigmoid({x})")


def pin_gelu_library():
    x = np.linspace(-8, 8, 1001)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="none").numpy()
    _close(O.gelu(x), ref, 1e-14, "GELU vs torch (exact erf form)")


def pin_utility_zero_weights():
    """W1 = W2 = 0 leaves u = sigmoid(b2) for every token (closed form)."""
    rng = np.random.default_rng(1)
    N, D, hid, Hkv = 7, 12, 5, 3
    h = rng.standard_normal((N, D))
    b2 = np.array([-3.0, 0.0, 2.5])
    u = O.utility(h, np.zeros((hid, D)), rng.standard_normal(hid), np.zeros((Hkv, hid)), b2)
    _close(u, np.broadcast_to(expit(b2), (N, Hkv)), 1e-15, "u with zero weights")


def pin_utility_hand_example():
    """One token, one hidden unit: a = 1 -> GELU = Phi(1); W2 = 2, b2 = -1 ->
    logit = 2 Phi(1) - 1."""
    phi1 = 0.8413447460685429
    u = O.utility(np.array([[1.0, 5.0]]), np.array([[1.0, 0.0]]), np.array([0.0]),
                  np.array([[2.0]]), np.array([-1.0]))
    _close(u, [[expit(2 * phi1 - 1)]], 1e-15, "hand example")


def pin_utility_library():
    """The perceptron equals torch Linear -> GELU -> Linear -> sigmoid in fp64."""
    rng = np.random.default_rng(2)
    h, W1, b1, W2, b2 = _mlp(rng, 33, 24, 16, 4)
    l1 = torch.nn.Linear(24, 16).double()
    l2 = torch.nn.Linear(16, 4).double()
    with torch.no_grad():
        l1.weight.copy_(torch.from_numpy(W1)); l1.bias.copy_(torch.from_numpy(b1))
        l2.weight.copy_(torch.from_numpy(W2)); l2.bias.copy_(torch.from_numpy(b2))
        ref = torch.sigmoid(l2(torch.nn.functional.gelu(l1(torch.from_numpy(h))))).numpy()
    _close(O.utility(h, W1, b1, W2, b2), ref, 1e-14, "utility vs torch MLP")


# ---------------------------------------------------------------- Eq. (2) ----

def pin_gate_threshold():
    """z = 1[u >= tau]: equality keeps the token; the next double above tau drops it."""
    u = O.utility(np.zeros((1, 3)), np.zeros((2, 3)), np.zeros(2), np.zeros((1, 2)), np.zeros(1))
    assert float(u[0, 0]) == 0.5
    assert O.gate(u, 0.5)[0, 0] == 1, "u == tau must be kept"
    assert O.gate(u, np.nextafter(0.5, 1.0))[0, 0] == 0
    assert O.gate(u, np.nextafter(0.5, 0.0))[0, 0] == 1
    uu = np.array([0.1, 0.2, 0.3, 0.7])
    assert list(O.gate(uu, 0.3)) == [0, 0, 1, 1]


def pin_gate_extremes():
    """tau = 0 keeps every token (u > 0); tau > 1 keeps none (u < 1)."""
    rng = np.random.default_rng(3)
    h, W1, b1, W2, b2 = _mlp(rng, 50, 10, 8, 2, scale=3.0)
    u = O.utility(h, W1, b1, W2, b2)
    assert O.gate(u, 0.0).all()
    assert not O.gate(u, 1.5).any()


# ----------------------------------------------------------- Eqs. (3)-(4) ----

def pin_keysets_golden():
    """With q = 0 every visible key gets the same weight, so with one-hot values the
    output is the indicator of the visible set divided by its size, and lse = ln|S|.
    The visible sets are hand-derived from Eq. (4)."""
    for case in _golden("keysets_eq4.json")["cases"]:
        T, w, z = case["T"], case["w"], np.array(case["z"], dtype=np.uint8)
        d = T
        Q = np.zeros((T, 1, d))
        K = np.random.default_rng(4).standard_normal((T, 1, d))
        V = np.eye(T).reshape(T, 1, d)
        o, lse = O.gated_attention(Q, K, V, z.reshape(T, 1), w, np.arange(T))
        for t in range(T):
            want = np.zeros(T)
            want[case["S"][t]] = 1.0 / len(case["S"][t])
            _close(o[t, 0], want, 1e-15, f"key set T={T} w={w} t={t}")
            _close([lse[t, 0]], [math.log(len(case["S"][t]))], 1e-15, "lse")


def pin_two_key_softmax():
    """Two visible keys with scaled logits 1 and 0 (d_k = 4, so q.k = 2 and 0):
    weights e/(e+1) and 1/(e+1); lse = ln(e + 1)."""
    q = np.array([2.0, 0.0, 0.0, 0.0])
    K = np.array([[1.0, 0, 0, 0], [0.0, 0, 0, 0]])
    V = np.array([[1.0, 0, 0, 0], [0.0, 1, 0, 0]])
    o, lse = O.attend(q, K, V, np.array([True, True]))
    p = math.e / (math.e + 1)
    _close(o, [p, 1 - p, 0, 0], 1e-15, "two-key softmax")
    _close([lse], [math.log(math.e + 1)], 1e-15, "two-key lse")


def pin_tau0_is_causal():
    """tau = 0 gates every key in (u > 0), so Eqs. (3)-(4) reduce to causal
    attention: torch SDPA (is_causal) in fp64."""
    rng = np.random.default_rng(5)
    T, Hq, Hkv, d, w = 40, 4, 2, 8, 5
    Q, K, V = _rand_qkv(rng, T, Hq, Hkv, d)
    h, W1, b1, W2, b2 = _mlp(rng, T, 6, 5, Hkv)
    z = O.gate(O.utility(h, W1, b1, W2, b2), 0.0)
    o, _ = O.gated_attention(Q, K, V, z, w, np.arange(T))
    _close(o, _sdpa(Q, K, V, None), 1e-12, "tau=0 vs causal SDPA")


def pin_tau_gt1_is_sliding_window():
    """tau > 1 gates every key out (u < 1), leaving sliding-window-w attention:
    torch SDPA with a band mask built from tril."""
    rng = np.random.default_rng(6)
    T, Hq, Hkv, d, w = 40, 4, 2, 8, 6
    Q, K, V = _rand_qkv(rng, T, Hq, Hkv, d)
    h, W1, b1, W2, b2 = _mlp(rng, T, 6, 5, Hkv)
    z = O.gate(O.utility(h, W1, b1, W2, b2), 1.5)
    o, _ = O.gated_attention(Q, K, V, z, w, np.arange(T))
    ones = torch.ones(T, T, dtype=torch.bool)
    band = (ones.tril(0) & ~ones.tril(-w)).numpy()
    _close(o, _sdpa(Q, K, V, band), 1e-12, "tau>1 vs sliding-window SDPA")


def pin_wide_window_is_causal():
    """w >= T puts every earlier key in the window whatever z is."""
    rng = np.random.default_rng(7)
    T, Hq, Hkv, d = 30, 2, 1, 8
    Q, K, V = _rand_qkv(rng, T, Hq, Hkv, d)
    z = (rng.random((T, Hkv)) < 0.3).astype(np.uint8)
    o, _ = O.gated_attention(Q, K, V, z, T, np.arange(T))
    _close(o, _sdpa(Q, K, V, None), 1e-12, "w>=T vs causal SDPA")


def pin_dense_brute_force(seeds=200):
    """Tiny inputs: enumerate Eq. (4) with explicit loops into a dense T x T mask and
    compute the masked softmax densely (whole matrices); compare per query."""
    for seed in range(seeds):
        rng = np.random.default_rng(1000 + seed)
        T = int(rng.integers(1, 20))
        w = int(rng.choice([1, 2, 4, 8]))
        Hkv, G, d = 1 + seed % 2, 1 + (seed // 2) % 2, 4
        Hq = Hkv * G
        Q, K, V = _rand_qkv(rng, T, Hq, Hkv, d)
        z = (rng.random((T, Hkv)) < 0.4).astype(np.uint8)
        o, _ = O.gated_attention(Q, K, V, z, w, np.arange(T))
        for hk in range(Hkv):
            M = np.full((T, T), -np.inf)
            for t in range(T):
                for s in range(T):
                    if (0 <= t - s < w) or (z[s, hk] == 1 and s <= t):
                        M[t, s] = 0.0
            for g in range(G):
                hq = hk * G + g
                S = Q[:, hq] @ K[:, hk].T / math.sqrt(d) + M
                P = np.exp(S - S.max(axis=1, keepdims=True))
                P /= P.sum(axis=1, keepdims=True)
                _close(o[:, hq], P @ V[:, hk], 1e-12, f"brute force seed {seed}")


def pin_cache_rows():
    """The persistent cache is the increasing list of gated-in positions; its length
    is the kept count sum(z); together with the window it is exactly the visible set
    of Eq. (4) for every query."""
    rng = np.random.default_rng(8)
    for w in (1, 3, 16):
        T = 60
        z = (rng.random(T) < 0.35).astype(np.uint8)
        for upto in (0, 1, 17, T):
            rows = O.cache_rows(z, upto)
            assert len(rows) == int(z[:upto].sum())
            assert list(rows) == [s for s in range(upto) if z[s] == 1]
            assert np.all(np.diff(rows) > 0)
        s = np.arange(T)
        for t in range(T):
            window = set(range(max(0, t - w + 1), t + 1))
            cached = set(O.cache_rows(z, max(0, t - w + 1)).tolist())
            assert set(np.nonzero(O.visible(t, s, z, w))[0].tolist()) == window | cached


def pin_rethreshold():
    """Post-hoc threshold change (§3.3): a hand example with a row exactly at the new
    threshold (kept: Eq. (2) uses >=), the extremes, and the composition law: gating at
    tau then re-thresholding at tau' gives the cache gated at max(tau, tau')."""
    pos = np.array([2, 5, 7, 9], dtype=np.int32)
    u = np.array([0.55, 0.7, 0.6, 0.9])
    assert O.rethreshold(pos, u, 0.6).tolist() == [5, 7, 9]
    assert O.rethreshold(pos, u, 0.95).tolist() == []
    assert O.rethreshold(pos, u, 0.5).tolist() == [2, 5, 7, 9]
    assert O.rethreshold(pos[:0], u[:0], 0.5).tolist() == []
    rng = np.random.default_rng(11)
    for _ in range(50):
        T = int(rng.integers(1, 200))
        uu = rng.random(T)
        tau, tau2 = rng.random(2)
        cached = O.cache_rows(O.gate(uu, tau), T)
        again = O.rethreshold(cached, uu[cached], tau2)
        assert again.tolist() == O.cache_rows(O.gate(uu, max(tau, tau2)), T).tolist()


def pin_soft_gate_values():
    """Eq. (5) at hand-picked points: u = tau gives 1/2; u - tau = +-beta gives the
    logistic function at +-1; large |u - tau| / beta saturates to 0 or 1."""
    g = O.soft_gate(np.array([0.5, 0.51, 0.49, 0.9, 0.1]), 0.5, 0.01)
    _close(g[0], 0.5, 1e-15, "alpha at u = tau")
    _close(g[1], 1.0 / (1.0 + math.exp(-1.0)), 1e-12, "alpha at u = tau + beta")
    _close(g[2], 1.0 / (1.0 + math.exp(1.0)), 1e-12, "alpha at u = tau - beta")
    _close(g[3:], [1.0, 0.0], 1e-15, "saturation")


def pin_soft_two_key_closed_form():
    """Eq. (6) by hand: one query at t = 1, w = 1, two keys with equal scores (q = 0);
    key 0 lies outside the window and gets c (alpha - 1) with alpha = 1/2 (u = tau),
    key 1 is the window.  With c = 2 the weights are e^{-1} : 1."""
    Q = np.zeros((1, 1, 4))
    K = np.zeros((2, 1, 4))
    V = np.array([[[1.0, 0.0, 0.0, 0.0]], [[0.0, 1.0, 0.0, 0.0]]])
    u = np.array([[0.5], [0.9]])
    o, lse = O.soft_gated_attention(Q, K, V, u, 0.5, 0.01, 2.0, 1, [1])
    e = math.exp(-1.0)
    _close(o[0, 0], [e / (1 + e), 1 / (1 + e), 0.0, 0.0], 1e-12, "two-key soft mask")
    _close(lse[0, 0], math.log(1 + e), 1e-12, "two-key lse")
    # the key after the query never counts, whatever its utility
    o2, _ = O.soft_gated_attention(Q, K, V, u, 0.5, 0.01, 2.0, 1, [0])
    _close(o2[0, 0], [1.0, 0.0, 0.0, 0.0], 1e-15, "causal")


def pin_soft_special_cases():
    """c = 0 and w >= T reduce Eq. (6) to causal attention (torch SDPA, fp64); with a
    vanishing temperature and utilities away from tau, the soft mask equals the hard
    gate of Eq. (4) (the pinned ``gated_attention``)."""
    rng = np.random.default_rng(21)
    T, Hq, Hkv, d, w = 40, 4, 2, 16, 6
    Q, K, V = _rand_qkv(rng, T, Hq, Hkv, d)
    u = rng.random((T, Hkv))
    u = np.where(np.abs(u - 0.5) < 0.02, u + 0.05, u)
    causal = np.tril(np.ones((T, T), dtype=bool))
    ref = _sdpa(Q, K, V, causal)
    o, _ = O.soft_gated_attention(Q, K, V, u, 0.5, 0.01, 0.0, w, np.arange(T))
    _close(o, ref, 1e-12, "c = 0 is causal attention")
    o, _ = O.soft_gated_attention(Q, K, V, u, 0.5, 0.01, 1e6, T, np.arange(T))
    _close(o, ref, 1e-12, "w >= T is causal attention")
    o_soft, _ = O.soft_gated_attention(Q, K, V, u, 0.5, 1e-12, 1e6, w, np.arange(T))
    o_hard, _ = O.gated_attention(Q, K, V, O.gate(u, 0.5), w, np.arange(T))
    _close(o_soft, o_hard, 1e-12, "beta -> 0 is the hard gate")


def pin_permutation_invariance():
    """Eq. (3) is a sum over the key set: listing the visible keys in another order (as
    a cache whose rows were written in another order would) changes nothing but
    rounding."""
    rng = np.random.default_rng(21)
    for _ in range(50):
        T, d = int(rng.integers(2, 40)), 8
        q = rng.standard_normal(d)
        K = rng.standard_normal((T, d))
        V = rng.standard_normal((T, d))
        mask = rng.random(T) < 0.6
        mask[int(rng.integers(T))] = True  # at least one key
        perm = rng.permutation(T)
        o1, l1 = O.attend(q, K, V, mask)
        o2, l2 = O.attend(q, K[perm], V[perm], mask[perm])
        _close(o1, o2, 1e-12, "permuted keys: output")
        _close(np.array([l1]), np.array([l2]), 1e-12, "permuted keys: lse")


def pin_merge_of_slices():
    """Eq. (3) over a key set split into disjoint slices: merging the attention of each
    slice alone (``merge``) gives the attention over the union (``attend`` on the whole
    set), output and lse, for random splits into 1-4 slices, empty slices included; a
    hand example with two one-key slices gives the two-key softmax."""
    rng = np.random.default_rng(31)
    for _ in range(100):
        T, d = int(rng.integers(1, 50)), 8
        q = rng.standard_normal(d) * 2.0
        K = rng.standard_normal((T, d))
        V = rng.standard_normal((T, d))
        mask = rng.random(T) < 0.7
        mask[int(rng.integers(T))] = True
        n = int(rng.integers(1, 5))
        part = rng.integers(0, n + 1, size=T)  # slice n never used when drawn: an extra empty one
        o_full, l_full = O.attend(q, K, V, mask)
        os_, ls_ = [], []
        for i in range(n + 1):
            sub = mask & (part == i)
            if sub.any():
                o_i, l_i = O.attend(q, K, V, sub)
            else:
                o_i, l_i = np.zeros(d), -np.inf
            os_.append(o_i)
            ls_.append(l_i)
        o_m, l_m = O.merge(np.stack(os_), np.array(ls_))
        _close(o_m, o_full, 1e-12, "merged slices: output")
        _close(np.array([l_m]), np.array([l_full]), 1e-12, "merged slices: lse")
    # two one-key slices: weights e^{x1} : e^{x2}
    o_m, l_m = O.merge(np.array([[1.0, 0.0], [0.0, 1.0]]), np.array([0.0, math.log(3.0)]))
    _close(o_m, np.array([0.25, 0.75]), 1e-15, "two one-key slices")
    _close(np.array([l_m]), np.array([math.log(4.0)]), 1e-15, "two one-key slices: lse")
    o_m, l_m = O.merge(np.zeros((2, 3)), np.array([-np.inf, -np.inf]))
    assert np.all(o_m == 0.0) and l_m == -np.inf, "all slices empty"


ALL_PINS = [
    pin_gelu_textbook, pin_gelu_library, pin_utility_zero_weights, pin_utility_hand_example,
    pin_utility_library, pin_gate_threshold, pin_gate_extremes, pin_keysets_golden,
    pin_two_key_softmax, pin_tau0_is_causal, pin_tau_gt1_is_sliding_window,
    pin_wide_window_is_causal, pin_dense_brute_force, pin_cache_rows, pin_rethreshold,
    pin_soft_gate_values, pin_soft_two_key_closed_form, pin_soft_special_cases,
    pin_permutation_invariance, pin_merge_of_slices,
]
