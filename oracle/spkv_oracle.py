"""Oracle for Self-Pruned KV attention (SP-KV): plain, slow fp64 CPU reference.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or run this module.  It shares no
code with the CUDA library; both sides receive the same seeded inputs from
``sparse_decode_attention_spkv_b200.inputs``.

Every function restates one passage of "Self-Pruned Key-Value Attention:
Learning When to Write by Predicting Future Utility" (arXiv 2605.14037):

* ``utility``          §2.1, Eq. (1): u = sigmoid(f(h)), f a 2-layer perceptron.
* ``gate``             §2.1, Eq. (2): z = 1[u >= tau].
* ``visible``          §2.1, Eq. (4): M = 0 iff 0 <= t-s < w, or (z_s = 1 and s <= t).
* ``attend``           §2.1, Eq. (3): softmax(q k^T / sqrt(d_k) + M) V.
* ``gated_attention``  Eqs. (3)-(4) for a set of queries over all heads (GQA:
                       query head h reads key head h // (Hq/Hkv), §1).
* ``cache_rows``       §2.1 "efficient implementation at deployment": the
                       persistent cache holds exactly the KV pairs with z = 1.
* ``rethreshold``      §3.3 (end of "Hybrids"): sparsity can be changed after the
                       fact by changing the threshold; with the stored utility of
                       every cached row, the cache for tau' keeps the rows with
                       u >= tau' (rows dropped earlier cannot come back).
* ``soft_gate``        §2.1 "soft relaxation at training time", Eq. (5):
                       alpha_s = sigmoid((u_s - tau) / beta).
* ``soft_mask``        Eq. (6): additive score 0 inside the causal window,
                       c (alpha_s - 1) outside it (and -inf for s > t: causal).
* ``soft_gated_attention``  Eq. (3) with the mask of Eq. (6), every key s <= t.
* ``merge``            Eq. (3) over a key set split into disjoint slices: the
                       softmax factorises, so the slices' outputs combine by their
                       log-sum-exp weights (a sequence decoded slice by slice).

Readings where the page is silent (each listed in the design notes):
* f is one perceptron per layer, d_model -> hid -> Hkv, with a GELU (exact erf
  form) between the layers; Eq. (1) indexes one output per key head.
* Inputs are the values the generator stored (fp32, or bf16 widened exactly);
  all arithmetic here is fp64.

Parity status: every function here is pinned by the CPU tests in
``tests/test_oracle_pins.py`` (closed forms, library special cases, a
hand-derived key-set fixture, brute force and invariants).
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

SQRT2 = np.sqrt(2.0)


def gelu(a: np.ndarray) -> np.ndarray:
    """GELU in its exact form a * Phi(a) = 0.5 a (1 + erf(a / sqrt 2))."""
    a = np.asarray(a, dtype=np.float64)
    return 0.5 * a * (1.0 + erf(a / SQRT2))


def sigmoid(x: np.ndarray) -> np.ndarray:
    """Logistic function, evaluated without overflow for large |x|."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def utility_logits(h, W1, b1, W2, b2) -> np.ndarray:
    """f(h) of Eq. (1): layer 1 (d_model -> hid), GELU, layer 2 (hid -> Hkv).

    h [N][d_model], W1 [hid][d_model], b1 [hid], W2 [Hkv][hid], b2 [Hkv];
    returns the pre-sigmoid logits [N][Hkv]."""
    h = np.asarray(h, dtype=np.float64)
    a = h @ np.asarray(W1, dtype=np.float64).T + np.asarray(b1, dtype=np.float64)
    x = gelu(a)
    return x @ np.asarray(W2, dtype=np.float64).T + np.asarray(b2, dtype=np.float64)


def utility(h, W1, b1, W2, b2) -> np.ndarray:
    """Eq. (1): u_s = sigmoid(f(h_s)) in (0, 1), one value per key head."""
    return sigmoid(utility_logits(h, W1, b1, W2, b2))


def gate(u, tau: float) -> np.ndarray:
    """Eq. (2): z_s = 1[u_s >= tau] (uint8)."""
    return (np.asarray(u, dtype=np.float64) >= float(tau)).astype(np.uint8)


def visible(t: int, s: np.ndarray, z: np.ndarray, w: int) -> np.ndarray:
    """Eq. (4) as a boolean: key s is visible to query t when it lies in the causal
    window (0 <= t - s < w) or when it was gated in (z_s = 1) and s <= t."""
    s = np.asarray(s, dtype=np.int64)
    in_win = (t - s >= 0) & (t - s < w)
    gated = (np.asarray(z, dtype=np.uint8) == 1) & (s <= t)
    return in_win | gated


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, mask: np.ndarray):
    """Eq. (3) for one query row: softmax over visible keys of q.k / sqrt(d_k).

    Returns (o, lse): the output row and the natural-log sum of exponentials of
    the scaled logits over the visible keys."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    d_k = q.shape[-1]
    logits = (K @ q) / np.sqrt(d_k)
    logits = np.where(mask, logits, -np.inf)
    m = np.max(logits)
    p = np.exp(logits - m)
    l = np.sum(p)
    return (p @ V) / l, m + np.log(l)


def gated_attention(Q, K, V, z, w: int, q_pos):
    """Eqs. (3)-(4) for one batch row.

    Q [n_q][Hq][d] queries at absolute positions q_pos [n_q];
    K, V [T][Hkv][d] keys/values of positions 0..T-1;
    z [T][Hkv] gates.  Returns o [n_q][Hq][d] and lse [n_q][Hq]."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    n_q, Hq, d = Q.shape
    T, Hkv, _ = K.shape
    G = Hq // Hkv
    s = np.arange(T)
    o = np.zeros((n_q, Hq, d))
    lse = np.zeros((n_q, Hq))
    for i, t in enumerate(q_pos):
        for hk in range(Hkv):
            mask = visible(int(t), s, z[:, hk], w)
            for g in range(G):
                h = hk * G + g
                o[i, h], lse[i, h] = attend(Q[i, h], K[:, hk], V[:, hk], mask)
    return o, lse


def cache_rows(z_col: np.ndarray, upto: int) -> np.ndarray:
    """Deployment (§2.1): the persistent cache of one key head holds the positions
    s < upto whose gate is 1, in increasing order (its "index list")."""
    z_col = np.asarray(z_col, dtype=np.uint8)[:upto]
    return np.nonzero(z_col == 1)[0].astype(np.int32)


def merge(o_parts, lse_parts):
    """Eq. (3) over the disjoint union of slices S_1..S_n of a key set: with o_i the
    attention output over S_i alone and lse_i = log sum_{s in S_i} e^{x_s},
    lse = log sum_i e^{lse_i} and o = sum_i e^{lse_i - lse} o_i.

    o_parts [n][..][d], lse_parts [n][..]; slices without keys (lse = -inf) count for
    nothing; if all are empty, o = 0 and lse = -inf.  Returns (o, lse)."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = np.max(lse_parts, axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    wgt = np.where(np.isfinite(lse_parts), np.exp(lse_parts - m_safe), 0.0)
    total = np.sum(wgt, axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(finite, total, 1.0)), -np.inf)
    scale = np.where(finite, 1.0 / np.where(finite, total, 1.0), 0.0)
    o = np.einsum("n...,n...d->...d", wgt * scale, o_parts)
    return o, lse


def rethreshold(cached_pos: np.ndarray, cached_u: np.ndarray, tau_new: float) -> np.ndarray:
    """Post-hoc threshold change (§3.3) applied to one key head's cache: of the cached
    positions (increasing) with their stored utilities, keep those with u >= tau_new,
    in the same order.  Eq. (2) with the new threshold, restricted to what is stored."""
    cached_pos = np.asarray(cached_pos, dtype=np.int64)
    keep = np.asarray(cached_u, dtype=np.float64) >= float(tau_new)
    return cached_pos[keep].astype(np.int32)


def soft_gate(u, tau: float, beta: float) -> np.ndarray:
    """Eq. (5): the differentiable stand-in for z, alpha = sigmoid((u - tau) / beta)."""
    return sigmoid((np.asarray(u, dtype=np.float64) - float(tau)) / float(beta))


def soft_mask(t: int, s: np.ndarray, alpha: np.ndarray, w: int, c: float) -> np.ndarray:
    """Eq. (6) for query t over keys s: 0 when 0 <= t - s < w (the causal window),
    c (alpha_s - 1) for the older keys, -inf for keys after t (causal language model)."""
    s = np.asarray(s, dtype=np.int64)
    alpha = np.asarray(alpha, dtype=np.float64)
    m = np.where(t - s < w, 0.0, float(c) * (alpha - 1.0))
    return np.where(s <= t, m, -np.inf)


def soft_gated_attention(Q, K, V, u, tau: float, beta: float, c: float, w: int, q_pos):
    """Eqs. (3), (5), (6) for one batch row: softmax(q k^T / sqrt(d_k) + M_soft) V.

    Q [n_q][Hq][d] at positions q_pos; K, V [T][Hkv][d]; u [T][Hkv] utilities.
    Returns o [n_q][Hq][d] and lse [n_q][Hq] (natural log)."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    n_q, Hq, d = Q.shape
    T, Hkv, _ = K.shape
    G = Hq // Hkv
    s = np.arange(T)
    alpha = soft_gate(u, tau, beta)
    o = np.zeros((n_q, Hq, d))
    lse = np.zeros((n_q, Hq))
    for i, t in enumerate(q_pos):
        for hk in range(Hkv):
            M = soft_mask(int(t), s, alpha[:, hk], w, c)
            logits_k = K[:, hk] / np.sqrt(d)
            for g in range(G):
                h = hk * G + g
                x = logits_k @ Q[i, h] + M
                m = np.max(x)
                p = np.exp(x - m)
                l = np.sum(p)
                o[i, h] = (p @ V[:, hk]) / l
                lse[i, h] = m + np.log(l)
    return o, lse
