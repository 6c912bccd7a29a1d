"""Plant plausible mistakes in the oracle (on the CPU) and check that some pin
catches each one: the pins are strong enough to trust the oracle."""
import numpy as np
import pytest
from scipy.special import erf

from oracle import spkv_oracle as O
from tests import oracle_pins as P


def _gelu_tanh(a):
    a = np.asarray(a, dtype=np.float64)
    return 0.5 * a * (1 + np.tanh(np.sqrt(2 / np.pi) * (a + 0.044715 * a ** 3)))


def _visible_window_off_by_one(t, s, z, w):
    s = np.asarray(s)
    return ((t - s >= 0) & (t - s <= w)) | ((np.asarray(z) == 1) & (s <= t))


def _visible_ignores_z(t, s, z, w):
    s = np.asarray(s)
    return (t - s >= 0) & (t - s < w)


def _visible_acausal(t, s, z, w):
    s = np.asarray(s)
    return ((t - s >= 0) & (t - s < w)) | (np.asarray(z) == 1)


def _gate_strict(u, tau):
    return (np.asarray(u, dtype=np.float64) > tau).astype(np.uint8)


def _attend_no_scale(q, K, V, mask):
    return _ORIG_ATTEND(np.asarray(q) * np.sqrt(np.asarray(q).shape[-1]), K, V, mask)


def _utility_no_b1(h, W1, b1, W2, b2):
    return _ORIG_LOGITS(h, W1, np.zeros_like(np.asarray(b1, dtype=np.float64)), W2, b2)


def _sigmoid_flipped(x):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(np.asarray(x, dtype=np.float64)))


def _gqa_modulo(Q, K, V, z, w, q_pos):
    # query head h reads key head h % Hkv instead of h // G
    Q = np.asarray(Q, dtype=np.float64)
    n_q, Hq, d = Q.shape
    T, Hkv, _ = np.asarray(K).shape
    o = np.zeros((n_q, Hq, d)); lse = np.zeros((n_q, Hq))
    for i, t in enumerate(q_pos):
        for h in range(Hq):
            hk = h % Hkv
            m = O.visible(int(t), np.arange(T), z[:, hk], w)
            o[i, h], lse[i, h] = O.attend(Q[i, h], np.asarray(K)[:, hk], np.asarray(V)[:, hk], m)
    return o, lse


def _gelu_wrong_scale(a):
    a = np.asarray(a, dtype=np.float64)
    return 0.5 * a * (1 + erf(a))


def _rethreshold_strict(cached_pos, cached_u, tau_new):
    keep = np.asarray(cached_u, dtype=np.float64) > tau_new
    return np.asarray(cached_pos)[keep].astype(np.int32)


def _rethreshold_inverted(cached_pos, cached_u, tau_new):
    keep = np.asarray(cached_u, dtype=np.float64) < tau_new
    return np.asarray(cached_pos)[keep].astype(np.int32)


def _soft_gate_flipped(u, tau, beta):
    return O.sigmoid((float(tau) - np.asarray(u, dtype=np.float64)) / float(beta))


def _soft_mask_window_off_by_one(t, s, alpha, w, c):
    s = np.asarray(s, dtype=np.int64)
    m = np.where(t - s <= w, 0.0, float(c) * (np.asarray(alpha) - 1.0))
    return np.where(s <= t, m, -np.inf)


def _soft_mask_sign(t, s, alpha, w, c):
    s = np.asarray(s, dtype=np.int64)
    m = np.where(t - s < w, 0.0, float(c) * (1.0 - np.asarray(alpha)))
    return np.where(s <= t, m, -np.inf)


def _soft_mask_acausal(t, s, alpha, w, c):
    s = np.asarray(s, dtype=np.int64)
    return np.where((t - s < w) & (t - s >= 0), 0.0, float(c) * (np.asarray(alpha) - 1.0))


def _attend_lse_without_max(q, K, V, mask):
    o, lse = _ORIG_ATTEND(q, K, V, mask)
    logits = np.where(mask, (np.asarray(K, dtype=np.float64) @ np.asarray(q, dtype=np.float64))
                      / np.sqrt(len(q)), -np.inf)
    return o, lse - np.max(logits)  # the max subtracted for stability never added back


def _cache_rows_inclusive(z_col, upto):
    z_col = np.asarray(z_col, dtype=np.uint8)[:upto + 1]  # one row past the boundary
    return np.nonzero(z_col == 1)[0].astype(np.int32)


def _utility_no_gelu(h, W1, b1, W2, b2):
    a = np.asarray(h, dtype=np.float64) @ np.asarray(W1, dtype=np.float64).T + np.asarray(b1)
    return a @ np.asarray(W2, dtype=np.float64).T + np.asarray(b2)


def _soft_gate_no_beta(u, tau, beta):
    return O.sigmoid(np.asarray(u, dtype=np.float64) - float(tau))


def _merge_unweighted(o_parts, lse_parts):
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    live = np.isfinite(lse_parts)
    o = np.sum(o_parts * live[..., None], axis=0) / np.maximum(np.sum(live, axis=0), 1)[..., None]
    m = np.max(lse_parts, axis=0)
    return o, np.where(np.isfinite(m), np.log(np.sum(np.exp(lse_parts), axis=0)), -np.inf)


def _merge_lse_is_max(o_parts, lse_parts):
    o, _ = _ORIG_MERGE(o_parts, lse_parts)
    return o, np.max(np.asarray(lse_parts, dtype=np.float64), axis=0)


_ORIG_ATTEND = O.attend
_ORIG_LOGITS = O.utility_logits
_ORIG_MERGE = O.merge

MUTANTS = {
    "gelu_tanh_approximation": ("gelu", _gelu_tanh),
    "gelu_missing_sqrt2": ("gelu", _gelu_wrong_scale),
    "window_off_by_one": ("visible", _visible_window_off_by_one),
    "gate_ignored": ("visible", _visible_ignores_z),
    "gated_keys_not_causal": ("visible", _visible_acausal),
    "gate_strict_inequality": ("gate", _gate_strict),
    "missing_inv_sqrt_dk": ("attend", _attend_no_scale),
    "lse_without_max": ("attend", _attend_lse_without_max),
    "dropped_b1": ("utility_logits", _utility_no_b1),
    "sigmoid_sign": ("sigmoid", _sigmoid_flipped),
    "gqa_modulo_mapping": ("gated_attention", _gqa_modulo),
    "rethreshold_strict_inequality": ("rethreshold", _rethreshold_strict),
    "rethreshold_inverted": ("rethreshold", _rethreshold_inverted),
    "soft_gate_flipped": ("soft_gate", _soft_gate_flipped),
    "soft_gate_missing_beta": ("soft_gate", _soft_gate_no_beta),
    "cache_rows_past_boundary": ("cache_rows", _cache_rows_inclusive),
    "perceptron_without_gelu": ("utility_logits", _utility_no_gelu),
    "soft_window_off_by_one": ("soft_mask", _soft_mask_window_off_by_one),
    "soft_bias_sign": ("soft_mask", _soft_mask_sign),
    "soft_not_causal": ("soft_mask", _soft_mask_acausal),
    "merge_unweighted_mean": ("merge", _merge_unweighted),
    "merge_lse_is_the_max": ("merge", _merge_lse_is_max),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for pin in P.ALL_PINS:
        try:
            if pin is P.pin_dense_brute_force:
                pin(seeds=40)
            else:
                pin()
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
