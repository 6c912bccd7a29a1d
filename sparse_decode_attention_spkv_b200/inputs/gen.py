"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds no SP-KV arithmetic: it only turns (seed, stream ids, element
index) into numbers.  The same definition is implemented for the device in
``inputs_gen.cu`` so that large workloads can be drawn in HBM, while any slice of
them can be regenerated here on the host.

Definition (applies to both implementations):

* ``mix64`` is the output function of Vigna's SplitMix64 generator
  (xor-shift 30 / multiply 0xBF58476D1CE4E5B9 / xor-shift 27 /
  multiply 0x94D049BB133111EB / xor-shift 31), all arithmetic mod 2**64.
* A stream key is derived from a seed and a tuple of small integer ids by
  ``key = seed; key = mix64(key + (id + 1) * GAMMA)`` for each id, with
  GAMMA = 0x9E3779B97F4A7C15 (the SplitMix64 increment).
* Draw ``i`` of a stream is ``d = mix64(key + (i + 1) * GAMMA)``.
* Uniforms: ``u1 = (d >> 32 + 0.5) / 2**32``, ``u2 = (d & 0xffffffff + 0.5) / 2**32``,
  both in (0, 1), computed in fp64.
* Normal (Box-Muller, cosine branch only): ``n = sqrt(-2 ln u1) * cos(2 pi u2)``
  in fp64; then ``x = n * scale`` in fp64, rounded to fp32 (round to nearest),
  and for bf16 tensors rounded again fp32 -> bf16 (round to nearest even).
* Uniform in [lo, hi): ``lo + (hi - lo) * u2`` in fp64.

fp64 ``log``/``cos``/``sqrt`` of the host C library and of CUDA may differ in the
last ulp; after rounding to fp32 or bf16 such a difference survives with a
probability of order 1e-9 (fp32) or 1e-13 (bf16) per value.  Small parity cases
are drawn on the host and copied, so they are exact by construction.
"""
from __future__ import annotations

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB

# Tensor kinds: stream ids used by every workload.
T_H = 1        # hidden states h
T_W1 = 2       # first utility-MLP layer
T_B1 = 3
T_W2 = 4       # second utility-MLP layer
T_Q = 5
T_K = 6
T_V = 7
T_KEEP = 8     # per-head target keep rates
T_CTX = 9      # per-row context lengths
T_CAL = 10     # calibration draw of hidden states
T_QDEC = 11    # per-step decode queries
T_KDEC = 12    # per-step decode keys
T_VDEC = 13    # per-step decode values
T_HDEC = 14    # per-step decode hidden states
T_U = 15       # utilities drawn directly (inputs of the soft-gated attention tests)


def _mix64_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * M1) & MASK64
    z = ((z ^ (z >> 27)) * M2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, *ids: int) -> int:
    """Key of the stream named by ``ids`` under ``seed`` (Python ints, exact)."""
    key = seed & MASK64
    for i in ids:
        key = _mix64_int(key + ((int(i) + 1) * GAMMA))
    return key


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * np.uint64(M1)
    z = z ^ (z >> np.uint64(27))
    z = z * np.uint64(M2)
    return z ^ (z >> np.uint64(31))


def draws(key: int, index: np.ndarray) -> np.ndarray:
    """64-bit draws ``mix64(key + (i+1)*GAMMA)`` for an array of indices."""
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        state = np.uint64(key) + (idx + np.uint64(1)) * np.uint64(GAMMA)
        return _mix64(state)


def _uniforms(d: np.ndarray):
    hi = (d >> np.uint64(32)).astype(np.float64)
    lo = (d & np.uint64(0xFFFFFFFF)).astype(np.float64)
    return (hi + 0.5) * (2.0 ** -32), (lo + 0.5) * (2.0 ** -32)


def normal_f64(key: int, index: np.ndarray, scale: float = 1.0) -> np.ndarray:
    """fp64 values ``scale * N(0,1)`` before any rounding."""
    u1, u2 = _uniforms(draws(key, index))
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2) * scale


def uniform_f64(key: int, index: np.ndarray, lo: float, hi: float) -> np.ndarray:
    _, u2 = _uniforms(draws(key, index))
    return lo + (hi - lo) * u2


def to_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest even); returns the 16-bit patterns."""
    b = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to(x64: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 values the way the generator stores them; result as fp32 values
    (exactly representable in ``dtype``)."""
    x32 = to_f32(x64)
    if dtype == "f32":
        return x32
    if dtype == "bf16":
        return bf16_bits_to_f32(f32_to_bf16_bits(x32))
    raise ValueError(dtype)


def normal(key: int, shape, scale: float, dtype: str, offset: int = 0) -> np.ndarray:
    """Tensor of ``shape`` whose flat element ``j`` is draw ``offset + j``."""
    n = int(np.prod(shape))
    idx = np.arange(offset, offset + n, dtype=np.uint64)
    return round_to(normal_f64(key, idx, scale), dtype).reshape(shape)


def normal_rows(key: int, row_len: int, rows: np.ndarray, scale: float, dtype: str) -> np.ndarray:
    """Selected rows of a row-major tensor with ``row_len`` elements per row."""
    rows = np.asarray(rows, dtype=np.uint64).reshape(-1, 1)
    idx = rows * np.uint64(row_len) + np.arange(row_len, dtype=np.uint64)[None, :]
    return round_to(normal_f64(key, idx.reshape(-1), scale), dtype).reshape(len(rows), row_len)


def rope_rows(key: int, head_dim: int, n_heads: int, rows: np.ndarray, positions: np.ndarray,
              scale: float, base: float, dtype: str) -> np.ndarray:
    """Rows of a [tokens][n_heads][head_dim] tensor with rotary position embedding
    (rotate-half pairing (i, i + head_dim/2), angle = position * base**(-2i/head_dim))
    applied in fp64 before rounding.  ``rows`` are token indices into the tensor,
    ``positions`` their absolute positions."""
    rows = np.asarray(rows, dtype=np.uint64)
    row_len = n_heads * head_dim
    idx = rows.reshape(-1, 1) * np.uint64(row_len) + np.arange(row_len, dtype=np.uint64)[None, :]
    x = normal_f64(key, idx.reshape(-1), scale).reshape(len(rows), n_heads, head_dim)
    half = head_dim // 2
    i = np.arange(half, dtype=np.float64)
    theta = np.power(float(base), -2.0 * i / head_dim)
    ang = np.asarray(positions, dtype=np.float64).reshape(-1, 1, 1) * theta[None, None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    y = np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)
    return round_to(y, dtype)
