"""Helpers shared by the GPU parity tests: seeded host inputs, the oracle's
expectations for them, and device copies.  Expected values come only from
``oracle/``; the CUDA path gets the same inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import spkv_oracle as O
from oracle.calibrate import calibrate
from sparse_decode_attention_spkv_b200.inputs import workloads as W

EXCLUDE = 1e-4   # |u - tau| below this: gate parity not required (near-threshold tokens)
TOL = {"f32": dict(max_abs=2e-3, rel=None), "bf16": dict(max_abs=2e-2, rel=1e-2)}


def weights(wl: W.Workload, layer: int = 0):
    """Host W1, b1, W2, b2 of a workload layer; b2 from the stored calibration when
    the workload is one of the five, else calibrated here by the oracle."""
    table = W.load_biases()
    if wl.name in table and wl.cid == W.WORKLOADS[wl.name].cid and \
            len(table[wl.name]["b2"][layer]) == wl.Hkv and wl.d_model == W.WORKLOADS[wl.name].d_model \
            and wl.hid == W.WORKLOADS[wl.name].hid:
        b2 = np.asarray(table[wl.name]["b2"][layer], dtype=np.float32)
    else:
        b2 = np.asarray(calibrate(wl, n_cal=2048)["b2"][layer], dtype=np.float32)
    return wl.w1(layer), wl.b1(layer), wl.w2(layer), b2


def host_rows(wl: W.Workload, layer: int, b: int, positions):
    """h, q, k, v host rows (fp32 values exactly representable in the dtype)."""
    return (wl.h_rows(layer, b, positions), wl.q_rows(layer, b, positions),
            wl.k_rows(layer, b, positions), wl.v_rows(layer, b, positions))


def dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.cuda()


def dev_f32(x) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def oracle_gates(h, W1, b1, W2, b2, tau):
    u = O.utility(h, W1, b1, W2, b2)
    return u, O.gate(u, tau)


def check_gates(u_gpu, z_gpu, u_ref, z_ref, tau, u_tol=1e-5):
    """u within u_tol; z bit-exact except where the oracle's u is within EXCLUDE of tau."""
    u_gpu = np.asarray(u_gpu, dtype=np.float64)
    z_gpu = np.asarray(z_gpu)
    assert u_gpu.shape == u_ref.shape
    err = np.max(np.abs(u_gpu - u_ref)) if u_ref.size else 0.0
    assert err <= u_tol, f"u max abs error {err:.3e}"
    near = np.abs(u_ref - tau) < EXCLUDE
    bad = (z_gpu != z_ref) & ~near
    assert not bad.any(), f"{int(bad.sum())} gates differ away from the threshold"
    return int(near.sum())


def check_attn(o_gpu, o_ref, dtype: str, what: str = ""):
    """Per-row max-abs bound, plus (bf16) per-row relative L2 bound."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    tol = TOL[dtype]
    err = np.max(np.abs(o_gpu - o_ref)) if o_ref.size else 0.0
    assert err <= tol["max_abs"], f"{what}: max abs error {err:.3e} > {tol['max_abs']}"
    if tol["rel"] is not None:
        d = o_gpu.reshape(-1, o_gpu.shape[-1]) - o_ref.reshape(-1, o_ref.shape[-1])
        rel = np.linalg.norm(d, axis=1) / np.maximum(np.linalg.norm(o_ref.reshape(-1, o_ref.shape[-1]), axis=1), 1e-30)
        assert np.max(rel) <= tol["rel"], f"{what}: relative error {np.max(rel):.3e} > {tol['rel']}"
    return err


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def oracle_gates_rows(wl: W.Workload, layer: int, b: int, T: int, W1, b1, W2, b2, block: int = 2048):
    """Oracle u, z [T][Hkv] of batch row b, positions 0..T-1 (hidden states regenerated on
    the host in blocks)."""
    us = []
    for s0 in range(0, T, block):
        h = wl.h_rows(layer, b, np.arange(s0, min(T, s0 + block)))
        us.append(O.utility(h, W1, b1, W2, b2))
    u = np.concatenate(us, axis=0)
    return u, O.gate(u, wl.tau)


def kv_rows(wl: W.Workload, layer: int, b: int, T: int, block: int = 4096):
    """Host K, V [T][Hkv][d] of batch row b, positions 0..T-1."""
    ks, vs = [], []
    for s0 in range(0, T, block):
        pos = np.arange(s0, min(T, s0 + block))
        ks.append(wl.k_rows(layer, b, pos))
        vs.append(wl.v_rows(layer, b, pos))
    return np.concatenate(ks), np.concatenate(vs)


def check_list(got, z_col, upto, u_col, tau):
    """Cache index list against the oracle's, where tokens within EXCLUDE of tau may go
    either way."""
    want = O.cache_rows(z_col, upto)
    near = set(np.nonzero(np.abs(u_col[:upto] - tau) < EXCLUDE)[0].tolist())
    a = [int(x) for x in got if int(x) not in near]
    c = [int(x) for x in want if int(x) not in near]
    assert a == c, f"cache list differs away from the threshold ({len(a)} vs {len(c)} rows)"
    return len(near)
