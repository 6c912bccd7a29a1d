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
