"""The synthetic workloads: shapes, sizes, dtypes and input recipes.

Five workloads follow the long-context decode and prefill regimes of
"Self-Pruned Key-Value Attention" (arXiv 2605.14037): 32k-token training context
(§3.1), batched decode (§3.4, Fig. 3 right), gate threshold tau = 0.5 (§3.1) and
window w = 128 (§2.1).  Everything here is a recipe (which stream, which scale,
which shape); no SP-KV arithmetic happens in this module.

Tensor index conventions (row-major, flat element j of a tensor is generator
draw j of that tensor's stream):
  h  [B][T_total][d_model]          hidden states of every position
  q  [B][T_total][Hq][head_dim]     queries of every position
  k  [B][T_total][Hkv][head_dim]    keys of every position
  v  [B][T_total][Hkv][head_dim]
  W1 [hid][d_model], b1 [hid], W2 [Hkv][hid]   per layer
The output bias b2 [Hkv] per layer is calibrated for the target keep rates and
stored in ``biases.json`` (written by the oracle's calibration script).
"""
from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

from . import gen

SEED = 0
_BIAS_FILE = os.path.join(os.path.dirname(__file__), "biases.json")


@dataclass
class Workload:
    name: str
    cid: int                 # stream id of the workload
    B: int
    Hq: int
    Hkv: int
    head_dim: int
    d_model: int
    hid: int
    window: int
    tau: float
    dtype: str               # "f32" or "bf16"
    layers: int
    ctx: List[int]           # tokens already processed per batch row when decode starts
    decode_steps: int
    chunk: int = 0           # prefill chunk length (0: no chunked prefill in this workload)
    bulk: int = 0            # decode hidden-state buffer (0: per-token retirement)
    rope_base: float = 0.0   # 0: no rotary embedding
    keep: str = ""           # description of the keep-rate recipe
    seed: int = SEED
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def T_total(self) -> int:
        return max(self.ctx) + self.decode_steps

    def key(self, layer: int, kind: int) -> int:
        return gen.stream_key(self.seed, self.cid, layer, kind)

    @property
    def qkv_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    # ---- per-head target keep rates (drawn, not computed) -------------------
    def keep_targets(self, layer: int) -> np.ndarray:
        key = self.key(layer, gen.T_KEEP)
        idx = np.arange(self.Hkv, dtype=np.uint64)
        if self.keep == "fixed25":
            return np.full(self.Hkv, 0.25)
        if self.keep == "fixed20":
            return np.full(self.Hkv, 0.20)
        if self.keep == "u05_50":
            return gen.uniform_f64(key, idx, 0.05, 0.50)
        if self.keep == "spread":
            r = gen.uniform_f64(key, idx, 0.05, 0.15)
            r[0:2] = 0.60
            r[2:4] = 0.02
            return r
        if self.keep == "u05_25":
            return gen.uniform_f64(key, idx, 0.05, 0.25)
        raise ValueError(self.keep)

    # ---- host copies of the small tensors -----------------------------------
    def w1(self, layer: int) -> np.ndarray:
        return gen.normal(self.key(layer, gen.T_W1), (self.hid, self.d_model), 0.02, self.dtype)

    def b1(self, layer: int) -> np.ndarray:
        return gen.normal(self.key(layer, gen.T_B1), (self.hid,), 0.02, "f32")

    def w2(self, layer: int) -> np.ndarray:
        return gen.normal(self.key(layer, gen.T_W2), (self.Hkv, self.hid), 0.02, "f32")

    def b2(self, layer: int) -> np.ndarray:
        table = load_biases()
        if self.name not in table:
            raise KeyError(f"no calibrated output bias for workload {self.name}; "
                           f"run oracle/calibrate.py")
        return np.asarray(table[self.name]["b2"][layer], dtype=np.float32)

    # ---- rows of the big tensors (host side) ---------------------------------
    def h_rows(self, layer: int, b: int, positions) -> np.ndarray:
        rows = b * self.T_total + np.asarray(positions, dtype=np.int64)
        return gen.normal_rows(self.key(layer, gen.T_H), self.d_model, rows, 1.0, self.dtype)

    def _qk_rows(self, kind: int, nh: int, layer: int, b: int, positions) -> np.ndarray:
        pos = np.asarray(positions, dtype=np.int64)
        rows = b * self.T_total + pos
        if self.rope_base:
            return gen.rope_rows(self.key(layer, kind), self.head_dim, nh, rows, pos,
                                 self.qkv_scale, self.rope_base, self.dtype)
        x = gen.normal_rows(self.key(layer, kind), nh * self.head_dim, rows, self.qkv_scale,
                            self.dtype)
        return x.reshape(len(pos), nh, self.head_dim)

    def q_rows(self, layer: int, b: int, positions) -> np.ndarray:
        return self._qk_rows(gen.T_Q, self.Hq, layer, b, positions)

    def k_rows(self, layer: int, b: int, positions) -> np.ndarray:
        return self._qk_rows(gen.T_K, self.Hkv, layer, b, positions)

    def v_rows(self, layer: int, b: int, positions) -> np.ndarray:
        pos = np.asarray(positions, dtype=np.int64)
        rows = b * self.T_total + pos
        x = gen.normal_rows(self.key(layer, gen.T_V), self.Hkv * self.head_dim, rows,
                            self.qkv_scale, self.dtype)
        return x.reshape(len(pos), self.Hkv, self.head_dim)

    def calib_h(self, layer: int, n: int) -> np.ndarray:
        return gen.normal(self.key(layer, gen.T_CAL), (n, self.d_model), 1.0, self.dtype)


def _ctx_c4() -> List[int]:
    key = gen.stream_key(SEED, 4, 0, gen.T_CTX)
    u = gen.uniform_f64(key, np.arange(32, dtype=np.uint64), 8192.0, 65536.0)
    return [int(x) for x in np.floor(u)]


WORKLOADS = {
    "tiny": Workload("tiny", 0, B=1, Hq=4, Hkv=2, head_dim=64, d_model=256, hid=64, window=128,
                     tau=0.5, dtype="f32", layers=1, ctx=[512], decode_steps=16, chunk=512,
                     keep="fixed25"),
    "decode32k": Workload("decode32k", 1, B=8, Hq=32, Hkv=8, head_dim=128, d_model=4096, hid=128,
                          window=128, tau=0.5, dtype="bf16", layers=32, ctx=[32768] * 8,
                          decode_steps=256, keep="u05_50"),
    "prefill16k": Workload("prefill16k", 2, B=1, Hq=32, Hkv=8, head_dim=128, d_model=4096,
                           hid=128, window=128, tau=0.5, dtype="bf16", layers=1, ctx=[16384],
                           decode_steps=0, chunk=4096, rope_base=1e4, keep="fixed20"),
    "ragged128k": Workload("ragged128k", 3, B=4, Hq=32, Hkv=8, head_dim=128, d_model=4096,
                           hid=128, window=128, tau=0.5, dtype="bf16", layers=1,
                           ctx=[131072, 98304, 65536, 32768], decode_steps=64, keep="spread"),
    "serving": Workload("serving", 4, B=32, Hq=32, Hkv=8, head_dim=128, d_model=4096, hid=128,
                        window=128, tau=0.5, dtype="bf16", layers=1, ctx=_ctx_c4(),
                        decode_steps=256, bulk=128, keep="u05_25"),
}

_BIASES: Optional[dict] = None


def load_biases() -> dict:
    global _BIASES
    if _BIASES is None:
        if os.path.exists(_BIAS_FILE):
            with open(_BIAS_FILE) as f:
                _BIASES = json.load(f)
        else:
            _BIASES = {}
    return _BIASES


def bias_file() -> str:
    return _BIAS_FILE


def small_case(name: str, **overrides) -> Workload:
    """A workload with some fields replaced (for parity cases at oracle-friendly sizes).
    Stream ids stay those of ``name`` unless ``cid`` is overridden."""
    base = WORKLOADS[name]
    d = dict(base.__dict__)
    d.update(overrides)
    return Workload(**d)
