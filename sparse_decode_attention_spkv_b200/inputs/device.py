"""Device side of the seeded input generator: fills torch CUDA tensors in place
with the same values ``gen.py`` defines (see its docstring)."""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspkv_inputs.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: run `python -m sparse_decode_attention_spkv_b200.build`")
_lib = ctypes.CDLL(_LIB_PATH)
_lib.spkv_gen_normal.restype = ctypes.c_int
_lib.spkv_gen_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_double,
                                 ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
_lib.spkv_gen_rope.restype = ctypes.c_int
_lib.spkv_gen_rope.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int,
                               ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                               ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return 1
    if t.dtype == torch.float32:
        return 0
    raise TypeError(t.dtype)


def _s():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def fill_normal(out: torch.Tensor, key: int, scale: float, offset: int = 0) -> torch.Tensor:
    """out.view(-1)[j] = draw (offset + j) * scale, rounded to out's dtype."""
    assert out.is_cuda and out.is_contiguous()
    rc = _lib.spkv_gen_normal(key, offset, out.numel(), scale, _dt(out), out.data_ptr(), _s())
    if rc != 0:
        raise RuntimeError("spkv_gen_normal failed")
    return out


def fill_rope(out: torch.Tensor, key: int, row0: int, tokens_per_batch: int, scale: float,
              base: float) -> torch.Tensor:
    """Rows row0.. of a [tokens][n_heads][head_dim] tensor with rotary embedding; token
    row r has position r % tokens_per_batch (out has shape [n_rows, n_heads, head_dim]
    or any shape with that flat layout)."""
    n_heads, head_dim = out.shape[-2], out.shape[-1]
    n_rows = out.numel() // (n_heads * head_dim)
    rc = _lib.spkv_gen_rope(key, row0, n_rows, n_heads, head_dim, tokens_per_batch, scale, base,
                            _dt(out), out.data_ptr(), _s())
    if rc != 0:
        raise RuntimeError("spkv_gen_rope failed")
    return out
