"""Thin ctypes binding of ``libspkv.so`` (C ABI in include/spkv.h).

Argument marshalling only: every step of the SP-KV path runs in the CUDA kernels
of the library.  PyTorch tensors provide device memory, their ``data_ptr()`` is
passed through, and the stream is the caller's current torch CUDA stream unless
one is given.  There is no fallback: if the library is missing, importing this
module raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspkv.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with "
                      "`python -m sparse_decode_attention_spkv_b200.build`")
lib = ctypes.CDLL(_LIB_PATH)
DEBUG_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspkv_debug.so")

OK, ERR_ARG, ERR_CAPACITY, ERR_CUDA, ERR_UNSUPPORTED, ERR_TIMEOUT, ERR_INDEX = range(7)
F32, BF16 = 0, 1
SRC_CHUNK, SRC_RING = 0, 1
FLAG_POOL_FULL, FLAG_TABLE_FULL, FLAG_TIMEOUT, FLAG_INDEX = 1, 2, 4, 8
PAGE_ROWS = 64
DECODE_STATE_SETTLED = 1
INPUTS_SETTLED = 1
SLICE_WINDOW = 1

_vp = ctypes.c_void_p
_i32 = ctypes.c_int


class spkv_params(ctypes.Structure):
    _fields_ = [("B", _i32), ("Hq", _i32), ("Hkv", _i32), ("head_dim", _i32), ("d_model", _i32),
                ("hid", _i32), ("window", _i32), ("tau", ctypes.c_float), ("dtype", _i32)]


class spkv_cache(ctypes.Structure):
    _fields_ = [("K_pool", _vp), ("V_pool", _vp), ("pos_pool", _vp), ("page_table", _vp),
                ("count", _vp), ("count_prev", _vp), ("pool_top", _vp), ("err_flag", _vp),
                ("u_pool", _vp), ("num_pages", _i32), ("page_rows", _i32),
                ("max_pages_per_head", _i32)]


class spkv_ring(ctypes.Structure):
    _fields_ = [("K_win", _vp), ("V_win", _vp), ("z_win", _vp), ("u_win", _vp)]


_P = ctypes.POINTER
_sigs = {
    "spkv_status_str": (ctypes.c_char_p, [_i32]),
    "spkv_version": (_i32, []),
    "spkv_cache_reset": (_i32, [_P(spkv_params), _P(spkv_cache), _P(spkv_ring), _vp]),
    "spkv_cache_check": (_i32, [_P(spkv_cache), _vp, _P(ctypes.c_uint32)]),
    "spkv_score": (_i32, [_P(spkv_params), _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "spkv_write_compact": (_i32, [_P(spkv_params), _P(spkv_cache), _P(spkv_ring), _i32, _vp, _vp,
                                  _vp, _vp, _vp, _i32, _i32, _vp]),
    "spkv_decode_append": (_i32, [_P(spkv_params), _P(spkv_cache), _P(spkv_ring), _vp, _vp, _vp,
                                  _vp, _vp, _i32, _vp]),
    "spkv_ring_write": (_i32, [_P(spkv_params), _P(spkv_ring), _vp, _vp, _vp, _vp, _i32, _vp, _i32,
                                _i32, _vp]),
    "spkv_rethreshold_workspace_bytes": (ctypes.c_size_t, [_P(spkv_params), _P(spkv_cache)]),
    "spkv_cache_rethreshold": (_i32, [_P(spkv_params), _P(spkv_cache), _P(spkv_ring),
                                      ctypes.c_float, _vp, ctypes.c_size_t, _vp]),
    "spkv_soft_attn_workspace_bytes": (ctypes.c_size_t, [_P(spkv_params), _i32]),
    "spkv_soft_attn": (_i32, [_P(spkv_params), _vp, _vp, _vp, _vp, _i32, ctypes.c_float,
                              ctypes.c_float, _vp, _vp, _vp, ctypes.c_size_t, _vp, _vp]),
    "spkv_decode_workspace_bytes": (ctypes.c_size_t, [_P(spkv_params), _P(spkv_cache)]),
    "spkv_decode_attn": (_i32, [_P(spkv_params), _P(spkv_cache), _P(spkv_ring), _vp, _vp, _vp, _vp,
                                _vp, ctypes.c_size_t, _vp]),
    "spkv_decode_attn_before_append": (_i32, [_P(spkv_params), _P(spkv_cache), _P(spkv_ring), _vp,
                                              _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                              ctypes.c_uint, _vp]),
    "spkv_decode_attn_before_append_supported": (_i32, [_P(spkv_params)]),
    "spkv_prefill_attn": (_i32, [_P(spkv_params), _P(spkv_cache), _P(spkv_ring), _vp, _vp, _vp, _i32,
                                 _i32, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "spkv_decode_attn_noalloc": (_i32, [_P(spkv_params), _P(spkv_cache), _P(spkv_ring), _vp, _vp,
                                        _vp, _vp, _vp]),
    "spkv_decode_score_append": (_i32, [_P(spkv_params), _P(spkv_cache), _P(spkv_ring), _vp, _vp,
                                        _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_uint,
                                        _vp]),
    "spkv_decode_score": (_i32, [_P(spkv_params), _P(spkv_ring), _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _vp, _vp]),
    "spkv_decode_attn_partial": (_i32, [_P(spkv_params), _P(spkv_cache), _P(spkv_ring), _vp, _vp,
                                        ctypes.c_uint, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "spkv_decode_attn_partial_supported": (_i32, [_P(spkv_params)]),
    "spkv_decode_merge": (_i32, [_P(spkv_params), _i32, _vp, _vp, _vp, _vp, _vp]),
    "spkv_debug_set_flag_wait_ns": (_i32, [ctypes.c_ulonglong]),
}
NOALLOC_SCRATCH_BYTES = 8 << 20
PREFILL_WORKSPACE_BYTES = 256


def _bind(handle):
    for _name, (_res, _args) in _sigs.items():
        _fn = getattr(handle, _name)
        _fn.restype = _res
        _fn.argtypes = _args
    return handle


_bind(lib)


def open_library(path: str):
    """Another build of the same C ABI (e.g. the debug build, libspkv_debug.so, whose
    kernels check page-table entries and positions), with the same signatures.  Assign
    it to ``spkv.lib`` to route the functions below through it."""
    return _bind(ctypes.CDLL(path))


class SpkvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {status_str(status)} ({status})")
        self.status = status


def status_str(status: int) -> str:
    return lib.spkv_status_str(status).decode()


def _check(fn: str, status: int) -> int:
    if status != OK:
        raise SpkvError(fn, status)
    return status


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def torch_dtype(dtype: int) -> torch.dtype:
    return torch.bfloat16 if dtype == BF16 else torch.float32


def make_params(B, Hq, Hkv, head_dim, d_model, hid, window, tau, dtype) -> spkv_params:
    return spkv_params(B, Hq, Hkv, head_dim, d_model, hid, window, float(tau), dtype)


@dataclass
class Cache:
    """Device tensors of one layer's gated cache and the ctypes view of them."""
    K_pool: torch.Tensor
    V_pool: torch.Tensor
    pos_pool: torch.Tensor
    page_table: torch.Tensor
    count: torch.Tensor
    count_prev: torch.Tensor
    pool_top: torch.Tensor
    err_flag: torch.Tensor
    u_pool: Optional[torch.Tensor]
    c: spkv_cache

    @staticmethod
    def allocate(p: spkv_params, num_pages: int, max_pages_per_head: int, device="cuda",
                 store_u: bool = False) -> "Cache":
        """store_u: keep the utility of every stored row (needed by
        spkv_cache_rethreshold)."""
        dt = torch_dtype(p.dtype)
        heads = p.B * p.Hkv
        K = torch.zeros((num_pages, PAGE_ROWS, p.head_dim), dtype=dt, device=device)
        V = torch.zeros_like(K)
        pos = torch.zeros((num_pages, PAGE_ROWS), dtype=torch.int32, device=device)
        table = torch.full((heads, max_pages_per_head), -1, dtype=torch.int32, device=device)
        count = torch.zeros(heads, dtype=torch.int32, device=device)
        count_prev = torch.zeros(heads, dtype=torch.int32, device=device)
        top = torch.zeros(1, dtype=torch.int32, device=device)
        err = torch.zeros(1, dtype=torch.int32, device=device)
        u = torch.zeros((num_pages, PAGE_ROWS), dtype=torch.float32, device=device) if store_u else None
        c = spkv_cache(K.data_ptr(), V.data_ptr(), pos.data_ptr(), table.data_ptr(),
                       count.data_ptr(), count_prev.data_ptr(), top.data_ptr(), err.data_ptr(),
                       u.data_ptr() if u is not None else None, num_pages, PAGE_ROWS,
                       max_pages_per_head)
        return Cache(K, V, pos, table, count, count_prev, top, err, u, c)


@dataclass
class Ring:
    K_win: torch.Tensor
    V_win: torch.Tensor
    z_win: torch.Tensor
    u_win: Optional[torch.Tensor]
    r: spkv_ring

    @staticmethod
    def allocate(p: spkv_params, device="cuda", store_u: bool = False) -> "Ring":
        """store_u: keep the pending utility of every slot (NaN: none pending)."""
        dt = torch_dtype(p.dtype)
        K = torch.zeros((p.B, p.Hkv, p.window, p.head_dim), dtype=dt, device=device)
        V = torch.zeros_like(K)
        z = torch.zeros((p.B, p.window, p.Hkv), dtype=torch.uint8, device=device)
        u = torch.full((p.B, p.window, p.Hkv), float("nan"), dtype=torch.float32,
                       device=device) if store_u else None
        return Ring(K, V, z, u, spkv_ring(K.data_ptr(), V.data_ptr(), z.data_ptr(),
                                          u.data_ptr() if u is not None else None))


# ---- entry points (same names as the C ABI) -------------------------------------------

def spkv_cache_reset(p, cache: Cache, ring: Optional[Ring] = None, stream=None):
    return _check("spkv_cache_reset", lib.spkv_cache_reset(
        ctypes.byref(p), ctypes.byref(cache.c), ctypes.byref(ring.r) if ring else None,
        _stream(stream)))


def spkv_cache_check(cache: Cache, stream=None):
    flags = ctypes.c_uint32(0)
    status = lib.spkv_cache_check(ctypes.byref(cache.c), _stream(stream), ctypes.byref(flags))
    return status, int(flags.value)


def spkv_score(p, h, n_tok, W1, b1, W2, b2, u_out, z_out, stream=None):
    return _check("spkv_score", lib.spkv_score(
        ctypes.byref(p), _ptr(h), n_tok, _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(u_out),
        _ptr(z_out), _stream(stream)))


def spkv_write_compact(p, cache: Cache, ring: Optional[Ring], src_kind, K_src, V_src, z, u,
                       src_pos, n_rows, src_batch_rows, stream=None):
    return _check("spkv_write_compact", lib.spkv_write_compact(
        ctypes.byref(p), ctypes.byref(cache.c), ctypes.byref(ring.r) if ring else None, src_kind,
        _ptr(K_src), _ptr(V_src), _ptr(z), _ptr(u), _ptr(src_pos), n_rows, src_batch_rows,
        _stream(stream)))


def _cache_ref(cache: Optional[Cache]):
    return ctypes.byref(cache.c) if cache is not None else None


def spkv_decode_append(p, cache: Optional[Cache], ring: Ring, t_pos, k_new, v_new, z_new, u_new,
                       retire, stream=None):
    """cache None: a window-only layer (retire must be 0)."""
    return _check("spkv_decode_append", lib.spkv_decode_append(
        ctypes.byref(p), _cache_ref(cache), ctypes.byref(ring.r), _ptr(t_pos), _ptr(k_new),
        _ptr(v_new), _ptr(z_new), _ptr(u_new), int(retire), _stream(stream)))


def spkv_ring_write(p, ring: Ring, K_src, V_src, z_src, u_src, gated_from, src_pos, n_rows,
                    src_batch_rows, stream=None):
    return _check("spkv_ring_write", lib.spkv_ring_write(
        ctypes.byref(p), ctypes.byref(ring.r), _ptr(K_src), _ptr(V_src), _ptr(z_src), _ptr(u_src),
        int(gated_from), _ptr(src_pos), n_rows, src_batch_rows, _stream(stream)))


def spkv_rethreshold_workspace_bytes(p, cache: Cache) -> int:
    return int(lib.spkv_rethreshold_workspace_bytes(ctypes.byref(p), ctypes.byref(cache.c)))


def alloc_rethreshold_workspace(p, cache: Cache, device="cuda") -> torch.Tensor:
    n = spkv_rethreshold_workspace_bytes(p, cache)
    if n == 0:
        raise SpkvError("spkv_rethreshold_workspace_bytes", ERR_ARG)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def spkv_cache_rethreshold(p, cache: Cache, ring: Optional[Ring], tau_new, workspace,
                           stream=None):
    return _check("spkv_cache_rethreshold", lib.spkv_cache_rethreshold(
        ctypes.byref(p), ctypes.byref(cache.c), ctypes.byref(ring.r) if ring else None,
        float(tau_new), _ptr(workspace), workspace.numel(), _stream(stream)))


def spkv_decode_workspace_bytes(p, cache: Optional[Cache]) -> int:
    return int(lib.spkv_decode_workspace_bytes(ctypes.byref(p), _cache_ref(cache)))


def alloc_decode_workspace(p, cache: Cache, device="cuda") -> torch.Tensor:
    n = spkv_decode_workspace_bytes(p, cache)
    if n == 0:
        raise SpkvError("spkv_decode_workspace_bytes", ERR_ARG)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def spkv_decode_attn(p, cache: Optional[Cache], ring: Ring, q, t_pos, o, lse, workspace,
                     stream=None):
    """cache None: a window-only layer (attends to the ring only)."""
    return _check("spkv_decode_attn", lib.spkv_decode_attn(
        ctypes.byref(p), _cache_ref(cache), ctypes.byref(ring.r), _ptr(q), _ptr(t_pos), _ptr(o),
        _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))


def spkv_decode_attn_before_append(p, cache: Optional[Cache], ring: Ring, q, t_pos, k_new, v_new,
                                   o, lse, workspace, flags=0, stream=None):
    """The decode attention of a step taken before the step's spkv_decode_append (the
    new rows k_new / v_new passed in); flags: 0 or DECODE_STATE_SETTLED.  See
    include/spkv.h."""
    return _check("spkv_decode_attn_before_append", lib.spkv_decode_attn_before_append(
        ctypes.byref(p), _cache_ref(cache), ctypes.byref(ring.r), _ptr(q), _ptr(t_pos),
        _ptr(k_new), _ptr(v_new), _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel(),
        int(flags), _stream(stream)))


def spkv_decode_attn_before_append_supported(p) -> bool:
    return bool(lib.spkv_decode_attn_before_append_supported(ctypes.byref(p)))


def alloc_prefill_workspace(device="cuda") -> torch.Tensor:
    """The optional tile-counter workspace of spkv_prefill_attn (zero-filled)."""
    return torch.zeros(PREFILL_WORKSPACE_BYTES, dtype=torch.uint8, device=device)


def spkv_prefill_attn(p, cache: Optional[Cache], ring: Ring, q, K_chunk, V_chunk, chunk_start,
                      chunk_len, o, lse, workspace=None, stream=None):
    """cache None: a window-only layer.  workspace: None (fixed tile order) or a tensor
    from alloc_prefill_workspace (tiles handed out to free CTAs)."""
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return _check("spkv_prefill_attn", lib.spkv_prefill_attn(
        ctypes.byref(p), _cache_ref(cache), ctypes.byref(ring.r), _ptr(q), _ptr(K_chunk),
        _ptr(V_chunk), chunk_start, chunk_len, _ptr(o), _ptr(lse), _ptr(workspace), ws_bytes,
        _stream(stream)))


def spkv_decode_attn_noalloc(p, cache: Optional[Cache], ring: Ring, q, t_pos, o, lse,
                             stream=None):
    """spkv_decode_attn for callers that cannot allocate a workspace: the scratch is a
    fixed array inside the library (see include/spkv.h).  cache None: a window-only
    layer."""
    return _check("spkv_decode_attn_noalloc", lib.spkv_decode_attn_noalloc(
        ctypes.byref(p), _cache_ref(cache), ctypes.byref(ring.r), _ptr(q), _ptr(t_pos), _ptr(o),
        _ptr(lse), _stream(stream)))


def spkv_decode_score_append(p, cache: Cache, ring: Ring, t_pos, h, W1, b1, W2, b2, k_new, v_new,
                             u_out, z_out, flags=0, stream=None):
    """flags: 0 or INPUTS_SETTLED (h written before the preceding kernel started; see
    include/spkv.h)."""
    return _check("spkv_decode_score_append", lib.spkv_decode_score_append(
        ctypes.byref(p), ctypes.byref(cache.c), ctypes.byref(ring.r), _ptr(t_pos), _ptr(h), _ptr(W1),
        _ptr(b1), _ptr(W2), _ptr(b2), _ptr(k_new), _ptr(v_new), _ptr(u_out), _ptr(z_out),
        int(flags), _stream(stream)))


def spkv_soft_attn_workspace_bytes(p, seq_len: int) -> int:
    return int(lib.spkv_soft_attn_workspace_bytes(ctypes.byref(p), int(seq_len)))


def spkv_soft_attn(p, q, K, V, u, seq_len, beta, c, o, lse, workspace, err_flag=None,
                   stream=None):
    """Soft-gated training-time attention (Eqs. (5)-(6)); see include/spkv.h."""
    return _check("spkv_soft_attn", lib.spkv_soft_attn(
        ctypes.byref(p), _ptr(q), _ptr(K), _ptr(V), _ptr(u), int(seq_len), float(beta), float(c),
        _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel(), _ptr(err_flag), _stream(stream)))


def spkv_decode_score(p, ring: Ring, t_pos, h, W1, b1, W2, b2, u_out, z_out, stream=None):
    """Score one decode step's new tokens and store their gates in their window slots
    (to run beside the attention; see include/spkv.h)."""
    return _check("spkv_decode_score", lib.spkv_decode_score(
        ctypes.byref(p), ctypes.byref(ring.r), _ptr(t_pos), _ptr(h), _ptr(W1), _ptr(b1), _ptr(W2),
        _ptr(b2), _ptr(u_out), _ptr(z_out), _stream(stream)))


def _ring_ref(ring: Optional[Ring]):
    return ctypes.byref(ring.r) if ring is not None else None


def spkv_decode_attn_partial(p, cache: Optional[Cache], ring: Optional[Ring], q, t_pos, flags,
                             o_part, lse_part, workspace, stream=None):
    """Decode attention over one slice of a split sequence (its cache rows, and the window
    with flags SLICE_WINDOW): fp32 o_part [B][Hq][d] and lse_part [B][Hq].  See
    include/spkv.h."""
    return _check("spkv_decode_attn_partial", lib.spkv_decode_attn_partial(
        ctypes.byref(p), _cache_ref(cache), _ring_ref(ring), _ptr(q), _ptr(t_pos), int(flags),
        _ptr(o_part), _ptr(lse_part), _ptr(workspace), workspace.numel(), _stream(stream)))


def spkv_decode_attn_partial_supported(p) -> bool:
    return bool(lib.spkv_decode_attn_partial_supported(ctypes.byref(p)))


def spkv_decode_merge(p, n_parts, o_parts, lse_parts, o, lse, stream=None):
    """Log-sum-exp combination of slice partials o_parts [n][B][Hq][d], lse_parts [n][B][Hq]
    (fp32) into o [B][Hq][d] and lse [B][Hq] (may be None)."""
    return _check("spkv_decode_merge", lib.spkv_decode_merge(
        ctypes.byref(p), int(n_parts), _ptr(o_parts), _ptr(lse_parts), _ptr(o), _ptr(lse),
        _stream(stream)))


def spkv_debug_set_flag_wait_ns(ns: int):
    """Limit of the re-threshold move kernel's page-flag waits (0: the default); for
    testing failure reporting (see include/spkv.h)."""
    return _check("spkv_debug_set_flag_wait_ns", lib.spkv_debug_set_flag_wait_ns(int(ns)))
