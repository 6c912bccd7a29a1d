"""Decode attention through the no-allocation entry point (GPU required).

Some callers cannot allocate the decode workspace themselves (a host that owns all
device memory through its own pool, a path that may not call cudaMalloc after
start-up).  spkv_decode_attn_noalloc serves them from a fixed scratch array inside
the library.  Here it must match the oracle and give what spkv_decode_attn gives, on
two calls in a row (the shared scratch keeps the previous call's contents), within
the tolerance the parity tests use; calls of different shapes in turn share the one
array.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import spkv_oracle as O
from sparse_decode_attention_spkv_b200.inputs import workloads as W
from tests import cases as C

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from sparse_decode_attention_spkv_b200 import runner as R
    from sparse_decode_attention_spkv_b200 import spkv as S


def _state(wl, T0, local=False):
    """A layer whose cache and ring hold T0 tokens (per-token-ready), built through the
    library, the inputs of the decode step at position T0, and the oracle's output of
    that step (window-only attention for a local layer)."""
    W1, b1, W2, b2 = C.weights(wl)
    p = S.make_params(wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau,
                      S.BF16 if wl.dtype == "bf16" else S.F32)
    if local:
        layer = R.Layer.create_local(p)
    else:
        mp = R.pages_for(T0 + 8)
        layer = R.Layer.create(p, C.dev(W1, wl.dtype), C.dev_f32(b1), C.dev_f32(W2),
                               C.dev_f32(b2), num_pages=wl.B * wl.Hkv * mp, max_pages_per_head=mp)
    rows = [C.host_rows(wl, 0, b, np.arange(T0 + 1)) for b in range(wl.B)]
    h, q, k, v = (np.stack([r[i] for r in rows]) for i in range(4))
    w = wl.window
    R.prefill_chunk(layer, C.dev(h[:, :T0], wl.dtype), C.dev(q[:, :T0], wl.dtype),
                    C.dev(k[:, :T0], wl.dtype), C.dev(v[:, :T0], wl.dtype), 0,
                    n_compact=max(0, T0 - w))
    t_pos = torch.full((wl.B,), T0, dtype=torch.int32, device="cuda")
    if local:
        S.spkv_decode_append(p, None, layer.ring, t_pos, C.dev(k[:, T0], wl.dtype),
                             C.dev(v[:, T0], wl.dtype), None, None, 0)
    else:
        u_t, z_t = R.score(layer, C.dev(h[:, T0], wl.dtype), wl.B)
        S.spkv_decode_append(p, layer.cache, layer.ring, t_pos, C.dev(k[:, T0], wl.dtype),
                             C.dev(v[:, T0], wl.dtype), z_t, u_t, 1)
    o_ref = np.zeros((wl.B, wl.Hq, wl.head_dim))
    for b in range(wl.B):
        if local:
            z = np.zeros((T0 + 1, wl.Hkv), dtype=np.uint8)
        else:
            _, z = C.oracle_gates(h[b], W1, b1, W2, b2, wl.tau)
        o_ref[b] = O.gated_attention(q[b, T0:T0 + 1], k[b], v[b], z, w, [T0])[0][0]
    return p, layer, C.dev(q[:, T0], wl.dtype), t_pos, o_ref


def _noalloc_twice(wl, p, layer, q, t_pos, o_ref, what):
    """Two no-allocation calls in a row, each checked against the oracle and against
    spkv_decode_attn on the same state."""
    cache = None if layer.local else layer.cache
    o_ws = torch.empty_like(q)
    lse_ws = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
    S.spkv_decode_attn(p, cache, layer.ring, q, t_pos, o_ws, lse_ws, layer.ws)
    for call in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((wl.B, wl.Hq), float("nan"), dtype=torch.float32, device="cuda")
        S.spkv_decode_attn_noalloc(p, cache, layer.ring, q, t_pos, o, lse)
        torch.cuda.synchronize()
        C.check_attn(C.to_np(o), o_ref, wl.dtype, f"{what} call {call} vs oracle")
        C.check_attn(C.to_np(o), C.to_np(o_ws), wl.dtype, f"{what} call {call} vs workspace call")
        assert np.allclose(lse.cpu().numpy(), lse_ws.cpu().numpy(), atol=1e-4), f"lse, call {call}"
    if cache is not None:
        status, flags = S.spkv_cache_check(cache)
        assert status == S.OK, flags


CASES = {
    "bf16_g4_d128": W.small_case("decode32k", cid=60, B=2, Hq=8, Hkv=2, d_model=128, hid=32,
                                 ctx=[3000], decode_steps=1, layers=1, keep="u05_50"),
    "f32_g2_d64": W.small_case("tiny", cid=61, ctx=[700], decode_steps=1),
    # 64 key heads (batch 8 x 8 key heads, the decode32k geometry): the control region
    # of the tensor-core kernel is larger than the CUDA-core kernel's
    "bf16_64_key_heads": W.small_case("decode32k", cid=62, B=8, d_model=128, hid=32,
                                      ctx=[1200], decode_steps=1, layers=1, keep="u05_50"),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_oracle_and_workspace_entry_point(name):
    wl = CASES[name]
    p, layer, q, t_pos, o_ref = _state(wl, wl.ctx[0])
    _noalloc_twice(wl, p, layer, q, t_pos, o_ref, name)


def test_noalloc_window_only_layer():
    """cache NULL (a local layer of a hybrid stack): the window alone."""
    wl = W.small_case("decode32k", cid=63, B=2, Hq=8, Hkv=2, d_model=128, hid=32, ctx=[600],
                      decode_steps=1, layers=1, keep="fixed25")
    p, layer, q, t_pos, o_ref = _state(wl, wl.ctx[0], local=True)
    _noalloc_twice(wl, p, layer, q, t_pos, o_ref, "window only")


def test_noalloc_shapes_in_turn():
    """Calls of different shapes share the array: a call of 64 key heads, then one of 4,
    then 64 again; each must match the oracle (each call clears its own counters)."""
    big = CASES["bf16_64_key_heads"]
    small = CASES["bf16_g4_d128"]
    sb = _state(big, big.ctx[0])
    ss = _state(small, small.ctx[0])
    for wl, (p, layer, q, t_pos, o_ref), what in ((big, sb, "64 heads"), (small, ss, "4 heads"),
                                                   (big, sb, "64 heads again")):
        o = torch.full_like(q, float("nan"))
        lse = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
        S.spkv_decode_attn_noalloc(p, layer.cache, layer.ring, q, t_pos, o, lse)
        torch.cuda.synchronize()
        C.check_attn(C.to_np(o), o_ref, wl.dtype, what)


def test_noalloc_rejects_shapes_beyond_the_scratch():
    """2048 key heads with 8 query heads each need more split scratch than the fixed
    array holds: the call is refused before anything is enqueued."""
    p = S.make_params(256, 64, 8, 128, 4096, 128, 128, 0.5, S.BF16)
    need = S.lib.spkv_decode_workspace_bytes(ctypes.byref(p), None)
    assert need > S.NOALLOC_SCRATCH_BYTES
    buf = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    a = buf.data_ptr()
    cache = S.spkv_cache(K_pool=a, V_pool=a, pos_pool=a, page_table=a, count=a, count_prev=a,
                         pool_top=a, err_flag=a, u_pool=None, num_pages=1,
                         page_rows=S.PAGE_ROWS, max_pages_per_head=1)
    ring = S.spkv_ring(K_win=a, V_win=a, z_win=a, u_win=None)
    st = S.lib.spkv_decode_attn_noalloc(ctypes.byref(p), ctypes.byref(cache), ctypes.byref(ring),
                                        a, a, a, None, None)
    assert st == S.ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert int(buf.sum()) == 0
