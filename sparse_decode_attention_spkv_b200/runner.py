"""Schedules of the SP-KV hot path, driven through the C ABI.

A ``Layer`` holds one attention layer's utility-perceptron weights, gated cache,
window ring and decode workspace on the device.  A local layer of a hybrid
local/global stack (``Layer.create_local``) has only the ring: it keeps no
long-range cache and attends to its window alone.  The functions below sequence the
library calls for the three schedules the workloads use:

* chunked prefill, compacting each chunk right after scoring it (the chunk's
  gated rows are in the cache before its attention runs; queries only use cache
  rows that have left their window);
* per-token decode: score the new token, retire the token leaving the window into
  the cache if gated in, store the new token in the ring, attend;
* buffered decode: tokens go to the ring ungated; every ``bulk`` steps the
  buffered hidden states are scored together and their gated rows compacted from
  the ring, before the oldest of them leaves the window.

Every step runs in the library's kernels; this module only allocates buffers and
orders calls.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from . import spkv as S


@dataclass
class Layer:
    p: S.spkv_params
    W1: Optional[torch.Tensor]
    b1: Optional[torch.Tensor]
    W2: Optional[torch.Tensor]
    b2: Optional[torch.Tensor]
    cache: Optional[S.Cache]
    ring: S.Ring
    ws: torch.Tensor
    pf_ws: Optional[torch.Tensor] = None  # tile counter of the prefill attention

    @property
    def local(self) -> bool:
        return self.cache is None

    @staticmethod
    def create_local(p: S.spkv_params, device="cuda") -> "Layer":
        """A window-only layer (the local layers of a hybrid stack, §3.3 "Hybrids"):
        no utility perceptron, no cache."""
        ring = S.Ring.allocate(p, device)
        ws = S.alloc_decode_workspace(p, None, device)
        return Layer(p, None, None, None, None, None, ring, ws, S.alloc_prefill_workspace(device))

    @staticmethod
    def create(p: S.spkv_params, W1, b1, W2, b2, num_pages: int, max_pages_per_head: int,
               device="cuda", store_u: bool = False) -> "Layer":
        """store_u: keep the utility of every cached row and pending window slot, so
        that the cache can be re-thresholded later (spkv_cache_rethreshold)."""
        cache = S.Cache.allocate(p, num_pages, max_pages_per_head, device, store_u=store_u)
        ring = S.Ring.allocate(p, device, store_u=store_u)
        ws = S.alloc_decode_workspace(p, cache, device)
        layer = Layer(p, W1, b1, W2, b2, cache, ring, ws, S.alloc_prefill_workspace(device))
        S.spkv_cache_reset(p, cache, ring)
        return layer

    @property
    def dtype(self) -> torch.dtype:
        return S.torch_dtype(self.p.dtype)


def pages_for(rows_per_head, window: int = 0, slack: int = 2) -> int:
    """Pages a head needs to hold ``rows_per_head`` rows (plus slack)."""
    return (int(rows_per_head) + S.PAGE_ROWS - 1) // S.PAGE_ROWS + slack


def score(layer: Layer, h: torch.Tensor, n_tok: int, u: Optional[torch.Tensor] = None):
    """a1: u, z for n_tok tokens of h [n_tok][d_model]."""
    dev = h.device
    z = torch.empty((n_tok, layer.p.Hkv), dtype=torch.uint8, device=dev)
    if u is None:
        u = torch.empty((n_tok, layer.p.Hkv), dtype=torch.float32, device=dev)
    S.spkv_score(layer.p, h, n_tok, layer.W1, layer.b1, layer.W2, layer.b2, u, z)
    return u, z


def prefill_chunk(layer: Layer, h, q, k, v, chunk_start: int, n_compact: Optional[int] = None,
                  src_pos: Optional[torch.Tensor] = None):
    """One chunk of chunked prefill for all batch rows.

    h [B][Tc][d_model], q [B][Tc][Hq][d], k, v [B][Tc][Hkv][d] (contiguous).  The
    first ``n_compact`` rows (default: all) are compacted after scoring; the rest
    stay only in the ring with their gates, to be retired by per-token decode.
    Returns (o [B][Tc][Hq][d], lse [B][Tc][Hq], u, z [B][Tc][Hkv])."""
    p = layer.p
    B, Tc = q.shape[0], q.shape[1]
    dev = q.device
    if n_compact is None:
        n_compact = Tc
    if src_pos is None:
        src_pos = torch.full((B,), chunk_start, dtype=torch.int32, device=dev)
    if layer.local:  # window only: attend, then keep the chunk's last rows in the ring
        o = torch.empty_like(q)
        lse = torch.empty((B, Tc, p.Hq), dtype=torch.float32, device=dev)
        S.spkv_prefill_attn(p, None, layer.ring, q, k, v, chunk_start, Tc, o, lse, layer.pf_ws)
        S.spkv_ring_write(p, layer.ring, k, v, None, None, Tc, src_pos, Tc, Tc)
        return o, lse, None, None
    u, z = score(layer, h, B * Tc)
    if n_compact > 0:
        S.spkv_write_compact(p, layer.cache, layer.ring, S.SRC_CHUNK, k, v, z, u, src_pos, n_compact,
                             Tc)
    o = torch.empty_like(q)
    lse = torch.empty((B, Tc, p.Hq), dtype=torch.float32, device=dev)
    S.spkv_prefill_attn(p, layer.cache, layer.ring, q, k, v, chunk_start, Tc, o, lse, layer.pf_ws)
    S.spkv_ring_write(p, layer.ring, k, v, z, u, n_compact, src_pos, Tc, Tc)
    return o, lse, u.view(B, Tc, p.Hkv), z.view(B, Tc, p.Hkv)


def decode_step(layer: Layer, t_pos: torch.Tensor, h_t, q_t, k_t, v_t, retire: bool = True,
                o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                fused: bool = True, score_stream=None, attn_first: bool = False,
                score_flags: int = 0):
    """One decode step for every batch row at positions t_pos [B] (device int32).

    h_t [B][d_model] (ignored when retire is False: buffered scoring), q_t [B][Hq][d],
    k_t, v_t [B][Hkv][d].  With ``fused`` the score and the ring/cache update are one
    launch (spkv_decode_score_append), else spkv_score then spkv_decode_append.  With a
    ``score_stream`` the update comes first (new gate 0), then the attention, and the new
    tokens are scored on that stream with their gates stored in the window
    (spkv_decode_score); the caller joins that stream before the gates are needed.  With
    a ``score_stream`` and ``attn_first`` the attention runs first, on the state before
    the step's update (spkv_decode_attn_before_append, the new rows passed in), and the
    update and the scoring both go to that stream.  ``score_flags`` go to the fused
    launch (0 or spkv.INPUTS_SETTLED).
    Returns (o [B][Hq][d], lse [B][Hq], z_t or None)."""
    p = layer.p
    z_t = u_t = None
    if layer.local:  # store the new token in the ring; nothing ever retires
        if o is None:
            o = torch.empty_like(q_t)
        if lse is None:
            lse = torch.empty((p.B, p.Hq), dtype=torch.float32, device=q_t.device)
        if score_stream is not None and attn_first:
            S.spkv_decode_attn_before_append(p, None, layer.ring, q_t, t_pos, k_t, v_t, o, lse,
                                             layer.ws)
            score_stream.wait_stream(torch.cuda.current_stream())
            S.spkv_decode_append(p, None, layer.ring, t_pos, k_t, v_t, None, None, 0,
                                 stream=score_stream)
            for x in (k_t, v_t, t_pos):
                x.record_stream(score_stream)
            return o, lse, None
        S.spkv_decode_append(p, None, layer.ring, t_pos, k_t, v_t, None, None, 0)
        S.spkv_decode_attn(p, None, layer.ring, q_t, t_pos, o, lse, layer.ws)
        return o, lse, None
    if retire and score_stream is not None and attn_first:
        z_t = torch.empty((p.B, p.Hkv), dtype=torch.uint8, device=q_t.device)
        u_t = torch.empty((p.B, p.Hkv), dtype=torch.float32, device=q_t.device)
        if o is None:
            o = torch.empty_like(q_t)
        if lse is None:
            lse = torch.empty((p.B, p.Hq), dtype=torch.float32, device=q_t.device)
        S.spkv_decode_attn_before_append(p, layer.cache, layer.ring, q_t, t_pos, k_t, v_t, o, lse,
                                         layer.ws)
        score_stream.wait_stream(torch.cuda.current_stream())
        S.spkv_decode_append(p, layer.cache, layer.ring, t_pos, k_t, v_t, None, None, 1,
                             stream=score_stream)
        S.spkv_decode_score(p, layer.ring, t_pos, h_t, layer.W1, layer.b1, layer.W2, layer.b2, u_t,
                            z_t, stream=score_stream)
        for x in (h_t, k_t, v_t, t_pos, z_t, u_t):
            x.record_stream(score_stream)
        return o, lse, z_t
    if retire and score_stream is not None:
        z_t = torch.empty((p.B, p.Hkv), dtype=torch.uint8, device=q_t.device)
        u_t = torch.empty((p.B, p.Hkv), dtype=torch.float32, device=q_t.device)
        S.spkv_decode_append(p, layer.cache, layer.ring, t_pos, k_t, v_t, None, None, 1)
        if o is None:
            o = torch.empty_like(q_t)
        if lse is None:
            lse = torch.empty((p.B, p.Hq), dtype=torch.float32, device=q_t.device)
        S.spkv_decode_attn(p, layer.cache, layer.ring, q_t, t_pos, o, lse, layer.ws)
        score_stream.wait_stream(torch.cuda.current_stream())
        S.spkv_decode_score(p, layer.ring, t_pos, h_t, layer.W1, layer.b1, layer.W2, layer.b2, u_t,
                            z_t, stream=score_stream)
        for x in (h_t, t_pos, z_t, u_t):
            x.record_stream(score_stream)
        return o, lse, z_t
    if retire and fused:
        z_t = torch.empty((p.B, p.Hkv), dtype=torch.uint8, device=q_t.device)
        u_t = torch.empty((p.B, p.Hkv), dtype=torch.float32, device=q_t.device)
        S.spkv_decode_score_append(p, layer.cache, layer.ring, t_pos, h_t, layer.W1, layer.b1,
                                   layer.W2, layer.b2, k_t, v_t, u_t, z_t, flags=score_flags)
    else:
        if retire:
            u_t, z_t = score(layer, h_t, p.B)
        S.spkv_decode_append(p, layer.cache, layer.ring, t_pos, k_t, v_t, z_t, u_t, retire)
    if o is None:
        o = torch.empty_like(q_t)
    if lse is None:
        lse = torch.empty((p.B, p.Hq), dtype=torch.float32, device=q_t.device)
    S.spkv_decode_attn(p, layer.cache, layer.ring, q_t, t_pos, o, lse, layer.ws)
    return o, lse, z_t


def bulk_compact(layer: Layer, h_buf: torch.Tensor, start_pos: torch.Tensor):
    """Buffered decode: score the ``n`` buffered tokens h_buf [B][n][d_model] whose
    positions start at start_pos [B] and compact their gated rows from the ring."""
    p = layer.p
    B, n = h_buf.shape[0], h_buf.shape[1]
    u, z = score(layer, h_buf, B * n)
    S.spkv_write_compact(p, layer.cache, layer.ring, S.SRC_RING, None, None, z, u, start_pos, n, n)
    return u.view(B, n, p.Hkv), z.view(B, n, p.Hkv)


def cache_lists(layer: Layer):
    """Host copy of every head's cache positions, as a list of int32 arrays."""
    count = layer.cache.count.cpu().numpy()
    table = layer.cache.page_table.cpu().numpy()
    pos = layer.cache.pos_pool.cpu().numpy()
    out = []
    for bh, n in enumerate(count):
        rows = [pos[table[bh, i // S.PAGE_ROWS], i % S.PAGE_ROWS] for i in range(int(n))]
        out.append(torch.tensor(rows, dtype=torch.int32).numpy())
    return out


def cache_rows_kv(layer: Layer, bh: int):
    """Host copies (K, V) [count][d] of one head's cache rows, in cache order."""
    n = int(layer.cache.count[bh].item())
    table = layer.cache.page_table[bh].cpu()
    idx = torch.arange(n)
    pages = table[idx // S.PAGE_ROWS].long()
    K = layer.cache.K_pool.cpu()[pages, idx % S.PAGE_ROWS]
    V = layer.cache.V_pool.cpu()[pages, idx % S.PAGE_ROWS]
    return K, V
