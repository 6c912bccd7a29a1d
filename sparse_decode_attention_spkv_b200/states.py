"""Device state of the decode workloads, built through the library.

``build_decode_state`` gives every layer of a decode workload its gated cache at the
workload's context (each batch row may have its own context length): the prefix is
scored and compacted chunk by chunk, and the last ``window`` tokens of every row go
to the ring.  Two end states:

* per-token retirement (default): the cache holds the gated tokens that have left
  the window, the ring holds the last ``window`` tokens with their gates;
* buffered (``compact_window=True``): every gated token of the context is already in
  the cache and the ring's gates are 0 ("already cached").

It also draws the per-step decode inputs into HBM.  ``DecodeStep`` is the launch
sequence of one per-token decode step over all layers.  Used by ``bench.py``,
``kernel_driver`` and the full-size GPU tests.
"""
from __future__ import annotations

import torch


def build_decode_state(wl, layers, steps_total, device, compact_window: bool = False,
                       chunk: int = 0, store_u: bool = False, row0: int = 0,
                       pos_range=None, with_ring: bool = True):
    """Returns (params, [Layer], inputs) where inputs["h"|"q"|"k"|"v"][i][l] are step i's
    tensors of layer l and inputs["t"][i] the positions [B] of step i.  store_u keeps the
    utilities of cached rows and pending window slots (for re-thresholding).

    row0: the global index of batch row 0 (a rank serving rows row0 .. row0+B-1 of a
    larger batch draws exactly those rows' inputs: every seeded stream is indexed by the
    global row).  pos_range (lo, hi), per-row lists (hi None: no upper bound): only the
    gated positions in [lo, hi) are written to the cache -- one slice of a sequence whose
    cache is split by position; with_ring False leaves the ring unwritten (a slice that
    does not hold the window)."""
    from sparse_decode_attention_spkv_b200 import runner as R
    from sparse_decode_attention_spkv_b200 import spkv as S
    from sparse_decode_attention_spkv_b200.inputs import device as D
    from sparse_decode_attention_spkv_b200.inputs import gen
    from sparse_decode_attention_spkv_b200.inputs import workloads as W

    B, Hq, Hkv, d, Dm, w = wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.window
    ctx = [int(c) for c in wl.ctx]
    assert len(ctx) == B and min(ctx) >= w
    Tmax = max(ctx)
    Tt = wl.T_total
    p = S.make_params(B, Hq, Hkv, d, Dm, wl.hid, w, wl.tau, S.BF16)
    bf = torch.bfloat16
    if not chunk:
        chunk = 4096 if B <= 8 else 1024
    h_c = torch.empty((B, chunk, Dm), dtype=bf, device=device)
    k_c = torch.empty((B, chunk, Hkv, d), dtype=bf, device=device)
    v_c = torch.empty_like(k_c)
    # per row: positions below `limit` are compacted from the chunks
    limit = torch.tensor([c if compact_window else c - w for c in ctx], dtype=torch.int32,
                         device=device)
    if pos_range is not None:  # a slice: positions outside [lo, hi) stay out of this cache
        lo_l, hi_l = pos_range
        lo_t = torch.tensor([int(x) for x in lo_l], dtype=torch.int32, device=device)
        hi_t = torch.tensor([c + steps_total if h is None else int(h) for c, h in zip(ctx, hi_l)],
                            dtype=torch.int32, device=device)
        limit = torch.minimum(limit, hi_t)
    else:
        lo_t = torch.zeros(B, dtype=torch.int32, device=device)
    keep_table = W.load_biases()[wl.name]["keep_target"]
    Ls = []
    for l in range(layers):
        W1 = torch.from_numpy(wl.w1(l)).to(bf).to(device)
        b1 = torch.from_numpy(wl.b1(l)).to(device)
        W2 = torch.from_numpy(wl.w2(l)).to(device)
        b2 = torch.from_numpy(wl.b2(l)).to(device)
        rows_head = [min(Tmax + steps_total,
                         int(keep_table[l][kh] * 1.15 * Tmax) + steps_total + 512) for kh in range(Hkv)]
        max_pages = R.pages_for(max(rows_head))
        num_pages = B * sum(R.pages_for(r) for r in rows_head)
        L = R.Layer.create(p, W1, b1, W2, b2, num_pages, max_pages, device, store_u=store_u)
        kh_, kk_, kv_ = wl.key(l, gen.T_H), wl.key(l, gen.T_K), wl.key(l, gen.T_V)
        n_lim = max(limit.tolist())
        for c0 in range(0, n_lim, chunk):
            n = min(chunk, n_lim - c0)
            for b in range(B):
                g = row0 + b
                D.fill_normal(h_c[b, :n], kh_, 1.0, offset=(g * Tt + c0) * Dm)
                D.fill_normal(k_c[b, :n], kk_, wl.qkv_scale, offset=(g * Tt + c0) * Hkv * d)
                D.fill_normal(v_c[b, :n], kv_, wl.qkv_scale, offset=(g * Tt + c0) * Hkv * d)
            hc = h_c[:, :n].contiguous() if n < chunk else h_c
            kc = k_c[:, :n].contiguous() if n < chunk else k_c
            vc = v_c[:, :n].contiguous() if n < chunk else v_c
            u, z = R.score(L, hc, B * n)
            z = z.view(B, n, Hkv)
            pos = torch.arange(c0, c0 + n, dtype=torch.int32, device=device)
            keep = (pos[None, :] < limit[:, None]) & (pos[None, :] >= lo_t[:, None])
            z.mul_(keep.to(torch.uint8)[:, :, None])  # beyond a row's prefix or outside the slice
            src = torch.full((B,), c0, dtype=torch.int32, device=device)
            S.spkv_write_compact(p, L.cache, L.ring, S.SRC_CHUNK, kc, vc, z, u, src, n, n)
        # the ring: each row's last w tokens, gated (per-token) or marked as cached
        kr = torch.empty((B, w, Hkv, d), dtype=bf, device=device)
        vr = torch.empty_like(kr)
        hr = torch.empty((B, w, Dm), dtype=bf, device=device)
        for b in range(B):
            s0 = ctx[b] - w
            g = row0 + b
            D.fill_normal(hr[b], kh_, 1.0, offset=(g * Tt + s0) * Dm)
            D.fill_normal(kr[b], kk_, wl.qkv_scale, offset=(g * Tt + s0) * Hkv * d)
            D.fill_normal(vr[b], kv_, wl.qkv_scale, offset=(g * Tt + s0) * Hkv * d)
        if with_ring:
            ur, zr = R.score(L, hr, B * w)
            src = torch.tensor([c - w for c in ctx], dtype=torch.int32, device=device)
            S.spkv_ring_write(p, L.ring, kr, vr, zr, ur, w if compact_window else 0, src, w, w)
        Ls.append(L)
    del h_c, k_c, v_c
    # per-step inputs [steps][layers][B][...]; row b's step i is position ctx[b] + i
    S_ = steps_total
    h_s = torch.empty((layers, B, S_, Dm), dtype=bf, device=device)
    q_s = torch.empty((layers, B, S_, Hq, d), dtype=bf, device=device)
    k_s = torch.empty((layers, B, S_, Hkv, d), dtype=bf, device=device)
    v_s = torch.empty_like(k_s)
    for l in range(layers):
        for b in range(B):
            t0 = ctx[b]
            g = row0 + b
            D.fill_normal(h_s[l, b], wl.key(l, gen.T_H), 1.0, offset=(g * Tt + t0) * Dm)
            D.fill_normal(q_s[l, b], wl.key(l, gen.T_Q), wl.qkv_scale, offset=(g * Tt + t0) * Hq * d)
            D.fill_normal(k_s[l, b], wl.key(l, gen.T_K), wl.qkv_scale, offset=(g * Tt + t0) * Hkv * d)
            D.fill_normal(v_s[l, b], wl.key(l, gen.T_V), wl.qkv_scale, offset=(g * Tt + t0) * Hkv * d)
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device=device)
    inputs = {
        "h": h_s.permute(2, 0, 1, 3).contiguous(),
        "q": q_s.permute(2, 0, 1, 3, 4).contiguous(),
        "k": k_s.permute(2, 0, 1, 3, 4).contiguous(),
        "v": v_s.permute(2, 0, 1, 3, 4).contiguous(),
        "t": (torch.arange(S_, dtype=torch.int32, device=device)[:, None] + ctx_t[None, :]).contiguous(),
        "h_layer_row": h_s,   # [layers][B][steps][d_model] (buffered scoring reads windows of it)
    }
    del q_s, k_s, v_s
    torch.cuda.synchronize()
    for L in Ls:
        status, flags = S.spkv_cache_check(L.cache)
        if status != S.OK:
            raise RuntimeError(f"cache setup failed: {S.status_str(status)} flags={flags}")
    return p, Ls, inputs


class DecodeStep:
    """Launch sequence of one decode step (all layers) on fixed buffers.

    Default: per layer, the fused score + retire + ring write, then the attention.  With
    ``split``, the scoring leaves the attention's path: per layer the retirement and ring
    write (gate of the new token left at 0), then the attention, and on a second stream
    the scoring of the layer's new tokens, which stores their gates in their window slots
    while the next layers run (a gate is read only when its token leaves the window).
    With ``split`` and ``attn_first`` (the default where the kernels support it) the
    attention runs first, on the state before the step's update, and the retirement, ring
    write and scoring all run on the second stream: the attention of the next layer
    follows the previous one directly.  With ``attn_first`` alone, each layer's attention
    (on the state before the update) is followed on the same stream by the fused score,
    retirement and ring write: for a single layer, whose next attention needs the update
    anyway, this saves the second stream's fork and join.  ``inputs_settled``: the hidden
    states given to ``launch`` are written before the step begins (no kernel that writes
    them can still be running), so the fused score may run its perceptron while the
    attention finishes (SPKV_INPUTS_SETTLED)."""

    def __init__(self, p, layers, device, split: bool = False, attn_first=None,
                 inputs_settled: bool = False):
        from sparse_decode_attention_spkv_b200 import spkv as S
        self.S, self.p, self.layers = S, p, layers
        self.score_flags = S.INPUTS_SETTLED if inputs_settled else 0
        if attn_first is None:
            attn_first = split and S.spkv_decode_attn_before_append_supported(p)
        if attn_first and not S.spkv_decode_attn_before_append_supported(p):
            raise ValueError("attention before the update is not built for these shapes")
        self.attn_first = bool(attn_first)
        n = len(layers)
        self.o = torch.empty((n, p.B, p.Hq, p.head_dim), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty((n, p.B, p.Hq), dtype=torch.float32, device=device)
        self.u = torch.empty((n, p.B, p.Hkv), dtype=torch.float32, device=device)
        self.z = torch.empty((n, p.B, p.Hkv), dtype=torch.uint8, device=device)
        self.split = split
        if split:
            self.side = torch.cuda.Stream(device=device)
            self.fork = [torch.cuda.Event() for _ in layers]

    def launch(self, h, q, k, v, t, ev=None):
        """h [L][B][D], q [L][B][Hq][d], k, v [L][B][Hkv][d], t [B]; ev: {layer: (start,
        end)} timing events around the decode-attention call of the listed layers (an
        event between two launches keeps the second from starting early, so only a
        sample of layers carries them)."""
        S, p = self.S, self.p
        main = torch.cuda.current_stream()
        for l, L in enumerate(self.layers):
            if self.attn_first:
                e = ev.get(l) if ev else None
                if e is not None:
                    e[0].record()
                # layer l's cache and ring were last written on the second stream, joined
                # at the end of the previous step: settled
                S.spkv_decode_attn_before_append(p, L.cache, L.ring, q[l], t, k[l], v[l],
                                                 self.o[l], self.lse[l], L.ws,
                                                 flags=S.DECODE_STATE_SETTLED)
                if e is not None:
                    e[1].record()
                if not self.split:  # score, retire t - w, store the new token: one launch
                    S.spkv_decode_score_append(p, L.cache, L.ring, t, h[l], L.W1, L.b1, L.W2,
                                               L.b2, k[l], v[l], self.u[l], self.z[l],
                                               flags=self.score_flags)
                    continue
                # retire t - w, store the new token (gate 0), then its gate: beside the
                # following layers' attention
                self.fork[l].record(main)
                self.side.wait_event(self.fork[l])
                S.spkv_decode_append(p, L.cache, L.ring, t, k[l], v[l], None, None, 1,
                                     stream=self.side)
                S.spkv_decode_score(p, L.ring, t, h[l], L.W1, L.b1, L.W2, L.b2, self.u[l],
                                    self.z[l], stream=self.side)
                continue
            if self.split:  # retire t - w, store the new token (gate 0 for now)
                S.spkv_decode_append(p, L.cache, L.ring, t, k[l], v[l], None, None, 1)
            else:  # score the new token, retire t - w, store the new token: one launch
                S.spkv_decode_score_append(p, L.cache, L.ring, t, h[l], L.W1, L.b1, L.W2, L.b2,
                                           k[l], v[l], self.u[l], self.z[l])
            e = ev.get(l) if ev else None
            if e is not None:
                e[0].record()
            S.spkv_decode_attn(p, L.cache, L.ring, q[l], t, self.o[l], self.lse[l], L.ws)
            if e is not None:
                e[1].record()
            if self.split:  # the new tokens' gates, beside the following layers
                self.fork[l].record(main)
                self.side.wait_event(self.fork[l])
                S.spkv_decode_score(p, L.ring, t, h[l], L.W1, L.b1, L.W2, L.b2, self.u[l],
                                    self.z[l], stream=self.side)
        if self.split:
            main.wait_stream(self.side)

    LAUNCHES_PER_LAYER = 2  # plus one on the second stream when split


def kv_bytes(p, layers, t_min):
    """Algorithmic K/V bytes of one decode step: every head reads its live cache rows and
    its window rows once (K and V, bf16).  (The cache holds only rows <= t - w in the
    per-token schedule, so count is the live row count.)"""
    return sum(kv_bytes_layers(p, layers, t_min))


def kv_bytes_layers(p, layers, t_min):
    """kv_bytes per layer (a list)."""
    n_win = min(p.window, t_min + 1)
    return [int((L.cache.count.to(torch.int64) + n_win).sum().item()) * 2 * p.head_dim * 2
            for L in layers]


class HybridStep:
    """Launch sequence of one decode step over a hybrid local/global stack: layer l is
    global (SP-KV: score, retire, attend over cache + window) when l % period ==
    period - 1, else local (window only, no cache).  With ``attn_first`` (the default
    where the kernels support it) every layer's attention runs on the state before the
    step's update, and the updates (and the global layers' scoring) go to a second
    stream, as in DecodeStep."""

    def __init__(self, p, global_layers, local_layers, period, device, attn_first=None):
        from sparse_decode_attention_spkv_b200 import spkv as S
        self.S, self.p, self.period = S, p, period
        self.glob, self.loc = global_layers, local_layers
        n = len(global_layers) + len(local_layers)
        self.n = n
        if attn_first is None:
            attn_first = S.spkv_decode_attn_before_append_supported(p)
        self.attn_first = bool(attn_first)
        if self.attn_first:
            self.side = torch.cuda.Stream(device=device)
            self.fork = [torch.cuda.Event() for _ in range(n)]
        self.o = torch.empty((n, p.B, p.Hq, p.head_dim), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty((n, p.B, p.Hq), dtype=torch.float32, device=device)
        self.u = torch.empty((len(global_layers), p.B, p.Hkv), dtype=torch.float32, device=device)
        self.z = torch.empty((len(global_layers), p.B, p.Hkv), dtype=torch.uint8, device=device)

    def launch(self, h, q, k, v, t):
        """h, q, k, v indexed by global-layer number (local layers reuse q, k, v of
        global layer l // period: their values do not change the work)."""
        S, p = self.S, self.p
        if self.attn_first:
            self._launch_attn_first(h, q, k, v, t)
            return
        gi = li = 0
        for l in range(self.n):
            g = l // self.period
            if l % self.period == self.period - 1:
                L = self.glob[gi]
                S.spkv_decode_score_append(p, L.cache, L.ring, t, h[g], L.W1, L.b1, L.W2, L.b2,
                                           k[g], v[g], self.u[gi], self.z[gi])
                S.spkv_decode_attn(p, L.cache, L.ring, q[g], t, self.o[l], self.lse[l], L.ws)
                gi += 1
            else:
                L = self.loc[li]
                S.spkv_decode_append(p, None, L.ring, t, k[g], v[g], None, None, 0)
                S.spkv_decode_attn(p, None, L.ring, q[g], t, self.o[l], self.lse[l], L.ws)
                li += 1

    def _launch_attn_first(self, h, q, k, v, t):
        S, p = self.S, self.p
        main = torch.cuda.current_stream()
        gi = li = 0
        for l in range(self.n):
            g = l // self.period
            glob = l % self.period == self.period - 1
            L = self.glob[gi] if glob else self.loc[li]
            cache = L.cache if glob else None
            # every layer's cache and ring were last written on the second stream, joined
            # at the end of the previous step: settled
            S.spkv_decode_attn_before_append(p, cache, L.ring, q[g], t, k[g], v[g], self.o[l],
                                             self.lse[l], L.ws, flags=S.DECODE_STATE_SETTLED)
            self.fork[l].record(main)
            self.side.wait_event(self.fork[l])
            if glob:
                S.spkv_decode_append(p, L.cache, L.ring, t, k[g], v[g], None, None, 1,
                                     stream=self.side)
                S.spkv_decode_score(p, L.ring, t, h[g], L.W1, L.b1, L.W2, L.b2, self.u[gi],
                                    self.z[gi], stream=self.side)
                gi += 1
            else:
                S.spkv_decode_append(p, None, L.ring, t, k[g], v[g], None, None, 0,
                                     stream=self.side)
                li += 1
        main.wait_stream(self.side)

    LAUNCHES_GLOBAL = 2
    LAUNCHES_LOCAL = 2
