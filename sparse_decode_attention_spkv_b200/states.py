"""Device state of the decode workloads, built through the library.

``build_decode_state`` gives every layer of a per-token-retirement decode workload
its gated cache at the full context (the prefix is scored and compacted chunk by
chunk; the last ``window`` tokens go to the ring with their gates), plus the
per-step decode inputs resident in HBM.  ``DecodeStep`` is the launch sequence of
one decode step over all layers.  Used by ``bench.py`` and ``kernel_driver``.
"""
from __future__ import annotations

import torch

def build_decode_state(wl, layers, steps_total, device):
    """All layers' gated caches at 32K context, built through the library (score and
    compact the prefix; the last 128 tokens go to the ring with their gates), plus
    per-step decode inputs resident in HBM."""
    from sparse_decode_attention_spkv_b200 import runner as R
    from sparse_decode_attention_spkv_b200 import spkv as S
    from sparse_decode_attention_spkv_b200.inputs import device as D
    from sparse_decode_attention_spkv_b200.inputs import gen

    B, Hq, Hkv, d, Dm, w = wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.window
    T0 = wl.ctx[0]
    Tt = wl.T_total
    p = S.make_params(B, Hq, Hkv, d, Dm, wl.hid, w, wl.tau, S.BF16)
    bf = torch.bfloat16
    chunk = 4096
    h_c = torch.empty((B, chunk, Dm), dtype=bf, device=device)
    k_c = torch.empty((B, chunk, Hkv, d), dtype=bf, device=device)
    v_c = torch.empty_like(k_c)
    from sparse_decode_attention_spkv_b200.inputs import workloads as W
    keep_table = W.load_biases()[wl.name]["keep_target"]
    Ls = []
    for l in range(layers):
        W1 = torch.from_numpy(wl.w1(l)).to(bf).to(device)
        b1 = torch.from_numpy(wl.b1(l)).to(device)
        W2 = torch.from_numpy(wl.w2(l)).to(device)
        b2 = torch.from_numpy(wl.b2(l)).to(device)
        rows_head = [min(T0 + steps_total, int(keep_table[l][kh] * 1.15 * T0) + steps_total + 256)
                     for kh in range(Hkv)]
        max_pages = R.pages_for(max(rows_head))
        num_pages = B * sum(R.pages_for(r) for r in rows_head)
        L = R.Layer.create(p, W1, b1, W2, b2, num_pages, max_pages, device)
        kh_, kk_, kv_ = wl.key(l, gen.T_H), wl.key(l, gen.T_K), wl.key(l, gen.T_V)
        for c0 in range(0, T0, chunk):
            n = min(chunk, T0 - c0)
            for b in range(B):
                D.fill_normal(h_c[b, :n], kh_, 1.0, offset=(b * Tt + c0) * Dm)
                D.fill_normal(k_c[b, :n], kk_, wl.qkv_scale, offset=(b * Tt + c0) * Hkv * d)
                D.fill_normal(v_c[b, :n], kv_, wl.qkv_scale, offset=(b * Tt + c0) * Hkv * d)
            hc = h_c[:, :n].contiguous() if n < chunk else h_c
            kc = k_c[:, :n].contiguous() if n < chunk else k_c
            vc = v_c[:, :n].contiguous() if n < chunk else v_c
            _, z = R.score(L, hc, B * n)
            n_compact = max(0, min(c0 + n, T0 - w) - c0)
            src = torch.full((B,), c0, dtype=torch.int32, device=device)
            if n_compact:
                S.spkv_write_compact(p, L.cache, L.ring, S.SRC_CHUNK, kc, vc, z, src, n_compact, n)
            S.spkv_ring_write(p, L.ring, kc, vc, z, n_compact, src, n, n)
        Ls.append(L)
    del h_c, k_c, v_c
    # per-step inputs [steps][layers][B][...] for positions T0, T0+1, ...
    S_ = steps_total
    h_s = torch.empty((layers, B, S_, Dm), dtype=bf, device=device)
    q_s = torch.empty((layers, B, S_, Hq, d), dtype=bf, device=device)
    k_s = torch.empty((layers, B, S_, Hkv, d), dtype=bf, device=device)
    v_s = torch.empty_like(k_s)
    for l in range(layers):
        for b in range(B):
            D.fill_normal(h_s[l, b], wl.key(l, gen.T_H), 1.0, offset=(b * Tt + T0) * Dm)
            D.fill_normal(q_s[l, b], wl.key(l, gen.T_Q), wl.qkv_scale, offset=(b * Tt + T0) * Hq * d)
            D.fill_normal(k_s[l, b], wl.key(l, gen.T_K), wl.qkv_scale, offset=(b * Tt + T0) * Hkv * d)
            D.fill_normal(v_s[l, b], wl.key(l, gen.T_V), wl.qkv_scale, offset=(b * Tt + T0) * Hkv * d)
    inputs = {
        "h": h_s.permute(2, 0, 1, 3).contiguous(),
        "q": q_s.permute(2, 0, 1, 3, 4).contiguous(),
        "k": k_s.permute(2, 0, 1, 3, 4).contiguous(),
        "v": v_s.permute(2, 0, 1, 3, 4).contiguous(),
        "t": (torch.arange(S_, dtype=torch.int32, device=device) + T0).view(S_, 1).repeat(1, B).contiguous(),
    }
    del h_s, q_s, k_s, v_s
    torch.cuda.synchronize()
    for L in Ls:
        status, flags = S.spkv_cache_check(L.cache)
        if status != S.OK:
            raise RuntimeError(f"cache setup failed: {S.status_str(status)} flags={flags}")
    return p, Ls, inputs


class DecodeStep:
    """Launch sequence of one decode step (all layers) on fixed buffers."""

    def __init__(self, p, layers, device):
        from sparse_decode_attention_spkv_b200 import spkv as S
        self.S, self.p, self.layers = S, p, layers
        n = len(layers)
        self.o = torch.empty((n, p.B, p.Hq, p.head_dim), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty((n, p.B, p.Hq), dtype=torch.float32, device=device)
        self.u = torch.empty((n, p.B, p.Hkv), dtype=torch.float32, device=device)
        self.z = torch.empty((n, p.B, p.Hkv), dtype=torch.uint8, device=device)

    def launch(self, h, q, k, v, t, ev=None):
        """h [L][B][D], q [L][B][Hq][d], k, v [L][B][Hkv][d], t [B]; ev: per-layer
        (start, end) timing events around the decode-attention launch."""
        S, p = self.S, self.p
        for l, L in enumerate(self.layers):
            S.spkv_score(p, h[l], p.B, L.W1, L.b1, L.W2, L.b2, self.u[l], self.z[l])
            S.spkv_decode_append(p, L.cache, L.ring, t, k[l], v[l], self.z[l], 1)
            if ev is not None:
                ev[l][0].record()
            S.spkv_decode_attn(p, L.cache, L.ring, q[l], t, self.o[l], self.lse[l], L.ws)
            if ev is not None:
                ev[l][1].record()

    LAUNCHES_PER_LAYER = 3


def kv_bytes(p, layers, t):
    """Algorithmic K/V bytes of one decode step at query position t: every head reads
    its live cache rows and its window rows once (K and V, bf16)."""
    total = 0
    n_win = min(p.window, t + 1)
    for L in layers:
        total += int((L.cache.count.to(torch.int64) + n_win).sum().item())
    return total * 2 * p.head_dim * 2
