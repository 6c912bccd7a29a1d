"""Sequence split: one sequence's key set decoded slice by slice and merged (GPU
required).

Each slice is a cache holding the gated rows of a range of positions (the last one
also holds the window and takes the per-token retirements).  Every slice's partial
(spkv_decode_attn_partial) is checked against the oracle's Eq. (3) over that slice's
keys alone, and the merge of the partials (spkv_decode_merge) against the oracle's
attention over the whole key set, at every decode step.  The slices live on one GPU
here; across GPUs only the exchange of the partials differs (tested with gloo ranks
on the CPU).
"""
import numpy as np
import pytest
import torch

from oracle import spkv_oracle as O
from sparse_decode_attention_spkv_b200.inputs import workloads as W
from tests import cases as C

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from sparse_decode_attention_spkv_b200 import runner as R
    from sparse_decode_attention_spkv_b200 import seqsplit as SS
    from sparse_decode_attention_spkv_b200 import spkv as S


def _slices(wl, T0, bounds, window_only_last=False):
    """Layers of a sequence split at the given position bounds (same for every row):
    slice i caches the gated rows with positions in [bounds[i], bounds[i+1]) that have
    left the window at T0; the last slice also holds the ring (with the gates of its
    tokens).  window_only_last: the last slice is the window alone (no cache).  Returns
    (p, layers, host rows h, q, k, v over T0 + steps, weights)."""
    W1, b1, W2, b2 = C.weights(wl)
    p = S.make_params(wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau,
                      S.BF16)
    T = T0 + wl.decode_steps
    rows = [C.host_rows(wl, 0, b, np.arange(T)) for b in range(wl.B)]
    h, q, k, v = (np.stack([r[i] for r in rows]) for i in range(4))
    w = wl.window
    n_sl = len(bounds) - 1
    mp = R.pages_for(T)
    layers = []
    for i in range(n_sl):
        if window_only_last and i == n_sl - 1:
            layers.append(R.Layer.create_local(p))
        else:
            layers.append(R.Layer.create(p, C.dev(W1, "bf16"), C.dev_f32(b1), C.dev_f32(W2),
                                         C.dev_f32(b2), num_pages=wl.B * wl.Hkv * mp,
                                         max_pages_per_head=mp))
    L0 = layers[0]
    u, z = R.score(L0, C.dev(h[:, :T0].reshape(-1, wl.d_model), "bf16"), wl.B * T0)
    z = z.view(wl.B, T0, wl.Hkv)
    u = u.view(wl.B, T0, wl.Hkv)
    kd, vd = C.dev(k[:, :T0], "bf16"), C.dev(v[:, :T0], "bf16")
    pos = torch.arange(T0, device="cuda")
    src = torch.zeros(wl.B, dtype=torch.int32, device="cuda")
    # rows that have left the window at T0 are cached; with a window-only last slice the
    # first step's retiring row (T0 - w) is cached too (the window slice keeps no cache)
    cut = T0 - w + (1 if window_only_last else 0)
    for i, L in enumerate(layers):
        if L.local:
            continue
        lo, hi = bounds[i], min(bounds[i + 1], cut)
        keep = ((pos >= lo) & (pos < hi)).to(torch.uint8)[None, :, None]
        S.spkv_write_compact(p, L.cache, L.ring, S.SRC_CHUNK, kd, vd, (z * keep).contiguous(), u,
                             src, T0, T0)
    last = layers[-1]
    src_w = torch.full((wl.B,), T0 - w, dtype=torch.int32, device="cuda")
    S.spkv_ring_write(p, last.ring, kd[:, T0 - w:].contiguous(), vd[:, T0 - w:].contiguous(),
                      z[:, T0 - w:].contiguous(), u[:, T0 - w:].contiguous(), 0, src_w, w, w)
    return p, layers, (h, q, k, v), (W1, b1, W2, b2)


def _run_and_check(name, wl, T0, bounds, window_only_last=False):
    p, layers, (h, q, k, v), (W1, b1, W2, b2) = _slices(wl, T0, bounds, window_only_last)
    w = wl.window
    sls = [SS.SliceDecode(p, None if L.local else L.cache, L.ring, i == len(layers) - 1, "cuda")
           for i, L in enumerate(layers)]
    u_ref, z_ref = C.oracle_gates(h.reshape(-1, wl.d_model), W1, b1, W2, b2, wl.tau)
    z_ref = z_ref.reshape(wl.B, -1, wl.Hkv)
    s_all = np.arange(h.shape[1])
    last = layers[-1]
    for i in range(wl.decode_steps):
        t = T0 + i
        t_pos = torch.full((wl.B,), t, dtype=torch.int32, device="cuda")
        kt, vt = C.dev(k[:, t], "bf16"), C.dev(v[:, t], "bf16")
        if last.local:  # a window-only slice: nothing retires (one step only)
            S.spkv_decode_append(p, None, last.ring, t_pos, kt, vt, None, None, 0)
        else:           # the token leaving the window goes to the last slice's cache
            u_t, z_t = R.score(last, C.dev(h[:, t], "bf16"), wl.B)
            S.spkv_decode_append(p, last.cache, last.ring, t_pos, kt, vt, z_t, u_t, 1)
        qt = C.dev(q[:, t], "bf16")
        o = torch.empty_like(qt)
        lse = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
        SS.merge_local(p, sls, qt, t_pos, o, lse)
        parts = [(sl.partial(qt, t_pos)[0].cpu().numpy().copy(), sl.lse_part.cpu().numpy().copy())
                 for sl in sls]
        torch.cuda.synchronize()
        o_g, lse_g = C.to_np(o), lse.cpu().numpy()
        for b in range(wl.B):
            o_ref, lse_ref = O.gated_attention(q[b, t:t + 1], k[b, :t + 1], v[b, :t + 1],
                                               z_ref[b, :t + 1], w, [t])
            C.check_attn(o_g[b], o_ref[0], "bf16", f"{name} step {i} row {b}: merged")
            assert np.max(np.abs(lse_g[b] - lse_ref[0])) < 1e-3, f"{name} step {i}: lse"
            # each slice alone: Eq. (3) over the slice's keys
            for j, (op, lp) in enumerate(parts):
                lo = bounds[j]
                hi = bounds[j + 1] if j < len(bounds) - 2 else t + 1
                for kh in range(wl.Hkv):
                    vis = O.visible(t, s_all[:t + 1], z_ref[b, :t + 1, kh], w)
                    if j == len(parts) - 1:   # the last slice: its range and the window
                        in_sl = (s_all[:t + 1] >= lo) | (t - s_all[:t + 1] < w)
                        if last.local:
                            in_sl = t - s_all[:t + 1] < w
                    else:
                        in_sl = (s_all[:t + 1] >= lo) & (s_all[:t + 1] < hi) & \
                            (t - s_all[:t + 1] >= w)
                    mask = vis & in_sl
                    for g in range(wl.G):
                        hq = kh * wl.G + g
                        if not mask.any():
                            assert lp[b, hq] == -np.inf and np.all(op[b, hq] == 0), \
                                f"{name} slice {j}: empty slice"
                            continue
                        o_s, l_s = O.attend(q[b, t, hq], k[b, :t + 1, kh], v[b, :t + 1, kh], mask)
                        C.check_attn(op[b, hq][None], o_s[None], "bf16",
                                     f"{name} step {i} slice {j} head {hq}")
                        assert abs(lp[b, hq] - l_s) < 1e-3, f"{name} slice {j}: lse"
    for L in layers:
        if not L.local:
            status, flags = S.spkv_cache_check(L.cache)
            assert status == S.OK, flags


CASES = {
    "g4_d128_two_slices": (W.small_case("decode32k", cid=70, B=2, Hq=8, Hkv=2, d_model=128,
                                        hid=32, ctx=[2000], decode_steps=4, layers=1,
                                        keep="u05_50"), 2000, [0, 700, 10 ** 9]),
    # a tiny middle slice: some heads keep no row in it (empty partial, lse = -inf)
    "g8_d64_three_slices": (W.small_case("decode32k", cid=71, B=2, Hq=8, Hkv=1, head_dim=64,
                                         d_model=128, hid=32, ctx=[1500], decode_steps=3,
                                         layers=1, keep="fixed25"), 1500, [0, 500, 504, 10 ** 9]),
    "g2_spread_keep_two_slices": (W.small_case("decode32k", cid=72, B=1, Hq=16, Hkv=8,
                                               d_model=128, hid=32, ctx=[1300], decode_steps=3,
                                               layers=1, keep="spread"), 1300, [0, 640, 10 ** 9]),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_split_decode_matches_oracle(name):
    wl, T0, bounds = CASES[name]
    _run_and_check(name, wl, T0, bounds)


def test_split_decode_window_only_slice():
    """Two slices: every cached row in the first; the second is the window alone (no
    cache), read through the ring; one step."""
    wl = W.small_case("decode32k", cid=73, B=2, Hq=8, Hkv=2, d_model=128, hid=32, ctx=[900],
                      decode_steps=1, layers=1, keep="u05_50")
    _run_and_check("window-only slice", wl, 900, [0, 10 ** 9, 10 ** 9], window_only_last=True)


def test_merge_of_one_part_is_the_part():
    """One part: the merge returns it (rounded to the output type) and its lse."""
    p = S.make_params(2, 4, 2, 128, 64, 32, 128, 0.5, S.F32)
    o_p = torch.randn((1, 2, 4, 128), device="cuda")
    l_p = torch.randn((1, 2, 4), device="cuda")
    o = torch.empty((2, 4, 128), device="cuda")
    lse = torch.empty((2, 4), device="cuda")
    S.spkv_decode_merge(p, 1, o_p, l_p, o, lse)
    torch.cuda.synchronize()
    assert torch.allclose(o, o_p[0], atol=1e-6) and torch.allclose(lse, l_p[0], atol=1e-6)


def test_split_decode_ragged128k_full_size():
    """ragged128k (contexts 128K, 96K, 64K, 32K), one layer, each row's cache split into
    two halves by position, one per-token decode step: the merged output equals the
    unsplit decode of the same state, and the oracle on sampled rows."""
    from sparse_decode_attention_spkv_b200.states import build_decode_state
    wl = W.small_case("ragged128k", layers=1)
    dev = torch.device("cuda")
    (lo0, hi0), (lo1, hi1) = SS.split_bounds(wl.ctx, 2, wl.window)
    p, (LA,), inp = build_decode_state(wl, 1, 1, dev, pos_range=(lo0, hi0), with_ring=False)
    _, (LB,), _ = build_decode_state(wl, 1, 1, dev, pos_range=(lo1, hi1))
    _, (LF,), _ = build_decode_state(wl, 1, 1, dev)
    t = inp["t"][0]
    h, q, k, v = inp["h"][0][0], inp["q"][0][0], inp["k"][0][0], inp["v"][0][0]
    o_full, _, z_full = R.decode_step(LF, t, h, q, k, v)
    u_t, z_t = R.score(LB, h, p.B)
    S.spkv_decode_append(p, LB.cache, LB.ring, t, k, v, z_t, u_t, 1)
    sls = [SS.SliceDecode(p, LA.cache, None, False, dev), SS.SliceDecode(p, LB.cache, LB.ring, True, dev)]
    o = torch.empty_like(q)
    SS.merge_local(p, sls, q, t, o)
    torch.cuda.synchronize()
    for L in (LA, LB, LF):
        status, flags = S.spkv_cache_check(L.cache)
        assert status == S.OK, flags
    # the two slices hold exactly the rows of the unsplit cache, none twice
    la, lb, lf = R.cache_lists(LA), R.cache_lists(LB), R.cache_lists(LF)
    for bh in range(p.B * p.Hkv):
        assert np.array_equal(np.concatenate([la[bh], lb[bh]]), lf[bh]), f"head {bh}: rows"
    C.check_attn(C.to_np(o), C.to_np(o_full), "bf16", "split vs unsplit decode")
    W1, b1, W2, b2 = C.weights(wl)
    t_np = t.cpu().numpy()
    o_np = C.to_np(o)
    for b in (3, 2):
        tb = int(t_np[b])
        u, z = C.oracle_gates_rows(wl, 0, b, tb + 1, W1, b1, W2, b2)
        K, V = C.kv_rows(wl, 0, b, tb + 1)
        o_ref, _ = O.gated_attention(wl.q_rows(0, b, [tb]), K, V, z, wl.window, [tb])
        C.check_attn(o_np[b], o_ref[0], "bf16", f"ragged128k split, row {b}")
