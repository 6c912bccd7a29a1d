"""Post-hoc re-threshold of a filled cache ("Self-Pruned Key-Value Attention", §3.3:
the sparsity can be changed after the fact by changing tau) against the oracle
(GPU required).

A cache is filled by chunked prefill with utilities kept (the last `window` tokens
pending in the ring), re-thresholded in place at tau' > tau, and then decoded with
per-token retirement at tau'.  Checked: stored utilities, the cache index lists and
stored rows after the change (oracle: ``rethreshold``), the ring's recomputed gates,
that no page leaves its head, and every decode output against Eqs. (3)-(4) with all
gates at tau'."""
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


CASES = {
    # few-token score on CUDA cores, head_dim 128, 4 query heads per key head
    "bf16_g4": (W.small_case("decode32k", cid=60, B=2, Hq=8, Hkv=2, d_model=256, hid=64,
                             ctx=[3000], decode_steps=150, layers=1, keep="u05_50"), 0.62),
    # fp32 path, head_dim 64
    "f32_tiny": (W.small_case("tiny", cid=61, B=2, ctx=[1500], decode_steps=140), 0.6),
    # d_model 4096, hid 128: the tensor-core score with the fused append
    "bf16_mma_score": (W.small_case("decode32k", cid=62, B=4, ctx=[1300], decode_steps=140,
                                    layers=1, keep="fixed25"), 0.55),
}


def _params(wl, tau):
    return S.make_params(wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, tau,
                         S.BF16 if wl.dtype == "bf16" else S.F32)


def _rows(wl, T):
    hs, qs, ks, vs = [], [], [], []
    for b in range(wl.B):
        h, q, k, v = C.host_rows(wl, 0, b, np.arange(T))
        hs.append(h); qs.append(q); ks.append(k); vs.append(v)
    return np.stack(hs), np.stack(qs), np.stack(ks), np.stack(vs)


def _check_list_two(got, want, u_col, taus):
    """Index lists equal away from both thresholds."""
    near = set()
    for tau in taus:
        near |= set(np.nonzero(np.abs(u_col - tau) < C.EXCLUDE)[0].tolist())
    a = [int(x) for x in got if int(x) not in near]
    c = [int(x) for x in want if int(x) not in near]
    assert a == c, f"cache list differs away from the thresholds ({len(a)} vs {len(c)} rows)"


@pytest.mark.parametrize("name", sorted(CASES))
def test_rethreshold_then_decode_matches_oracle(name):
    wl, tau2 = CASES[name]
    T0, steps, w = wl.ctx[0], wl.decode_steps, wl.window
    T = T0 + steps
    W1, b1, W2, b2 = C.weights(wl)
    p = _params(wl, wl.tau)
    mp = R.pages_for(T)
    layer = R.Layer.create(p, C.dev(W1, wl.dtype), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                           num_pages=wl.B * wl.Hkv * mp, max_pages_per_head=mp, store_u=True)
    h, q, k, v = _rows(wl, T)
    for c0 in range(0, T0, 512):  # per-token-ready prefill: the last w tokens stay pending
        c1 = min(T0, c0 + 512)
        R.prefill_chunk(layer, C.dev(h[:, c0:c1], wl.dtype), C.dev(q[:, c0:c1], wl.dtype),
                        C.dev(k[:, c0:c1], wl.dtype), C.dev(v[:, c0:c1], wl.dtype), c0,
                        n_compact=max(0, min(c1, T0 - w) - c0))
    u_ref = O.utility(h.reshape(-1, wl.d_model), W1, b1, W2, b2).reshape(wl.B, T, wl.Hkv)
    z_ref = O.gate(u_ref, wl.tau)

    # utilities stored with the cached rows and the pending window slots
    lists0 = R.cache_lists(layer)
    upool = layer.cache.u_pool.cpu().numpy()
    table0 = layer.cache.page_table.cpu().numpy()
    for b in range(wl.B):
        for kh in range(wl.Hkv):
            bh = b * wl.Hkv + kh
            C.check_list(lists0[bh], z_ref[b, :, kh], T0 - w, u_ref[b, :, kh], wl.tau)
            idx = np.arange(len(lists0[bh]))
            got_u = upool[table0[bh, idx // S.PAGE_ROWS], idx % S.PAGE_ROWS]
            assert np.max(np.abs(got_u - u_ref[b, lists0[bh], kh]), initial=0.0) <= 1e-5
    u_win = layer.ring.u_win.cpu().numpy()          # [B][w][Hkv]
    slots = np.arange(T0 - w, T0) % w
    assert np.max(np.abs(u_win[:, slots] - u_ref[:, T0 - w:T0])) <= 1e-5

    # re-threshold in place
    top0 = int(layer.cache.pool_top.item())
    ws = S.alloc_rethreshold_workspace(p, layer.cache)
    S.spkv_cache_rethreshold(p, layer.cache, layer.ring, tau2, ws)
    status, flags = S.spkv_cache_check(layer.cache)
    assert status == S.OK, flags
    assert int(layer.cache.pool_top.item()) == top0
    assert int(ws[:4].view(torch.int32).item()) == 0  # work counter left at zero
    lists1 = R.cache_lists(layer)
    upool1 = layer.cache.u_pool.cpu().numpy()
    table1 = layer.cache.page_table.cpu().numpy()
    assert np.array_equal(table1, table0)  # every page stays with its head
    for b in range(wl.B):
        for kh in range(wl.Hkv):
            bh = b * wl.Hkv + kh
            u_cached = u_ref[b, lists0[bh], kh]
            want = O.rethreshold(lists0[bh], u_cached, tau2)
            _check_list_two(lists1[bh], want, u_ref[b, :, kh], (wl.tau, tau2))
            assert int(layer.cache.count_prev[bh]) == len(lists1[bh])
            Kc, Vc = R.cache_rows_kv(layer, bh)
            assert np.array_equal(Kc.float().numpy(), k[b, lists1[bh], kh])
            assert np.array_equal(Vc.float().numpy(), v[b, lists1[bh], kh])
            idx = np.arange(len(lists1[bh]))
            moved_u = upool1[table1[bh, idx // S.PAGE_ROWS], idx % S.PAGE_ROWS]
            before = dict(zip(lists0[bh].tolist(), upool[table0[bh, np.arange(len(lists0[bh])) // S.PAGE_ROWS],
                                                           np.arange(len(lists0[bh])) % S.PAGE_ROWS].tolist()))
            assert all(before[int(s)] == float(x) for s, x in zip(lists1[bh], moved_u))
    z_win = layer.ring.z_win.cpu().numpy()
    with np.errstate(invalid="ignore"):
        assert np.array_equal(z_win, (u_win >= np.float32(tau2)).astype(np.uint8))

    # per-token decode at tau'
    layer.p = _params(wl, tau2)
    z2 = O.gate(u_ref, tau2)
    for i in range(steps):
        t = T0 + i
        t_pos = torch.full((wl.B,), t, dtype=torch.int32, device="cuda")
        o, _, _ = R.decode_step(layer, t_pos, C.dev(h[:, t], wl.dtype), C.dev(q[:, t], wl.dtype),
                                C.dev(k[:, t], wl.dtype), C.dev(v[:, t], wl.dtype))
        if i % 7 == 0 or i == steps - 1:
            o = C.to_np(o)
            for b in range(wl.B):
                o_ref, _ = O.gated_attention(q[b, t:t + 1], k[b, :t + 1], v[b, :t + 1],
                                             z2[b, :t + 1], w, [t])
                C.check_attn(o[b], o_ref[0], wl.dtype, f"{name} step {i} b={b}")
    status, flags = S.spkv_cache_check(layer.cache)
    assert status == S.OK, flags
    lists2 = R.cache_lists(layer)
    table2 = layer.cache.page_table.cpu().numpy()
    for b in range(wl.B):
        for kh in range(wl.Hkv):
            bh = b * wl.Hkv + kh
            _check_list_two(lists2[bh], O.cache_rows(z2[b, :, kh], T - w), u_ref[b, :, kh],
                            (wl.tau, tau2))
            owned = int((table0[bh] >= 0).sum())
            assert np.array_equal(table2[bh, :owned], table0[bh, :owned])  # owned pages reused


def test_rethreshold_below_gate_threshold_keeps_everything():
    """tau' below the threshold the rows were gated with removes nothing (the dropped
    rows are not recovered)."""
    wl, _ = CASES["bf16_g4"]
    T0 = 1000
    W1, b1, W2, b2 = C.weights(wl)
    p = _params(wl, wl.tau)
    mp = R.pages_for(T0)
    layer = R.Layer.create(p, C.dev(W1, wl.dtype), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                           num_pages=wl.B * wl.Hkv * mp, max_pages_per_head=mp, store_u=True)
    h, q, k, v = _rows(wl, T0)
    R.prefill_chunk(layer, C.dev(h, wl.dtype), C.dev(q, wl.dtype), C.dev(k, wl.dtype),
                    C.dev(v, wl.dtype), 0)
    before = R.cache_lists(layer)
    K0 = [R.cache_rows_kv(layer, bh) for bh in range(wl.B * wl.Hkv)]
    ws = S.alloc_rethreshold_workspace(p, layer.cache)
    S.spkv_cache_rethreshold(p, layer.cache, layer.ring, 0.1, ws)
    assert S.spkv_cache_check(layer.cache)[0] == S.OK
    after = R.cache_lists(layer)
    for bh in range(wl.B * wl.Hkv):
        assert np.array_equal(before[bh], after[bh])
        K1, V1 = R.cache_rows_kv(layer, bh)
        assert torch.equal(K0[bh][0], K1) and torch.equal(K0[bh][1], V1)
    # and tau' > 1 empties every head
    S.spkv_cache_rethreshold(p, layer.cache, None, 1.5, ws)
    assert S.spkv_cache_check(layer.cache)[0] == S.OK
    assert int(layer.cache.count.sum().item()) == 0
