"""CUDA path vs the oracle, element by element, at sizes the oracle finishes in
seconds that still span several tiles and a ragged tail (GPU required)."""
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


def _params(wl):
    return S.make_params(wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau,
                         S.BF16 if wl.dtype == "bf16" else S.F32)


def _layer(wl, rows_per_head, layer=0):
    W1, b1, W2, b2 = C.weights(wl, layer)
    p = _params(wl)
    mp = R.pages_for(rows_per_head)
    return R.Layer.create(p, C.dev(W1, wl.dtype), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                          num_pages=wl.B * wl.Hkv * mp, max_pages_per_head=mp), (W1, b1, W2, b2)


def _rows(wl, T, layer=0):
    """Host h, q, k, v [B][T][...] for positions 0..T-1."""
    hs, qs, ks, vs = [], [], [], []
    for b in range(wl.B):
        h, q, k, v = C.host_rows(wl, layer, b, np.arange(T))
        hs.append(h); qs.append(q); ks.append(k); vs.append(v)
    return np.stack(hs), np.stack(qs), np.stack(ks), np.stack(vs)


SCORE_CASES = {
    "tiny_f32_528": (W.small_case("tiny", ctx=[528], decode_steps=0), 528),
    "llama_bf16_300": (W.small_case("decode32k", B=1, ctx=[300], decode_steps=0, layers=1), 300),
    "llama_bf16_1": (W.small_case("decode32k", B=1, ctx=[1], decode_steps=0, layers=1), 1),
    "llama_bf16_33": (W.small_case("decode32k", B=1, ctx=[33], decode_steps=0, layers=1), 33),
    # 65..127 tokens: the CUDA-core tile kernel (less than one 128-token tile)
    "llama_bf16_100": (W.small_case("decode32k", B=1, ctx=[100], decode_steps=0, layers=1), 100),
    # 128 tokens or more, bf16, hid 128: the tcgen05 score (128-token tiles, d_model split
    # over a cluster of 4); a whole 4096-token chunk, a ragged count, and d_model 256 (one
    # K block per rank) with 16 key heads
    "llama_bf16_4096": (W.small_case("decode32k", B=1, ctx=[4096], decode_steps=0, layers=1), 4096),
    "llama_bf16_1000": (W.small_case("decode32k", B=1, ctx=[1000], decode_steps=0, layers=1), 1000),
    "bf16_dm256_hkv16_200": (W.small_case("decode32k", cid=64, B=1, Hq=16, Hkv=16, d_model=256,
                                          hid=128, ctx=[200], decode_steps=0, layers=1), 200),
}


@pytest.mark.parametrize("name", sorted(SCORE_CASES))
def test_score_matches_oracle(name):
    wl, n = SCORE_CASES[name]
    layer, (W1, b1, W2, b2) = _layer(wl, 64)
    h = wl.h_rows(0, 0, np.arange(n))
    u, z = R.score(layer, C.dev(h, wl.dtype), n)
    u_ref, z_ref = C.oracle_gates(h, W1, b1, W2, b2, wl.tau)
    C.check_gates(C.to_np(u), z.cpu().numpy(), u_ref, z_ref, wl.tau)


def test_score_empty_is_noop():
    wl, _ = SCORE_CASES["tiny_f32_528"]
    layer, _ = _layer(wl, 64)
    z = torch.full((4, wl.Hkv), 7, dtype=torch.uint8, device="cuda")
    S.spkv_score(layer.p, C.dev(np.zeros((1, wl.d_model)), wl.dtype), 0, layer.W1, layer.b1,
                 layer.W2, layer.b2, None, z)
    assert int(z.min()) == 7


def _lists_equal(layer, z_ref, upto, positions_offset=0):
    lists = R.cache_lists(layer)
    B, _, Hkv = z_ref.shape
    for b in range(B):
        for kh in range(Hkv):
            want = O.cache_rows(z_ref[b, :, kh], upto) + positions_offset
            got = lists[b * Hkv + kh]
            assert np.array_equal(got, want), f"cache list of head ({b},{kh}) differs"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_compact_chunks_and_ring(dtype):
    """Chunk compaction over several calls (ragged sizes), then ring compaction:
    index lists and stored rows are exact."""
    wl = W.small_case("decode32k", cid=40, B=2, Hq=8, Hkv=2, d_model=128, hid=64, dtype=dtype,
                      ctx=[3000], decode_steps=0, layers=1, keep="fixed25")
    T = 2500
    layer, (W1, b1, W2, b2) = _layer(wl, T)
    h, q, k, v = _rows(wl, T)
    _, z_ref = C.oracle_gates(h.reshape(-1, wl.d_model), W1, b1, W2, b2, wl.tau)
    z_ref = z_ref.reshape(wl.B, T, wl.Hkv)
    zd = torch.from_numpy(z_ref).cuda()
    kd, vd = C.dev(k, dtype), C.dev(v, dtype)
    # chunks [0,1000), [1000,1777), [1777,2372) from the chunk tensors
    for c0, c1 in [(0, 1000), (1000, 1777), (1777, 2372)]:
        src_pos = torch.full((wl.B,), c0, dtype=torch.int32, device="cuda")
        S.spkv_write_compact(layer.p, layer.cache, layer.ring, S.SRC_CHUNK,
                             kd[:, c0:].contiguous(), vd[:, c0:].contiguous(),
                             zd[:, c0:].contiguous(), None, src_pos, c1 - c0, T - c0)
    # the last 128 rows through the ring
    w = wl.window
    src_pos = torch.full((wl.B,), 2372, dtype=torch.int32, device="cuda")
    S.spkv_ring_write(layer.p, layer.ring, kd[:, 2372:].contiguous(), vd[:, 2372:].contiguous(),
                      zd[:, 2372:].contiguous(), None, 0, src_pos, T - 2372, T - 2372)
    S.spkv_write_compact(layer.p, layer.cache, layer.ring, S.SRC_RING, None, None,
                         zd[:, 2372:].contiguous(), None, src_pos, T - 2372, T - 2372)
    assert T - 2372 == w
    status, flags = S.spkv_cache_check(layer.cache)
    assert status == S.OK and flags == 0
    _lists_equal(layer, z_ref, T)
    for b in range(wl.B):
        for kh in range(wl.Hkv):
            rows = O.cache_rows(z_ref[b, :, kh], T)
            K, V = R.cache_rows_kv(layer, b * wl.Hkv + kh)
            assert np.array_equal(K.float().numpy(), k[b, rows, kh])
            assert np.array_equal(V.float().numpy(), v[b, rows, kh])


def test_compact_capacity_is_flagged():
    wl = W.small_case("decode32k", cid=41, B=1, Hq=4, Hkv=1, d_model=128, hid=32, dtype="bf16",
                      ctx=[1000], decode_steps=0, layers=1, keep="fixed25")
    W1, b1, W2, b2 = C.weights(wl)
    p = _params(wl)
    layer = R.Layer.create(p, C.dev(W1, "bf16"), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                           num_pages=2, max_pages_per_head=8)
    z = torch.ones((1, 1000, 1), dtype=torch.uint8, device="cuda")
    kv = torch.randn((1, 1000, 1, 128), device="cuda").to(torch.bfloat16)
    S.spkv_write_compact(p, layer.cache, layer.ring, S.SRC_CHUNK, kv, kv, z, None,
                         torch.zeros(1, dtype=torch.int32, device="cuda"), 1000, 1000)
    status, flags = S.spkv_cache_check(layer.cache)
    assert status == S.ERR_CAPACITY and flags & S.FLAG_POOL_FULL
    assert int(layer.cache.count[0]) == 2 * S.PAGE_ROWS
    assert np.array_equal(R.cache_lists(layer)[0], np.arange(128))


PREFILL_CASES = {
    # name: (workload, T, chunk)
    "tiny_f32_one_chunk": (W.small_case("tiny", ctx=[512], decode_steps=0), 512, 512),
    "bf16_g4_chunks": (W.small_case("decode32k", cid=42, B=2, Hq=8, Hkv=2, d_model=256, hid=64,
                                    ctx=[1000], decode_steps=0, layers=1, keep="fixed20"), 1000, 256),
    "bf16_g1_d64": (W.small_case("decode32k", cid=43, B=1, Hq=2, Hkv=2, head_dim=64, d_model=128,
                                 hid=32, ctx=[700], decode_steps=0, layers=1, keep="fixed25"), 700, 300),
    "f32_g8_d128": (W.small_case("tiny", cid=44, B=1, Hq=8, Hkv=1, head_dim=128, ctx=[400],
                                 decode_steps=0), 400, 160),
    # tensor-core path (bf16, head_dim 128, window 128, chunks of multiples of 128)
    "tc_g2_two_chunks": (W.small_case("decode32k", cid=52, B=2, Hq=4, Hkv=2, d_model=128, hid=32,
                                      ctx=[1024], decode_steps=0, layers=1, keep="fixed25"), 1024, 512),
    "tc_g8_three_chunks": (W.small_case("decode32k", cid=53, B=1, Hq=16, Hkv=2, d_model=128,
                                        hid=32, ctx=[1152], decode_steps=0, layers=1,
                                        keep="u05_50"), 1152, 384),
    "tc_g4_dense_pages": (W.small_case("decode32k", cid=54, B=1, Hq=8, Hkv=2, d_model=128, hid=32,
                                       ctx=[1536], decode_steps=0, layers=1, keep="spread"), 1536, 768),
    # more 128-query tiles (8 x 2 head pairs x 16 key heads = 256 per chunk) than SMs: the
    # persistent CTAs take several tiles each, from the tile counter
    "tc_g4_many_tiles": (W.small_case("decode32k", cid=55, B=4, Hq=16, Hkv=4, d_model=128, hid=32,
                                      ctx=[2048], decode_steps=0, layers=1, keep="u05_50"), 2048, 1024),
}


@pytest.mark.parametrize("name", sorted(PREFILL_CASES))
def test_chunked_prefill_matches_oracle(name):
    wl, T, chunk = PREFILL_CASES[name]
    layer, (W1, b1, W2, b2) = _layer(wl, T)
    h, q, k, v = _rows(wl, T)
    u_ref, z_ref = C.oracle_gates(h.reshape(-1, wl.d_model), W1, b1, W2, b2, wl.tau)
    z_ref = z_ref.reshape(wl.B, T, wl.Hkv)
    u_ref = u_ref.reshape(wl.B, T, wl.Hkv)
    outs, zs, us = [], [], []
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        o, lse, u, z = R.prefill_chunk(layer, C.dev(h[:, c0:c1], wl.dtype),
                                       C.dev(q[:, c0:c1], wl.dtype), C.dev(k[:, c0:c1], wl.dtype),
                                       C.dev(v[:, c0:c1], wl.dtype), c0)
        outs.append(C.to_np(o)); zs.append(z.cpu().numpy()); us.append(C.to_np(u))
    o_gpu = np.concatenate(outs, axis=1)
    C.check_gates(np.concatenate(us, 1), np.concatenate(zs, 1), u_ref, z_ref, wl.tau)
    for b in range(wl.B):
        o_ref, _ = O.gated_attention(q[b], k[b], v[b], z_ref[b], wl.window, np.arange(T))
        C.check_attn(o_gpu[b], o_ref, wl.dtype, f"{name} b={b}")
    _lists_equal(layer, z_ref, T)


def test_prefill_tile_order_leaves_results_unchanged():
    """Tiles handed out by the counter (workspace given) or in the fixed order (no
    workspace): each tile's arithmetic is the same, so the outputs agree bit for bit;
    the counter is back at zero after every call."""
    wl, T, chunk = PREFILL_CASES["tc_g4_many_tiles"]
    outs = {}
    for mode in ("counter", "fixed"):
        layer, _ = _layer(wl, T)
        if mode == "fixed":
            layer.pf_ws = None
        h, q, k, v = _rows(wl, T)
        res = []
        for c0 in range(0, T, chunk):
            o, lse, _, _ = R.prefill_chunk(layer, C.dev(h[:, c0:c0 + chunk], wl.dtype),
                                           C.dev(q[:, c0:c0 + chunk], wl.dtype),
                                           C.dev(k[:, c0:c0 + chunk], wl.dtype),
                                           C.dev(v[:, c0:c0 + chunk], wl.dtype), c0)
            res.append((o.clone(), lse.clone()))
            if layer.pf_ws is not None:
                assert int(layer.pf_ws.count_nonzero()) == 0
        outs[mode] = res
    for (o1, l1), (o2, l2) in zip(outs["counter"], outs["fixed"]):
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _decode_run(wl, T0, steps, layer_rows, retire=True, bulk=0, fused=True):
    """Prefill T0 tokens (per-token-ready state when retire) then decode `steps`
    tokens; returns gpu outputs [steps][B][Hq][d], z per step and the layer."""
    layer, (W1, b1, W2, b2) = _layer(wl, layer_rows)
    T = T0 + steps
    h, q, k, v = _rows(wl, T)
    w = wl.window
    chunk = 512
    for c0 in range(0, T0, chunk):
        c1 = min(T0, c0 + chunk)
        n_compact = max(0, min(c1, T0 - w) - c0) if retire else c1 - c0
        R.prefill_chunk(layer, C.dev(h[:, c0:c1], wl.dtype), C.dev(q[:, c0:c1], wl.dtype),
                        C.dev(k[:, c0:c1], wl.dtype), C.dev(v[:, c0:c1], wl.dtype), c0,
                        n_compact=n_compact)
    outs, zs = [], []
    for i in range(steps):
        t = T0 + i
        t_pos = torch.full((wl.B,), t, dtype=torch.int32, device="cuda")
        o, lse, z = R.decode_step(layer, t_pos, C.dev(h[:, t], wl.dtype), C.dev(q[:, t], wl.dtype),
                                  C.dev(k[:, t], wl.dtype), C.dev(v[:, t], wl.dtype), retire=retire,
                                  fused=fused)
        outs.append(C.to_np(o))
        zs.append(None if z is None else z.cpu().numpy())
        if bulk and (i + 1) % bulk == 0:
            start = torch.full((wl.B,), t - bulk + 1, dtype=torch.int32, device="cuda")
            R.bulk_compact(layer, C.dev(h[:, t - bulk + 1:t + 1], wl.dtype), start)
    return layer, outs, zs, (h, q, k, v), (W1, b1, W2, b2)


DECODE_CASES = {
    "tiny_f32_c0": W.small_case("tiny"),
    "bf16_g4": W.small_case("decode32k", cid=45, B=3, Hq=8, Hkv=2, d_model=256, hid=64,
                            ctx=[2000], decode_steps=8, layers=1, keep="u05_50"),
    "bf16_g8_d64": W.small_case("decode32k", cid=46, B=2, Hq=8, Hkv=1, head_dim=64, d_model=128,
                                hid=32, ctx=[900], decode_steps=6, layers=1, keep="fixed25"),
    "bf16_g2": W.small_case("decode32k", cid=47, B=2, Hq=4, Hkv=2, d_model=128, hid=32,
                            ctx=[1500], decode_steps=6, layers=1, keep="fixed25"),
    "f32_g1_d128": W.small_case("tiny", cid=48, B=2, Hq=2, Hkv=2, head_dim=128, ctx=[700],
                                decode_steps=5),
    "bf16_short_ctx": W.small_case("decode32k", cid=49, B=2, Hq=8, Hkv=2, d_model=128, hid=32,
                                   ctx=[40], decode_steps=100, layers=1, keep="fixed25"),
}


@pytest.mark.parametrize("name", sorted(DECODE_CASES))
def test_per_token_decode_matches_oracle(name):
    wl = DECODE_CASES[name]
    T0, steps = wl.ctx[0], wl.decode_steps
    T = T0 + steps
    layer, outs, zs, (h, q, k, v), (W1, b1, W2, b2) = _decode_run(wl, T0, steps, T)
    u_ref, z_ref = C.oracle_gates(h.reshape(-1, wl.d_model), W1, b1, W2, b2, wl.tau)
    z_ref = z_ref.reshape(wl.B, T, wl.Hkv)
    u_ref = u_ref.reshape(wl.B, T, wl.Hkv)
    for i in range(steps):
        t = T0 + i
        near = np.abs(u_ref[:, t] - wl.tau) < C.EXCLUDE
        assert np.all((zs[i] == z_ref[:, t]) | near), f"gate of token {t}"
        for b in range(wl.B):
            o_ref, _ = O.gated_attention(q[b, t:t + 1], k[b, :t + 1], v[b, :t + 1],
                                         z_ref[b, :t + 1], wl.window, [t])
            C.check_attn(outs[i][b], o_ref[0], wl.dtype, f"{name} step {i} b={b}")
    # cache holds exactly the gated tokens that have left the window of the last query
    _lists_equal(layer, z_ref, max(0, T - wl.window))


def test_buffered_decode_matches_oracle():
    """Buffered schedule: tokens enter the ring ungated; every 128 steps the buffer
    is scored and compacted from the ring.  Same outputs as Eq. (3)-(4)."""
    wl = W.small_case("decode32k", cid=50, B=2, Hq=8, Hkv=2, d_model=128, hid=32, ctx=[1000],
                      decode_steps=256, layers=1, keep="fixed25")
    T0, steps = 1000, 256
    T = T0 + steps
    layer, outs, _, (h, q, k, v), (W1, b1, W2, b2) = _decode_run(wl, T0, steps, T, retire=False,
                                                                 bulk=128)
    _, z_ref = C.oracle_gates(h.reshape(-1, wl.d_model), W1, b1, W2, b2, wl.tau)
    z_ref = z_ref.reshape(wl.B, T, wl.Hkv)
    for i in list(range(0, steps, 17)) + [127, 128, 255]:
        t = T0 + i
        for b in range(wl.B):
            o_ref, _ = O.gated_attention(q[b, t:t + 1], k[b, :t + 1], v[b, :t + 1],
                                         z_ref[b, :t + 1], wl.window, [t])
            C.check_attn(outs[i][b], o_ref[0], wl.dtype, f"bulk step {i} b={b}")
    _lists_equal(layer, z_ref, T)


def test_schedules_agree():
    """Per-token and buffered schedules give the same decode outputs (the key set
    of Eq. (4) does not depend on when a token was compacted)."""
    wl = W.small_case("decode32k", cid=51, B=2, Hq=8, Hkv=2, d_model=128, hid=32, ctx=[700],
                      decode_steps=128, layers=1, keep="fixed25")
    _, a, _, _, _ = _decode_run(wl, 700, 128, 900, retire=True)
    _, b, _, _, _ = _decode_run(wl, 700, 128, 900, retire=False, bulk=128)
    for i in range(128):
        C.check_attn(a[i], b[i], "bf16", f"step {i}")


def test_fused_and_separate_decode_steps_agree():
    """spkv_decode_score_append (one launch) against spkv_score + spkv_decode_append:
    identical gates, cache lists and outputs."""
    wl = W.small_case("decode32k", cid=55, B=3, Hq=8, Hkv=2, d_model=256, hid=64, ctx=[600],
                      decode_steps=150, layers=1, keep="u05_50")
    la, a, za, _, _ = _decode_run(wl, 600, 150, 800, fused=True)
    lb, b, zb, _, _ = _decode_run(wl, 600, 150, 800, fused=False)
    for i in range(150):
        assert np.array_equal(za[i], zb[i])
        assert np.array_equal(a[i], b[i]), f"step {i}"
    for x, y in zip(R.cache_lists(la), R.cache_lists(lb)):
        assert np.array_equal(x, y)


def test_fused_step_with_settled_inputs_is_unchanged():
    """SPKV_INPUTS_SETTLED on the fused score + update (the tensor-core perceptron runs
    before the wait for the preceding kernel; only the ring and cache wait) leaves the
    step's gates, utilities, outputs and cache bit for bit as they are without it.  The
    hidden states are copied in before each step, so they are settled."""
    wl = W.small_case("decode32k", cid=58, B=4, ctx=[1100], decode_steps=24, layers=1,
                      keep="fixed25")
    T0, steps, w = wl.ctx[0], wl.decode_steps, wl.window
    T = T0 + steps
    W1, b1, W2, b2 = C.weights(wl)
    p = _params(wl)
    mp = R.pages_for(T)
    layers = [R.Layer.create(p, C.dev(W1, wl.dtype), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                             num_pages=wl.B * wl.Hkv * mp, max_pages_per_head=mp, store_u=True)
              for _ in range(2)]
    h, q, k, v = _rows(wl, T)
    for L in layers:
        for c0 in range(0, T0, 512):
            c1 = min(T0, c0 + 512)
            R.prefill_chunk(L, C.dev(h[:, c0:c1], wl.dtype), C.dev(q[:, c0:c1], wl.dtype),
                            C.dev(k[:, c0:c1], wl.dtype), C.dev(v[:, c0:c1], wl.dtype), c0,
                            n_compact=max(0, min(c1, T0 - w) - c0))
    for i in range(steps):
        t = T0 + i
        t_pos = torch.full((wl.B,), t, dtype=torch.int32, device="cuda")
        res = []
        for L, flags in zip(layers, (0, S.INPUTS_SETTLED)):
            o, lse, z = R.decode_step(L, t_pos, C.dev(h[:, t], wl.dtype), C.dev(q[:, t], wl.dtype),
                                      C.dev(k[:, t], wl.dtype), C.dev(v[:, t], wl.dtype),
                                      score_flags=flags)
            res.append((o.clone(), lse.clone(), z.clone()))
        (oa, la, za), (ob, lb, zb) = res
        assert torch.equal(za, zb) and torch.equal(oa, ob) and torch.equal(la, lb), f"step {i}"
    torch.cuda.synchronize()
    for L in layers:
        assert S.spkv_cache_check(L.cache)[0] == S.OK
    for x, y in zip(R.cache_lists(layers[0]), R.cache_lists(layers[1])):
        assert np.array_equal(x, y)
    for bh in range(wl.B * wl.Hkv):  # the stored rows, in list order
        (ka, va), (kb, vb) = (R.cache_rows_kv(L, bh) for L in layers)
        assert torch.equal(ka, kb) and torch.equal(va, vb), f"head {bh}"


SPLIT_CASES = {
    # d_model 4096, hid 128: tensor-core score, gates stored by the score kernel
    "mma": W.small_case("decode32k", cid=55, B=4, ctx=[1100], decode_steps=140, layers=1,
                        keep="fixed25"),
    # few-token CUDA-core score
    "small": W.small_case("decode32k", cid=56, B=3, Hq=8, Hkv=2, d_model=256, hid=64, ctx=[900],
                          decode_steps=135, layers=1, keep="u05_50"),
    # batch above the few-token kernels: spkv_score, then the gates stored by a second kernel
    "batch20": W.small_case("decode32k", cid=57, B=20, Hq=4, Hkv=2, d_model=128, hid=32,
                            ctx=[700], decode_steps=130, layers=1, keep="fixed25"),
}


@pytest.mark.parametrize("name", sorted(SPLIT_CASES))
def test_split_decode_step_matches_fused(name):
    """The decode step with the scoring on a second stream (the retirement and ring
    write with the new gate at 0, the attention, then spkv_decode_score storing the new
    gates in the window) gives the fused step's outputs, gates, utilities and cache bit
    for bit, and the oracle's outputs; retirements after w steps use the stored gates."""
    wl = SPLIT_CASES[name]
    T0, steps, w = wl.ctx[0], wl.decode_steps, wl.window
    T = T0 + steps
    W1, b1, W2, b2 = C.weights(wl)
    p = _params(wl)
    mp = R.pages_for(T)
    layers = [R.Layer.create(p, C.dev(W1, wl.dtype), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                             num_pages=wl.B * wl.Hkv * mp, max_pages_per_head=mp, store_u=True)
              for _ in range(2)]
    h, q, k, v = _rows(wl, T)
    for L in layers:
        for c0 in range(0, T0, 512):
            c1 = min(T0, c0 + 512)
            R.prefill_chunk(L, C.dev(h[:, c0:c1], wl.dtype), C.dev(q[:, c0:c1], wl.dtype),
                            C.dev(k[:, c0:c1], wl.dtype), C.dev(v[:, c0:c1], wl.dtype), c0,
                            n_compact=max(0, min(c1, T0 - w) - c0))
    side = torch.cuda.Stream()
    _, z_ref = C.oracle_gates(h.reshape(-1, wl.d_model), W1, b1, W2, b2, wl.tau)
    z_ref = z_ref.reshape(wl.B, T, wl.Hkv)
    for i in range(steps):
        t = T0 + i
        t_pos = torch.full((wl.B,), t, dtype=torch.int32, device="cuda")
        args = (C.dev(h[:, t], wl.dtype), C.dev(q[:, t], wl.dtype), C.dev(k[:, t], wl.dtype),
                C.dev(v[:, t], wl.dtype))
        o_a, _, z_a = R.decode_step(layers[0], t_pos, *args)
        o_b, _, z_b = R.decode_step(layers[1], t_pos, *args, score_stream=side)
        torch.cuda.current_stream().wait_stream(side)
        assert torch.equal(o_a, o_b), f"step {i}: outputs differ"
        assert torch.equal(z_a, z_b), f"step {i}: gates differ"
        if i % 29 == 0 or i == steps - 1:
            og = C.to_np(o_b)
            for b in range(wl.B):
                o_ref, _ = O.gated_attention(q[b, t:t + 1], k[b, :t + 1], v[b, :t + 1],
                                             z_ref[b, :t + 1], w, [t])
                C.check_attn(og[b], o_ref[0], wl.dtype, f"split {name} step {i} b={b}")
    torch.cuda.synchronize()
    for x, y in ((layers[0].ring.z_win, layers[1].ring.z_win),
                 (layers[0].ring.u_win, layers[1].ring.u_win),
                 (layers[0].cache.count, layers[1].cache.count)):
        assert torch.equal(x, y)
    la, lb = R.cache_lists(layers[0]), R.cache_lists(layers[1])
    for bh in range(wl.B * wl.Hkv):
        assert np.array_equal(la[bh], lb[bh])
    for L in layers:
        assert S.spkv_cache_check(L.cache)[0] == S.OK


ATTN_FIRST_CASES = dict(SPLIT_CASES)
# from an empty state: t = 0 (no key but the new token), t < w, the first retirement at t = w
ATTN_FIRST_CASES["from_empty"] = W.small_case("decode32k", cid=59, B=2, Hq=8, Hkv=2, d_model=128,
                                              hid=32, ctx=[0], decode_steps=150, layers=1,
                                              keep="u05_50")
# head_dim 64, 8 query heads per key head
ATTN_FIRST_CASES["d64_g8"] = W.small_case("decode32k", cid=63, B=2, Hq=8, Hkv=1, head_dim=64,
                                          d_model=128, hid=32, ctx=[300], decode_steps=140,
                                          layers=1, keep="fixed25")


@pytest.mark.parametrize("name", sorted(ATTN_FIRST_CASES))
def test_attention_first_decode_step(name):
    """The decode step with the attention first (spkv_decode_attn_before_append on the
    state before the step's retirement and ring write, the new rows passed in; the
    update and the scoring after it on a second stream): outputs against the oracle at
    every step, and gates, utilities, ring and cache bit for bit equal to the fused
    step's (the update kernels are the same, only their order changes)."""
    wl = ATTN_FIRST_CASES[name]
    T0, steps, w = wl.ctx[0], wl.decode_steps, wl.window
    T = T0 + steps
    W1, b1, W2, b2 = C.weights(wl)
    p = _params(wl)
    assert S.spkv_decode_attn_before_append_supported(p)
    mp = R.pages_for(T)
    layers = [R.Layer.create(p, C.dev(W1, wl.dtype), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                             num_pages=wl.B * wl.Hkv * mp, max_pages_per_head=mp, store_u=True)
              for _ in range(2)]
    h, q, k, v = _rows(wl, T)
    for L in layers:
        for c0 in range(0, T0, 512):
            c1 = min(T0, c0 + 512)
            R.prefill_chunk(L, C.dev(h[:, c0:c1], wl.dtype), C.dev(q[:, c0:c1], wl.dtype),
                            C.dev(k[:, c0:c1], wl.dtype), C.dev(v[:, c0:c1], wl.dtype), c0,
                            n_compact=max(0, min(c1, T0 - w) - c0))
    side = torch.cuda.Stream()
    _, z_ref = C.oracle_gates(h.reshape(-1, wl.d_model), W1, b1, W2, b2, wl.tau)
    z_ref = z_ref.reshape(wl.B, T, wl.Hkv)
    for i in range(steps):
        t = T0 + i
        t_pos = torch.full((wl.B,), t, dtype=torch.int32, device="cuda")
        args = (C.dev(h[:, t], wl.dtype), C.dev(q[:, t], wl.dtype), C.dev(k[:, t], wl.dtype),
                C.dev(v[:, t], wl.dtype))
        o_a, _, z_a = R.decode_step(layers[0], t_pos, *args)
        o_b, lse_b, z_b = R.decode_step(layers[1], t_pos, *args, score_stream=side,
                                        attn_first=True)
        torch.cuda.current_stream().wait_stream(side)
        assert torch.equal(z_a, z_b), f"step {i}: gates differ"
        og = C.to_np(o_b)
        assert np.all(np.isfinite(og)) and np.all(np.isfinite(lse_b.cpu().numpy()))
        for b in range(wl.B):
            o_ref, _ = O.gated_attention(q[b, t:t + 1], k[b, :t + 1], v[b, :t + 1],
                                         z_ref[b, :t + 1], w, [t])
            C.check_attn(og[b], o_ref[0], wl.dtype, f"attn-first {name} step {i} b={b}")
    torch.cuda.synchronize()
    for x, y in ((layers[0].ring.z_win, layers[1].ring.z_win),
                 (layers[0].ring.u_win, layers[1].ring.u_win),
                 (layers[0].ring.K_win, layers[1].ring.K_win),
                 (layers[0].ring.V_win, layers[1].ring.V_win),
                 (layers[0].cache.count, layers[1].cache.count)):
        assert torch.equal(x.nan_to_num() if x.is_floating_point() else x,
                           y.nan_to_num() if y.is_floating_point() else y)
    la, lb = R.cache_lists(layers[0]), R.cache_lists(layers[1])
    for bh in range(wl.B * wl.Hkv):
        assert np.array_equal(la[bh], lb[bh])
    for L in layers:
        assert S.spkv_cache_check(L.cache)[0] == S.OK


def test_cache_row_order_does_not_change_decode():
    """Permutation invariance (the split-K chunking and the merge): every head's cache
    rows shuffled in place (K, V and positions moved together, pages unchanged) give
    the same decode output up to rounding, and both orders match the oracle.  The
    attention runs before the step's update (it leaves the state untouched), so it can
    be called on the same state twice."""
    wl = W.small_case("decode32k", cid=65, B=2, Hq=8, Hkv=2, d_model=256, hid=64, ctx=[3000],
                      decode_steps=1, layers=1, keep="u05_50")
    T0, w = wl.ctx[0], wl.window
    T = T0 + 1
    W1, b1, W2, b2 = C.weights(wl)
    p = _params(wl)
    mp = R.pages_for(T)
    L = R.Layer.create(p, C.dev(W1, wl.dtype), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                       num_pages=wl.B * wl.Hkv * mp, max_pages_per_head=mp)
    h, q, k, v = _rows(wl, T)
    for c0 in range(0, T0, 512):
        c1 = min(T0, c0 + 512)
        R.prefill_chunk(L, C.dev(h[:, c0:c1], wl.dtype), C.dev(q[:, c0:c1], wl.dtype),
                        C.dev(k[:, c0:c1], wl.dtype), C.dev(v[:, c0:c1], wl.dtype), c0,
                        n_compact=max(0, min(c1, T0 - w) - c0))
    t_pos = torch.full((wl.B,), T0, dtype=torch.int32, device="cuda")
    args = (C.dev(q[:, T0], wl.dtype), t_pos, C.dev(k[:, T0], wl.dtype), C.dev(v[:, T0], wl.dtype))

    def attend():
        o = torch.empty_like(args[0])
        lse = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
        S.spkv_decode_attn_before_append(p, L.cache, L.ring, args[0], args[1], args[2], args[3], o,
                                         lse, L.ws)
        return C.to_np(o)

    o1 = attend()
    gen = torch.Generator().manual_seed(65)
    count = L.cache.count.cpu()
    moved = 0
    for bh in range(wl.B * wl.Hkv):
        n = int(count[bh])
        idx = torch.arange(n)
        pages = L.cache.page_table[bh].cpu()[idx // S.PAGE_ROWS].long().cuda()
        rows = (idx % S.PAGE_ROWS).cuda()
        perm = torch.randperm(n, generator=gen).cuda()
        for pool in (L.cache.K_pool, L.cache.V_pool, L.cache.pos_pool):
            pool[pages, rows] = pool[pages, rows][perm]
        moved += n
    assert moved > 1000
    o2 = attend()
    assert np.max(np.abs(o1 - o2)) <= 2e-2
    _, z_ref = C.oracle_gates(h.reshape(-1, wl.d_model), W1, b1, W2, b2, wl.tau)
    z_ref = z_ref.reshape(wl.B, T, wl.Hkv)
    for b in range(wl.B):
        o_ref, _ = O.gated_attention(q[b, T0:T], k[b, :T], v[b, :T], z_ref[b], w, [T0])
        C.check_attn(o1[b], o_ref[0], wl.dtype, f"cache in order, b={b}")
        C.check_attn(o2[b], o_ref[0], wl.dtype, f"cache rows shuffled, b={b}")


def test_attention_first_lse():
    """lse of the attention-first step against the oracle's log-sum-exp (natural log of
    the softmax denominator over the key set, scores scaled by 1/sqrt(d))."""
    wl = ATTN_FIRST_CASES["small"]
    T0, steps, w = wl.ctx[0], 3, wl.window
    T = T0 + steps
    W1, b1, W2, b2 = C.weights(wl)
    p = _params(wl)
    mp = R.pages_for(T)
    L = R.Layer.create(p, C.dev(W1, wl.dtype), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                       num_pages=wl.B * wl.Hkv * mp, max_pages_per_head=mp)
    h, q, k, v = _rows(wl, T)
    R.prefill_chunk(L, C.dev(h[:, :T0], wl.dtype), C.dev(q[:, :T0], wl.dtype),
                    C.dev(k[:, :T0], wl.dtype), C.dev(v[:, :T0], wl.dtype), 0, n_compact=T0 - w)
    _, z_ref = C.oracle_gates(h.reshape(-1, wl.d_model), W1, b1, W2, b2, wl.tau)
    z_ref = z_ref.reshape(wl.B, T, wl.Hkv)
    side = torch.cuda.Stream()
    for i in range(steps):
        t = T0 + i
        t_pos = torch.full((wl.B,), t, dtype=torch.int32, device="cuda")
        _, lse, _ = R.decode_step(L, t_pos, C.dev(h[:, t], wl.dtype), C.dev(q[:, t], wl.dtype),
                                  C.dev(k[:, t], wl.dtype), C.dev(v[:, t], wl.dtype),
                                  score_stream=side, attn_first=True)
        torch.cuda.current_stream().wait_stream(side)
        got = lse.cpu().numpy()
        for b in range(wl.B):
            _, lse_ref = O.gated_attention(q[b, t:t + 1], k[b, :t + 1], v[b, :t + 1],
                                           z_ref[b, :t + 1], w, [t])
            assert np.max(np.abs(got[b] - lse_ref[0])) <= 2e-2, (i, b)


def test_tau_zero_decode_is_causal_attention():
    """tau = 0 gates every token in (u >= 0 always): the cache holds every position that
    left the window and per-token decode equals plain causal attention over the whole
    context (torch SDPA in fp64 as the reference of that special case)."""
    wl = W.small_case("decode32k", cid=58, B=2, Hq=8, Hkv=2, d_model=128, hid=32, ctx=[700],
                      decode_steps=4, layers=1, keep="fixed25")
    T0, steps = wl.ctx[0], wl.decode_steps
    T = T0 + steps
    W1, b1, W2, b2 = C.weights(wl)
    p = S.make_params(wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, 0.0, S.BF16)
    mp = R.pages_for(T)
    layer = R.Layer.create(p, C.dev(W1, "bf16"), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                           num_pages=wl.B * wl.Hkv * mp, max_pages_per_head=mp)
    h, q, k, v = _rows(wl, T)
    R.prefill_chunk(layer, C.dev(h[:, :T0], "bf16"), C.dev(q[:, :T0], "bf16"),
                    C.dev(k[:, :T0], "bf16"), C.dev(v[:, :T0], "bf16"), 0,
                    n_compact=T0 - wl.window)
    G = wl.Hq // wl.Hkv
    for i in range(steps):
        t = T0 + i
        t_pos = torch.full((wl.B,), t, dtype=torch.int32, device="cuda")
        o, _, z = R.decode_step(layer, t_pos, C.dev(h[:, t], "bf16"), C.dev(q[:, t], "bf16"),
                                C.dev(k[:, t], "bf16"), C.dev(v[:, t], "bf16"))
        assert int(z.min()) == 1
        og = C.to_np(o)
        for b in range(wl.B):
            Kx = torch.from_numpy(k[b, :t + 1]).double().permute(1, 0, 2)   # [Hkv][t+1][d]
            Vx = torch.from_numpy(v[b, :t + 1]).double().permute(1, 0, 2)
            Qx = torch.from_numpy(q[b, t]).double().view(wl.Hkv, G, 1, wl.head_dim)
            ref = torch.nn.functional.scaled_dot_product_attention(
                Qx, Kx[:, None], Vx[:, None]).view(wl.Hq, wl.head_dim).numpy()
            C.check_attn(og[b], ref, "bf16", f"tau=0 step {i} b={b}")
    assert int(layer.cache.count.min().item()) == T - wl.window
