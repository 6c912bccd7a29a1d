"""CUDA path vs the oracle at the workloads' full sizes, in the launch configuration
the benchmark times, on sampled outputs the oracle computes one by one (GPU required).

* decode32k: one layer at 32768-token context, batch 8, one per-token decode step
  (the benchmark's per-layer launches);
* prefill16k: the whole 16384-token chunked prefill, sampled query positions;
* ragged128k: contexts {128K, 96K, 64K, 32K}, one decode step, sampled rows;
* serving: batch 32, contexts in [8K, 64K], 130 buffered decode steps with a bulk
  score + compaction after step 128, sampled rows and steps.
Gates outside the exclusion band, cache index lists and attention outputs are checked.
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
    from sparse_decode_attention_spkv_b200 import spkv as S
    from sparse_decode_attention_spkv_b200.states import DecodeStep, build_decode_state
    from sparse_decode_attention_spkv_b200.inputs import device as D
    from sparse_decode_attention_spkv_b200.inputs import gen


def _one_layer(name, **kw):
    return W.small_case(name, layers=1, **kw)


def _check_row(wl, L, b, t, o_gpu_b, z_new_b, nrows_retired):
    """Oracle for batch row b at query position t (token t already in the ring)."""
    W1, b1, W2, b2 = C.weights(wl)
    u, z = C.oracle_gates_rows(wl, 0, b, t + 1, W1, b1, W2, b2)
    if z_new_b is not None:
        near = np.abs(u[t] - wl.tau) < C.EXCLUDE
        assert np.all((z_new_b == z[t]) | near), "gate of the new token"
    lists = R.cache_lists(L)
    for kh in range(wl.Hkv):
        C.check_list(lists[b * wl.Hkv + kh], z[:, kh], nrows_retired, u[:, kh], wl.tau)
    K, V = C.kv_rows(wl, 0, b, t + 1)
    q = wl.q_rows(0, b, [t])
    o_ref, _ = O.gated_attention(q, K, V, z, wl.window, [t])
    C.check_attn(o_gpu_b, o_ref[0], "bf16", f"{wl.name} row {b}")


def _decode_one_step(wl, rows, order="fused"):
    """One decode step of a full-size state.  order "attn-first" is the bench's launch
    configuration for several layers: attention on the state before the step's update
    (settled-state flag), update and scoring on the second stream, the whole step
    captured in a CUDA graph and replayed; "attn-first-one-stream" (the single-layer
    configuration) follows the attention with the fused score and update on the same
    stream, also captured."""
    p, Ls, inp = build_decode_state(wl, 1, 2, torch.device("cuda"))
    step = DecodeStep(p, Ls, "cuda", split=order == "attn-first", attn_first=order != "fused",
                      inputs_settled=order == "attn-first-one-stream")  # inputs built ahead
    if order != "fused":
        L = Ls[0]  # one eager attention (read-only) sets the kernel attributes before capture
        S.spkv_decode_attn_before_append(p, L.cache, L.ring, inp["q"][0][0], inp["t"][0],
                                         inp["k"][0][0], inp["v"][0][0], step.o[0], step.lse[0],
                                         L.ws)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step.launch(inp["h"][0], inp["q"][0], inp["k"][0], inp["v"][0], inp["t"][0])
        g.replay()
    else:
        step.launch(inp["h"][0], inp["q"][0], inp["k"][0], inp["v"][0], inp["t"][0])
    torch.cuda.synchronize()
    status, flags = S.spkv_cache_check(Ls[0].cache)
    assert status == S.OK, flags
    o = step.o[0].float().cpu().numpy()
    z = step.z[0].cpu().numpy()
    t = inp["t"][0].cpu().numpy()
    for b in rows:
        _check_row(wl, Ls[0], b, int(t[b]), o[b], z[b], int(t[b]) - wl.window + 1)


def test_decode32k_one_layer_full_size():
    _decode_one_step(_one_layer("decode32k"), rows=[5])


def test_ragged128k_full_size():
    _decode_one_step(_one_layer("ragged128k"), rows=[3, 0])


def test_decode32k_attention_first_graph_full_size():
    _decode_one_step(_one_layer("decode32k"), rows=[2, 7], order="attn-first")


def test_ragged128k_attention_first_graph_full_size():
    _decode_one_step(_one_layer("ragged128k"), rows=[0, 2], order="attn-first")


def test_ragged128k_attention_first_one_stream_full_size():
    _decode_one_step(_one_layer("ragged128k"), rows=[1, 3], order="attn-first-one-stream")


def test_serving_buffered_full_size():
    wl = _one_layer("serving")
    steps = 130
    p, Ls, inp = build_decode_state(wl, 1, steps, torch.device("cuda"), compact_window=True)
    L = Ls[0]
    sample = {5: [], 127: [], 129: []}
    for i in range(steps):
        o, _, _ = R.decode_step(L, inp["t"][i], None, inp["q"][i][0], inp["k"][i][0],
                                inp["v"][i][0], retire=False)
        if i in sample:
            sample[i] = o.float().cpu().numpy()
        if i == 127:  # the 128-token buffer is full: score it and compact it from the ring
            start = inp["t"][0].clone()
            R.bulk_compact(L, inp["h_layer_row"][0][:, 0:128].contiguous(), start)
    torch.cuda.synchronize()
    status, flags = S.spkv_cache_check(L.cache)
    assert status == S.OK, flags
    t0 = inp["t"][0].cpu().numpy()
    W1, b1, W2, b2 = C.weights(wl)
    for b in (0, 17):
        T_end = int(t0[b]) + steps
        u, z = C.oracle_gates_rows(wl, 0, b, T_end, W1, b1, W2, b2)
        K, V = C.kv_rows(wl, 0, b, T_end)
        for i, o in sample.items():
            t = int(t0[b]) + i
            q = wl.q_rows(0, b, [t])
            o_ref, _ = O.gated_attention(q, K[:t + 1], V[:t + 1], z[:t + 1], wl.window, [t])
            C.check_attn(o[b], o_ref[0], "bf16", f"serving row {b} step {i}")
        lists = R.cache_lists(L)
        for kh in range(wl.Hkv):  # everything up to the end of the first buffer is cached
            C.check_list(lists[b * wl.Hkv + kh], z[:, kh], int(t0[b]) + 128, u[:, kh], wl.tau)


def test_prefill16k_full_size():
    wl = W.WORKLOADS["prefill16k"]
    T, chunk = wl.ctx[0], wl.chunk
    W1, b1, W2, b2 = C.weights(wl)
    p = S.make_params(1, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau, S.BF16)
    mp = R.pages_for(T)
    L = R.Layer.create(p, C.dev(W1, "bf16"), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                       num_pages=wl.Hkv * mp, max_pages_per_head=mp)
    Tt = wl.T_total
    outs = []
    for c0 in range(0, T, chunk):
        h = torch.empty((1, chunk, wl.d_model), dtype=torch.bfloat16, device="cuda")
        q = torch.empty((1, chunk, wl.Hq, wl.head_dim), dtype=torch.bfloat16, device="cuda")
        k = torch.empty((1, chunk, wl.Hkv, wl.head_dim), dtype=torch.bfloat16, device="cuda")
        v = torch.empty_like(k)
        D.fill_normal(h, wl.key(0, gen.T_H), 1.0, offset=c0 * wl.d_model)
        D.fill_rope(q, wl.key(0, gen.T_Q), c0, Tt, wl.qkv_scale, wl.rope_base)
        D.fill_rope(k, wl.key(0, gen.T_K), c0, Tt, wl.qkv_scale, wl.rope_base)
        D.fill_normal(v, wl.key(0, gen.T_V), wl.qkv_scale, offset=c0 * wl.Hkv * wl.head_dim)
        o, _, _, _ = R.prefill_chunk(L, h, q, k, v, c0)
        outs.append(o[0].float().cpu().numpy())
    o_gpu = np.concatenate(outs)
    status, flags = S.spkv_cache_check(L.cache)
    assert status == S.OK, flags
    u, z = C.oracle_gates_rows(wl, 0, 0, T, W1, b1, W2, b2)
    lists = R.cache_lists(L)
    for kh in range(wl.Hkv):
        C.check_list(lists[kh], z[:, kh], T, u[:, kh], wl.tau)
    K, V = C.kv_rows(wl, 0, 0, T)
    rng = np.random.default_rng(0)
    ts = sorted(set([0, 1, 127, 128, 129, 4095, 4096, 4097, 8191, 8192, 12287, 16383] +
                    rng.integers(0, T, 20).tolist()))
    Q = wl.q_rows(0, 0, ts)
    for i, t in enumerate(ts):
        o_ref, _ = O.gated_attention(Q[i:i + 1], K[:t + 1], V[:t + 1], z[:t + 1], wl.window, [t])
        C.check_attn(o_gpu[t], o_ref[0], "bf16", f"prefill16k query {t}")


def test_decode32k_rethreshold_full_size():
    """One decode32k layer (32768-token context, utilities kept) re-thresholded from
    0.5 to 0.6 in place, then one per-token decode step at 0.6: sampled heads' index
    lists and stored rows, and sampled batch rows' outputs, against the oracle."""
    wl = _one_layer("decode32k")
    tau2 = 0.6
    p, Ls, inp = build_decode_state(wl, 1, 2, torch.device("cuda"), store_u=True)
    L = Ls[0]
    before = R.cache_lists(L)
    ws = S.alloc_rethreshold_workspace(p, L.cache)
    S.spkv_cache_rethreshold(p, L.cache, L.ring, tau2, ws)
    status, flags = S.spkv_cache_check(L.cache)
    assert status == S.OK, flags
    after = R.cache_lists(L)
    L.p = S.make_params(p.B, p.Hq, p.Hkv, p.head_dim, p.d_model, p.hid, p.window, tau2, p.dtype)
    step = DecodeStep(L.p, Ls, "cuda")
    step.launch(inp["h"][0], inp["q"][0], inp["k"][0], inp["v"][0], inp["t"][0])
    torch.cuda.synchronize()
    assert S.spkv_cache_check(L.cache)[0] == S.OK
    o = step.o[0].float().cpu().numpy()
    t = inp["t"][0].cpu().numpy()
    W1, b1, W2, b2 = C.weights(wl)
    for b in (1, 6):
        tb = int(t[b])
        u, _ = C.oracle_gates_rows(wl, 0, b, tb + 1, W1, b1, W2, b2)
        z2 = O.gate(u, tau2)
        K, V = C.kv_rows(wl, 0, b, tb + 1)
        for kh in (0, 5):
            bh = b * wl.Hkv + kh
            want = O.rethreshold(before[bh], u[before[bh], kh], tau2)
            near = set(np.nonzero((np.abs(u[:, kh] - tau2) < C.EXCLUDE) |
                                  (np.abs(u[:, kh] - wl.tau) < C.EXCLUDE))[0].tolist())
            got = [int(x) for x in after[bh] if int(x) not in near]
            assert got == [int(x) for x in want if int(x) not in near]
            Kc, Vc = R.cache_rows_kv(L, bh)
            assert np.array_equal(Kc.float().numpy(), K[after[bh], kh])
            assert np.array_equal(Vc.float().numpy(), V[after[bh], kh])
        q = wl.q_rows(0, b, [tb])
        o_ref, _ = O.gated_attention(q, K, V, z2, wl.window, [tb])
        C.check_attn(o[b], o_ref[0], "bf16", f"rethreshold decode row {b}")


def test_soft_attention_16k_full_size():
    """Soft-gated training-time attention (Eqs. (5)-(6)) over a 16384-token sequence
    with the prefill16k shapes, utilities from the utility perceptron (each side
    computes its own: GPU spkv_score, oracle in fp64; Eq. (5) is smooth, so their
    rounding differences do not flip anything), sampled query positions."""
    from sparse_decode_attention_spkv_b200.inputs import gen as G_
    wl = W.WORKLOADS["prefill16k"]
    T = wl.ctx[0]
    beta, c = 0.01, 1e6
    W1, b1, W2, b2 = C.weights(wl)
    p = S.make_params(1, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau, S.BF16)
    h = torch.empty((T, wl.d_model), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((1, T, wl.Hq, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    k = torch.empty((1, T, wl.Hkv, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    D.fill_normal(h, wl.key(0, G_.T_H), 1.0)
    D.fill_rope(q, wl.key(0, G_.T_Q), 0, wl.T_total, wl.qkv_scale, wl.rope_base)
    D.fill_rope(k, wl.key(0, G_.T_K), 0, wl.T_total, wl.qkv_scale, wl.rope_base)
    D.fill_normal(v, wl.key(0, G_.T_V), wl.qkv_scale)
    u = torch.empty((T, wl.Hkv), dtype=torch.float32, device="cuda")
    z = torch.empty((T, wl.Hkv), dtype=torch.uint8, device="cuda")
    S.spkv_score(p, h, T, C.dev(W1, "bf16"), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2), u, z)
    o = torch.empty_like(q)
    ws = torch.empty(S.spkv_soft_attn_workspace_bytes(p, T), dtype=torch.uint8, device="cuda")
    S.spkv_soft_attn(p, q, k, v, u, T, beta, c, o, None, ws)
    o_gpu = o[0].float().cpu().numpy()
    u_ref, _ = C.oracle_gates_rows(wl, 0, 0, T, W1, b1, W2, b2)
    K, V = C.kv_rows(wl, 0, 0, T)
    rng = np.random.default_rng(1)
    ts = sorted(set([0, 127, 128, 4096, 16383] + rng.integers(0, T, 10).tolist()))
    Q = wl.q_rows(0, 0, ts)
    for i, t in enumerate(ts):
        o_ref, _ = O.soft_gated_attention(Q[i:i + 1], K[:t + 1], V[:t + 1], u_ref[:t + 1], wl.tau,
                                          beta, c, wl.window, [t])
        C.check_attn(o_gpu[t], o_ref[0], "bf16", f"soft attention query {t}")
