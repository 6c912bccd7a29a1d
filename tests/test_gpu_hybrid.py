"""Hybrid local/global stacks ("Self-Pruned Key-Value Attention", §3.3 "Hybrids":
SP-KV applied only to the global layers of a transformer that alternates local and
global attention; the local layers keep no long-range cache).  A local layer here has
no cache at all: its prefill and decode attend to the causal window only, which is
Eq. (4) with every gate 0 (tau > 1).  Checked against the oracle layer by layer
through chunked prefill and per-token decode (GPU required)."""
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
    # 3 local : 1 global, tensor-core prefill and decode
    "bf16_3to1": (W.small_case("decode32k", cid=80, B=2, Hq=8, Hkv=2, d_model=256, hid=64,
                               ctx=[1152], decode_steps=24, layers=4, keep="fixed25"), 4),
    # fp32, head_dim 64, 1 local : 1 global, ragged prefill chunks
    "f32_1to1": (W.small_case("tiny", cid=81, B=2, ctx=[700], decode_steps=20, layers=2), 2),
}


def _params(wl):
    return S.make_params(wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau,
                         S.BF16 if wl.dtype == "bf16" else S.F32)


@pytest.mark.parametrize("name,attn_first", [(n, False) for n in sorted(CASES)] +
                         [("bf16_3to1", True)])
def test_hybrid_stack_matches_oracle(name, attn_first):
    """attn_first: every layer's decode attention on the state before the step's update
    (spkv_decode_attn_before_append), the update and scoring on a second stream."""
    wl, period = CASES[name]
    side = torch.cuda.Stream() if attn_first else None
    T0, steps, w = wl.ctx[0], wl.decode_steps, wl.window
    T = T0 + steps
    p = _params(wl)
    layers, host, gates = [], [], []
    for l in range(wl.layers):
        h, q, k, v = (np.stack(x) for x in zip(*[C.host_rows(wl, l, b, np.arange(T))
                                                  for b in range(wl.B)]))
        host.append((h, q, k, v))
        if l % period != period - 1:
            layers.append(R.Layer.create_local(p))
            gates.append(np.zeros((wl.B, T, wl.Hkv), dtype=np.uint8))
        else:
            W1, b1, W2, b2 = C.weights(wl, l)
            mp = R.pages_for(T)
            layers.append(R.Layer.create(p, C.dev(W1, wl.dtype), C.dev_f32(b1), C.dev_f32(W2),
                                         C.dev_f32(b2), num_pages=wl.B * wl.Hkv * mp,
                                         max_pages_per_head=mp))
            _, z = C.oracle_gates(h.reshape(-1, wl.d_model), W1, b1, W2, b2, wl.tau)
            gates.append(z.reshape(wl.B, T, wl.Hkv))
    chunk = 384
    for l, L in enumerate(layers):
        h, q, k, v = host[l]
        for c0 in range(0, T0, chunk):
            c1 = min(T0, c0 + chunk)
            o, _, _, _ = R.prefill_chunk(L, C.dev(h[:, c0:c1], wl.dtype), C.dev(q[:, c0:c1], wl.dtype),
                                         C.dev(k[:, c0:c1], wl.dtype), C.dev(v[:, c0:c1], wl.dtype),
                                         c0, n_compact=max(0, min(c1, T0 - w) - c0))
            if c0 == 0 or c1 == T0:
                og = C.to_np(o)
                for b in range(wl.B):
                    o_ref, _ = O.gated_attention(q[b, c0:c1], k[b, :c1], v[b, :c1], gates[l][b, :c1],
                                                 w, np.arange(c0, c1))
                    C.check_attn(og[b], o_ref, wl.dtype, f"{name} layer {l} prefill [{c0},{c1}) b={b}")
    for i in range(steps):
        t = T0 + i
        t_pos = torch.full((wl.B,), t, dtype=torch.int32, device="cuda")
        for l, L in enumerate(layers):
            h, q, k, v = host[l]
            o, _, _ = R.decode_step(L, t_pos, C.dev(h[:, t], wl.dtype), C.dev(q[:, t], wl.dtype),
                                    C.dev(k[:, t], wl.dtype), C.dev(v[:, t], wl.dtype),
                                    score_stream=side, attn_first=attn_first)
            if side is not None:
                torch.cuda.current_stream().wait_stream(side)
            og = C.to_np(o)
            for b in range(wl.B):
                o_ref, _ = O.gated_attention(q[b, t:t + 1], k[b, :t + 1], v[b, :t + 1],
                                             gates[l][b, :t + 1], w, [t])
                C.check_attn(og[b], o_ref[0], wl.dtype, f"{name} layer {l} step {i} b={b}")
    for L in layers:
        if not L.local:
            assert S.spkv_cache_check(L.cache)[0] == S.OK


def test_window_only_equals_tau_above_one():
    """A cache-less layer and a cache-backed layer whose threshold no utility reaches
    (tau > 1: nothing is ever gated in) give the same decode outputs, bit for bit."""
    wl = W.small_case("decode32k", cid=82, B=2, Hq=8, Hkv=2, d_model=128, hid=32, ctx=[600],
                      decode_steps=5, layers=1, keep="fixed25")
    T0, steps = wl.ctx[0], wl.decode_steps
    T = T0 + steps
    h, q, k, v = (np.stack(x) for x in zip(*[C.host_rows(wl, 0, b, np.arange(T))
                                              for b in range(wl.B)]))
    p_hi = S.make_params(wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, 1.5, S.BF16)
    W1, b1, W2, b2 = C.weights(wl)
    mp = R.pages_for(T)
    glob = R.Layer.create(p_hi, C.dev(W1, "bf16"), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                          num_pages=wl.B * wl.Hkv * mp, max_pages_per_head=mp)
    loc = R.Layer.create_local(p_hi)
    for L in (glob, loc):
        R.prefill_chunk(L, C.dev(h[:, :T0], "bf16"), C.dev(q[:, :T0], "bf16"),
                        C.dev(k[:, :T0], "bf16"), C.dev(v[:, :T0], "bf16"), 0,
                        n_compact=T0 - wl.window)
    for i in range(steps):
        t = T0 + i
        t_pos = torch.full((wl.B,), t, dtype=torch.int32, device="cuda")
        outs = [R.decode_step(L, t_pos, C.dev(h[:, t], "bf16"), C.dev(q[:, t], "bf16"),
                              C.dev(k[:, t], "bf16"), C.dev(v[:, t], "bf16"))[0] for L in (glob, loc)]
        assert torch.equal(outs[0], outs[1])
    assert int(glob.cache.count.sum().item()) == 0
