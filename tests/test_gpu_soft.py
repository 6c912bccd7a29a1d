"""Soft-gated attention of SP-KV training (§2.1, Eqs. (5)-(6)) on the GPU against the
oracle, element by element (GPU required).

The utilities u are drawn directly from the seeded generator (uniform around tau, so
that every regime of Eq. (6) occurs: biases near 0, of moderate size, and about -c),
and the same values go to both sides.  Cases cover the tensor-core path (bf16,
head_dim 128, window 128, sequence a multiple of 128) and the CUDA-core path (fp32,
head_dim 64, ragged lengths), c = 0 (plain causal attention) and a vanishing
temperature (the hard gate of Eq. (4))."""
import numpy as np
import pytest
import torch

from oracle import spkv_oracle as O
from sparse_decode_attention_spkv_b200.inputs import gen
from sparse_decode_attention_spkv_b200.inputs import workloads as W
from tests import cases as C

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from sparse_decode_attention_spkv_b200 import spkv as S


def _case(name, T, beta=0.01, c=1e6, **kw):
    base = "tiny" if kw.get("dtype") == "f32" else "decode32k"
    wl = W.small_case(base, ctx=[T], decode_steps=0, layers=1, **kw)
    return wl, T, beta, c


CASES = {
    "bf16_tc_512": _case("bf16_tc_512", 512, cid=70, B=1, Hq=8, Hkv=2),
    "bf16_tc_b2_g4_384": _case("bf16_tc_b2_g4_384", 384, cid=71, B=2, Hq=16, Hkv=4),
    "bf16_tc_c0": _case("bf16_tc_c0", 256, c=0.0, cid=72, B=1, Hq=4, Hkv=2),
    "bf16_tc_hard_limit": _case("bf16_tc_hard_limit", 384, beta=1e-7, cid=73, B=1, Hq=4, Hkv=2),
    "bf16_simple_ragged_300": _case("bf16_simple_ragged_300", 300, cid=74, B=1, Hq=8, Hkv=2),
    "bf16_simple_g1_d64": _case("bf16_simple_g1_d64", 200, cid=75, B=2, Hq=2, Hkv=2, head_dim=64),
    "f32_tiny_260": _case("f32_tiny_260", 260, cid=76, B=1, dtype="f32"),
}


def _inputs(wl, T):
    q = np.stack([wl.q_rows(0, b, np.arange(T)) for b in range(wl.B)])
    k = np.stack([wl.k_rows(0, b, np.arange(T)) for b in range(wl.B)])
    v = np.stack([wl.v_rows(0, b, np.arange(T)) for b in range(wl.B)])
    n = wl.B * T * wl.Hkv
    u = gen.to_f32(gen.uniform_f64(wl.key(0, gen.T_U), np.arange(n), wl.tau - 0.3, wl.tau + 0.3))
    return q, k, v, u.reshape(wl.B, T, wl.Hkv)


@pytest.mark.parametrize("name", sorted(CASES))
def test_soft_gated_attention_matches_oracle(name):
    wl, T, beta, c = CASES[name]
    p = S.make_params(wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau,
                      S.BF16 if wl.dtype == "bf16" else S.F32)
    q, k, v, u = _inputs(wl, T)
    o = torch.empty((wl.B, T, wl.Hq, wl.head_dim), dtype=torch.bfloat16 if wl.dtype == "bf16"
                    else torch.float32, device="cuda")
    lse = torch.empty((wl.B, T, wl.Hq), dtype=torch.float32, device="cuda")
    ws = torch.empty(S.spkv_soft_attn_workspace_bytes(p, T), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.spkv_soft_attn(p, C.dev(q, wl.dtype), C.dev(k, wl.dtype), C.dev(v, wl.dtype), C.dev_f32(u), T,
                     beta, c, o, lse, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    o_gpu, lse_gpu = C.to_np(o), lse.cpu().numpy()
    for b in range(wl.B):
        o_ref, lse_ref = O.soft_gated_attention(q[b], k[b], v[b], u[b], wl.tau, beta, c, wl.window,
                                                np.arange(T))
        C.check_attn(o_gpu[b], o_ref, wl.dtype, f"{name} b={b}")
        assert np.allclose(lse_gpu[b], lse_ref, atol=2e-3, rtol=1e-4), f"{name} lse"


def test_soft_zero_length_and_bad_arguments():
    wl, T, beta, c = CASES["bf16_tc_512"]
    p = S.make_params(wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau, S.BF16)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    assert S.lib.spkv_soft_attn(S.ctypes.byref(p), None, None, None, None, 0, 0.01, 1e6, None, None,
                                None, 0, None, None) == S.OK
    t = torch.empty(1024, dtype=torch.uint8, device="cuda")
    a = t.data_ptr()
    for b_, c_ in ((0.0, 1e6), (-1.0, 1e6), (0.01, -1.0), (0.01, float("inf"))):
        assert S.lib.spkv_soft_attn(S.ctypes.byref(p), a, a, a, a, 128, b_, c_, a, None, a, 1 << 20,
                                    None, None) == S.ERR_ARG
    assert S.lib.spkv_soft_attn(S.ctypes.byref(p), a, a, a, a, 128, 0.01, 1e6, a, None, a, 16,
                                None, None) == S.ERR_ARG  # workspace too small
    torch.cuda.synchronize()
    assert int(ws.numel()) == 256
