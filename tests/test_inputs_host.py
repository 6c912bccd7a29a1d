"""Host side of the seeded input generator (no GPU)."""
import numpy as np
import torch

from sparse_decode_attention_spkv_b200.inputs import gen, workloads as W


def test_splitmix_reference_values():
    # SplitMix64 from state 0: the first outputs of Vigna's reference generator.
    assert gen.draws(0, np.array([0], dtype=np.uint64))[0] == np.uint64(0xE220A8397B1DCDAF)
    assert gen.draws(0, np.array([1], dtype=np.uint64))[0] == np.uint64(0x6E789E6AA1B965F4)
    assert gen.draws(0, np.array([2], dtype=np.uint64))[0] == np.uint64(0x06C45D188009454F)


def test_streams_are_deterministic_and_distinct():
    k1 = gen.stream_key(0, 1, 2, 3)
    assert k1 == gen.stream_key(0, 1, 2, 3)
    assert k1 != gen.stream_key(0, 1, 2, 4) != gen.stream_key(1, 1, 2, 3)
    a = gen.normal(k1, (1000,), 1.0, "f32")
    b = gen.normal(k1, (1000,), 1.0, "f32")
    assert np.array_equal(a, b)
    # offsets address the same flat elements
    assert np.array_equal(gen.normal(k1, (10,), 1.0, "f32", offset=500), a[500:510])


def test_normal_moments():
    x = gen.normal_f64(gen.stream_key(0, 99), np.arange(1 << 20, dtype=np.uint64))
    assert abs(x.mean()) < 5e-3 and abs(x.std() - 1.0) < 5e-3
    assert abs(np.mean(x ** 4) - 3.0) < 0.05


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(100000).astype(np.float32)
    # exact ties: low 16 bits 0x8000
    ties = (rng.integers(0, 1 << 15, 1000).astype(np.uint32) << 16 | 0x8000).view(np.float32)
    x = np.concatenate([x, ties[np.isfinite(ties)]])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(gen.f32_to_bf16_bits(x), want)


def test_rows_match_full_tensor():
    wl = W.small_case("decode32k", ctx=[64], decode_steps=0)
    k = wl.k_rows(0, 0, np.arange(64))
    k2 = wl.k_rows(0, 0, [5, 17])
    assert np.array_equal(k[[5, 17]], k2)
    assert k.shape == (64, 8, 128)


def test_rope_rotation_preserves_pair_norms():
    key = gen.stream_key(0, 7)
    rows = np.arange(16)
    plain = gen.normal_rows(key, 2 * 8, rows, 1.0, "f32").reshape(16, 2, 8)
    x64 = gen.normal_f64(key, np.arange(16 * 16, dtype=np.uint64)).reshape(16, 2, 8)
    rot = gen.rope_rows(key, 8, 2, rows, rows * 7, 1.0, 1e4, "f32")
    n0 = x64[..., :4] ** 2 + x64[..., 4:] ** 2
    n1 = rot[..., :4].astype(np.float64) ** 2 + rot[..., 4:].astype(np.float64) ** 2
    assert np.allclose(n0, n1, rtol=1e-6)
    assert np.array_equal(gen.rope_rows(key, 8, 2, rows[:1], [0], 1.0, 1e4, "f32")[0], plain[0])


def test_workload_biases_present():
    table = W.load_biases()
    for name, wl in W.WORKLOADS.items():
        assert name in table
        assert len(table[name]["b2"]) == wl.layers
        assert all(len(r) == wl.Hkv for r in table[name]["b2"])
