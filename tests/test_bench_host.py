"""Host-side logic of bench.py (no GPU): the profile key that ties a committed ncu
capture to the kernel code it was taken on, and the scaling of its traffic."""
import json
import os

import bench


def test_code_hash_ignores_comments_and_blank_lines(tmp_path):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    a.write_text("int x = 1;  // one\n\nint y = 2;\n")
    b.write_text("// a header comment\nint x = 1;\n   \nint y = 2;   // two\n")
    assert bench._code_hash([a]) == bench._code_hash([b])
    b.write_text("int x = 1;\nint y = 3;\n")
    assert bench._code_hash([a]) != bench._code_hash([b])


def test_profiled_traffic_scales_with_the_launch(monkeypatch, tmp_path):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "decode_attn_decode32k.json").write_text(json.dumps(
        {"source_hash": "abc", "traffic_bytes_per_launch": 1020,
         "algorithmic_bytes_per_launch": 1000}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "_kernel_source_hash", lambda: "abc")
    assert abs(bench._profiled_traffic(2000.0) - 2040.0) < 1e-9
    monkeypatch.setattr(bench, "_kernel_source_hash", lambda: "other")
    assert bench._profiled_traffic(2000.0) is None  # the kernel changed since the capture


def test_committed_profile_key_is_well_formed():
    with open(os.path.join(bench.ROOT, "profiles", "decode_attn_decode32k.json")) as f:
        key = json.load(f)
    assert {"source_hash", "traffic_bytes_per_launch", "algorithmic_bytes_per_launch"} <= set(key)
    assert float(key["traffic_bytes_per_launch"]) >= float(key["algorithmic_bytes_per_launch"])


def test_reference_arm_line(monkeypatch):
    """--impl reference: rank 0 prints the oracle's line with the contract's keys; its
    per-step sample is bounded (about 600 oracle units over all timed steps)."""
    import argparse
    args = argparse.Namespace(steps=1, warmup=3, cpu_units=1)
    out = bench.run_reference(args, world=1, rank=0)
    assert out["impl"] == "reference" and out["unit"] == "tokens/s" and out["value"] > 0
    assert out["e2e"]["value"] == out["value"]
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["e2e"]["d2h_bytes_per_step"] == 0
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["value"] == out["value"]
    assert bench.run_reference(args, world=2, rank=1) is None  # other ranks: no work, no line
