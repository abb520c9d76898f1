"""Host-side arithmetic of bench.py (no GPU): the prefill layer's attainable
floor, and the committed-profile traffic lookup that goes null once a kernel's
source changes."""
import os

import bench


def test_prefill_attainable_floor():
    # GLM-shaped prefill: 18,432 rows x 3 x H x I int8 MACs; union 213 + shared expert
    ops = 2.0 * 2048 * 9 * 3 * 6144 * 2048
    a = bench.attainable(ops, 213, 20_054_016, 6534.8, 1633.5, 9.19)
    assert a["bound"] == "hbm"
    assert abs(a["hbm_floor_us"] - 214 * 20_054_016 / 6534.8e9 * 1e6) < 0.1
    assert abs(a["int8_floor_us"] - ops / (2 * 1633.5e12) * 1e6) < 0.1
    assert abs(a["frac"] - a["floor_us"] / 9190.0) < 1e-4
    t = bench.attainable(ops, 1, 20_054_016, 6534.8, 1633.5, 1.0)   # few experts: tensor-bound
    assert t["bound"] == "tensor" and t["floor_us"] == t["int8_floor_us"]


def test_profiled_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    import hashlib
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (prof / "k_test.md").write_text(f"traffic_bytes_per_launch: 1234\nsource: k.cu sha256[:16] {sha}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k_test", "k.cu") == 1234
    src.write_text("kernel v2\n")
    assert bench.profiled_traffic("k_test", "k.cu") is None
    assert bench.profiled_traffic("missing", "k.cu") is None
    assert os.path.exists(str(src))
