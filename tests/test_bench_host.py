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


def test_reference_arm_prints_one_line_per_workload():
    """bench.py --impl reference (the oracle on the host cores, a bounded sample)
    prints the contract's JSON line with the oracle as its cpu_baseline."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for wl, unit in (("decode", "GB/s"), ("prefill", "TOPS")):
        r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                            "--workload", wl, "--steps", "1", "--warmup", "0", "--cpu-seconds", "1"],
                           capture_output=True, text=True, timeout=600,
                           env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
        assert r.returncode == 0, r.stderr[-2000:]
        lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
        assert len(lines) == 1
        d = json.loads(lines[0])
        assert d["impl"] == "reference" and d["unit"] == unit and d["value"] > 0
        assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
        assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_decode_config_names_the_batch_and_expert_count():
    """--tokens / --experts change the decode line's config on both arms; the
    default line keeps the GLM-5.2 layer with batch 1."""
    import json
    import subprocess
    import sys
    import moe_inputs as mi
    d0 = bench.decode_config(mi.WORKLOADS["decode"], 1)
    assert "256 routed experts" in d0["workload"] and "batch 1," in d0["workload"] and d0["T"] == 1
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--tokens", "4", "--experts", "64", "--steps", "1", "--warmup", "0",
                        "--cpu-seconds", "1"],
                       capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][0])
    assert d["config"]["T"] == 4 and d["config"]["E"] == 64 and d["config"]["global_batch"] == 4
    assert "64 routed experts" in d["config"]["workload"] and "batch 4," in d["config"]["workload"]
    bad = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--tokens", "17"],
                         capture_output=True, text=True, timeout=600,
                         env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert bad.returncode != 0 and "1 to 16 tokens" in bad.stderr
