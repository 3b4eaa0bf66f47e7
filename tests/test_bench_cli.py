"""bench.py pieces that need no GPU: the reference arm's JSON line (the fp64
oracle on the host cores) and the lookup of DRAM traffic recorded for a
kernel source."""
import json
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] >= 3
    assert d["config"]["workload"].startswith("decode: hidden 2048, 512 experts")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_traffic_lookup_matches_source_hash(tmp_path, monkeypatch):
    import bench
    sha = bench.src_hash("decode.cu")
    assert len(sha) == 16
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.txt").write_text(f"# comment\nk_decode {sha} 12345\nk_decode 0000000000000000 1\n")
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    assert bench.traffic_from_profiles("k_decode", sha) == 12345.0
    assert bench.traffic_from_profiles("k_decode", "ffffffffffffffff") is None
    assert bench.traffic_from_profiles("expert_ffn_prefill_512", sha) is None


def test_expert_stats():
    import numpy as np
    import bench
    steps = [np.array([[0, 1], [1, 2]]), np.array([[3, 4], [3, 5]])]
    st = bench.expert_stats(steps, hot=2)
    assert st["distinct_experts_per_step"] == 3.0          # {0,1,2} and {3,4,5}
    assert st["top2_share"] == 0.5                         # experts 1 and 3 take 4 of 8 selections
    assert st["steps"] == 2


def _pk():
    return {"hbm_gbs": 6557.4, "bf16_tflops": 1667.0, "source": "measured"}


def test_roofline_bytes_exclude_intermediates():
    """Algorithmic bytes: distinct blobs + x once + y once; y_perm, h and
    x_perm are not credited.  FLOPs: 2*3*H*I per assignment incl. the shared expert."""
    import bench
    H, I, E, k, T, blob = 2048, 512, 512, 10, 8192, 1769472
    r = bench.layer_roofline("prefill", False, H, I, E, k, T, 512, blob, 2.0, _pk(), 1965.0)
    assert r["algorithmic_bytes_per_launch"] == 513 * blob + T * H * 2 + T * H * 4
    assert r["algorithmic_flops_per_launch"] == 2 * 3 * H * I * T * (k + 1)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    r = bench.layer_roofline("prefill", False, H, I, E, k, 512, 512, blob, 0.2, _pk(), 1965.0)
    assert r["bound"] == "hbm" and r["algorithmic_bytes_per_launch"] == 513 * blob + 512 * H * 6
    # fused decode: 11 blobs + router rows + x + logits + y
    r = bench.layer_roofline("decode", True, H, I, E, k, 1, k, blob, 0.01, _pk(), 1965.0)
    assert r["algorithmic_bytes_per_launch"] == 11 * blob + E * H * 2 + H * 2 + E * 4 + H * 4


def test_verify_roofline_names_the_binding_roof():
    """Verify windows: max(HBM, FP32 ALU) with both fractions reported."""
    import bench
    H, I, k, blob = 2048, 512, 10, 983040
    alu = bench.fp32_peak_tflops(1965.0)
    assert abs(alu - 148 * 128 * 2 * 1.965e9 / 1e12) < 1e-9
    # 16 tokens over 40 distinct experts: FLOPs 16 x 69.2 M vs 41 blobs
    r = bench.layer_roofline("verify", False, H, I, 512, k, 16, 40, blob, 0.1, _pk(), 1965.0)
    t_hbm = r["algorithmic_bytes_per_launch"] / (6557.4e9)
    t_alu = r["algorithmic_flops_per_launch"] / (alu * 1e12)
    assert r["bound"] == ("alu" if t_alu > t_hbm else "hbm")
    assert "hbm_frac" in r and "alu_frac" in r
    assert abs(r["binding_roof_time_us"] - max(t_hbm, t_alu) * 1e6) < 1e-2
    # a window of 2 over 20 experts is HBM-bound
    r = bench.layer_roofline("verify", False, H, I, 512, k, 2, 20, blob, 0.03, _pk(), 1965.0)
    assert r["bound"] == "hbm"


def test_both_arms_print_the_same_config():
    import argparse
    import bench
    args = argparse.Namespace(layers=0, unfused=False)
    for kind, T in (("decode", 1), ("verify", 16), ("prefill", 8192)):
        n_layers, mode, fused = bench.workload_shape(kind, args)
        bits = 2 if kind == "verify" else 4
        blob = 983040 if bits == 2 else 1769472
        a = bench.layer_config(kind, 2048, 512, 10, 512, bits, T, n_layers, blob, mode, fused, 1)
        assert a["workload"].startswith(f"{kind}: hidden 2048, 512 experts + 1 shared, top-10")
        assert a["layer_copies"] == (2 if kind == "prefill" else 16)


def test_src_hash_covers_headers(tmp_path, monkeypatch):
    """An edit to any internal header changes every kernel's source hash."""
    import shutil
    import bench
    root = tmp_path
    shutil.copytree(ROOT / "quantized_expert_ffn_route_b200" / "csrc", root / "quantized_expert_ffn_route_b200" / "csrc")
    (root / "include").mkdir()
    shutil.copy(ROOT / "include" / "moe.h", root / "include" / "moe.h")
    monkeypatch.setattr(bench, "ROOT", root)
    h0 = bench.src_hash("decode.cu")
    p = root / "quantized_expert_ffn_route_b200" / "csrc" / "qdot.cuh"
    p.write_text(p.read_text() + "\n// edit\n")
    assert bench.src_hash("decode.cu") != h0


def test_oracle_baseline_adds_a_one_thread_run():
    import bench
    import oracle
    calls = []
    r = bench.oracle_baseline(lambda n: calls.append(oracle.max_threads()), 0.05, 3, 2, "tiny calls")
    assert r["kind"] == "oracle" and r["cores"] == bench.host_cores() and r["value"] > 0
    one = r["one_thread"]
    assert one["cores"] == 1 and one["value"] > 0 and "1 thread" in one["sample"]
    assert 1 in calls and bench.host_cores() in calls           # both runs used their thread count
    assert oracle.max_threads() == bench.host_cores()            # restored afterwards


def test_reference_arm_of_the_three_tier_workload():
    """The reference arm runs the oracle on the three-tier workload's steps and
    prints the same `config` the measured arm builds."""
    import bench
    import workloads as W
    out = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference", "--workload", "paging_ssd",
                          "--steps", "1", "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    d = json.loads([l for l in out.stdout.splitlines() if l.strip()][-1])
    c = W.PAGING_SSD
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["config"] == bench.paging_ssd_config(c["E"], c["k"], 983040, c, 1)
    assert "4096 experts" in d["config"]["workload"] and "O_DIRECT" in d["config"]["workload"]


def test_ffn_mode_override():
    import argparse
    import bench
    for name, want in (("auto", 0), ("gemv", 1), ("gemm", 2)):
        args = argparse.Namespace(layers=0, unfused=False, ffn_mode=name)
        assert bench.workload_shape("verify", args)[1] == want
    assert bench.workload_shape("prefill", argparse.Namespace(layers=0, unfused=False, ffn_mode="auto"))[1] == 2


def test_host_memory_guard_stops_with_a_message():
    import bench
    bench.require_host_memory("tiny", 1 << 20, spare=0)          # a megabyte is always there
    with pytest.raises(SystemExit) as ei:
        bench.require_host_memory("huge", 1 << 60)
    assert "huge" in str(ei.value) and "page-locked" in str(ei.value)
