"""bench.py pieces that need no GPU: the reference arm's JSON line (the fp64
oracle on the host cores) and the lookup of DRAM traffic recorded for a
kernel source."""
import json
import subprocess
import sys
from pathlib import Path

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
