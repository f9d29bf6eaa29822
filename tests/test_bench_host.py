"""Host-side logic of bench.py, on the CPU: the reference arm's JSON line and
the guard that reports measured DRAM traffic only for the sources it was
captured from."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fake_tree(tmp_path, text):
    csrc = tmp_path / "ternary_weight_moe_forward_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "decode.cuh").write_text(text)
    return tmp_path


def test_digest_follows_the_sources(tmp_path, monkeypatch):
    root = _fake_tree(tmp_path, "int x;\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    d0 = bench.csrc_digest()
    assert d0 == bench.csrc_digest()
    (root / "ternary_weight_moe_forward_b200" / "csrc" / "decode.cuh").write_text("int y;\n")
    assert bench.csrc_digest() != d0


def test_traffic_only_for_matching_sources(tmp_path, monkeypatch):
    root = _fake_tree(tmp_path, "int x;\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    prof = tmp_path / "summary.md"
    monkeypatch.setattr(bench, "PROFILE_T64", str(prof))
    assert bench.measured_traffic() is None                      # no summary
    prof.write_text(f"csrc_sha256: {bench.csrc_digest()}\ntraffic_bytes: 12345\n")
    assert bench.measured_traffic() == 12345
    prof.write_text("csrc_sha256: 00\ntraffic_bytes: 12345\n")
    assert bench.measured_traffic() is None                      # sources changed since the capture
    prof.write_text(f"csrc_sha256: {bench.csrc_digest()}\n")
    assert bench.measured_traffic() is None                      # no figure


def test_algorithmic_bytes_of_the_expert_kernel():
    # codes of gate, up and down (2 bits each) and one fp32 alpha per output row
    per_expert = 3 * 512 * 2048 // 4 + (2 * 512 + 2048) * 4
    assert per_expert == 798720
    assert bench.experts_bytes(222, 64) == 222 * per_expert + 64 * 2048 + 64 * 2048 * 4


def test_reference_arm_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["higher_is_better"] is True and line["config"]["workload"] == bench.WORKLOAD
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_per_batch_entry_by_expert_path():
    # split: (route, after gate/up, end) in ms, per layer
    split = [(0, (0.010, 0.020, 0.030)), (1, (0.012, 0.022, 0.031))]
    fused = bench.per_T_entry(1, True, [0.02, 0.02], [0.025], split, [8, 8], 6650.0)
    assert fused["expert_path"] == "fused"
    assert "us_gate_up" not in fused and "gate_up_hbm_frac" not in fused
    assert abs(fused["us_experts"] - 1e3 * (0.020 + 0.019) / 2) < 1e-9
    two = bench.per_T_entry(64, False, [0.07], [0.08], split, [222, 222], 6650.0)
    assert two["expert_path"] == "two-kernel"
    assert abs(two["us_gate_up"] - 1e3 * (0.010 + 0.010) / 2) < 1e-9
    assert abs(two["us_down_combine"] - 1e3 * (0.010 + 0.009) / 2) < 1e-9
    assert abs(two["tokens_per_s"] - 64 / 0.07e-3) < 1e-6 * two["tokens_per_s"]
