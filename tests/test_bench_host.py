"""Host-side parts of bench.py on the CPU: the algorithmic FLOP count, the
recorded-traffic lookup, the clock-log parsing and the reference arm's JSON
line (the fp64 oracle on the tiny workload)."""
import hashlib
import json
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_selected_flops_counts_every_kept_pair():
    # 3 tiles of 128 tokens, the last one ragged (300 = 128 + 128 + 44)
    idx = np.array([[[0, 2], [1, 2], [0, 1]], [[2, 0], [1, 0], [2, 1]]])
    n = [128, 128, 44]
    want = sum(4 * 64 * n[i] * n[j] for h in range(2) for i in range(3) for j in idx[h, i])
    assert bench.selected_flops(idx, 300, 128, 64) == want


def test_landmark_flops_count_every_row_and_omitted_tile():
    # 2 heads, 300 tokens in 3 tiles, k = 2: every row sees 1 landmark
    assert bench.landmark_flops(2, 300, 3, 2, 64) == 4 * 64 * 2 * 300 * 1
    # the 1,024-view stage: 5.95e13 landmark FLOPs beside 4.87e14 selected
    assert abs(bench.landmark_flops(16, 1_406_976, 10_992, 660, 64) - 5.95e13) / 5.95e13 < 1e-3


def _fake_root(tmp_path, attn_src, recorded_sha, nbytes=123456.0):
    csrc = tmp_path / "linear_hybrid_attention_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "attn.cu").write_bytes(attn_src)
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "sparse_attn_w_traffic.json").write_text(json.dumps(
        {"dram_bytes_per_launch": nbytes, "attn_cu_sha256": recorded_sha,
         "summary": "profiles/sparse_attn_w.md"}))
    return str(tmp_path)


def test_recorded_traffic_only_for_the_measured_kernel(tmp_path, monkeypatch):
    src = b"// kernel source\n"
    sha = hashlib.sha256(src).hexdigest()
    monkeypatch.setattr(bench, "ROOT", _fake_root(tmp_path / "a", src, sha))
    value, where = bench.recorded_traffic("w")
    assert value == 123456.0 and where == "profiles/sparse_attn_w.md"
    # the kernel changed after the capture: no traffic figure
    monkeypatch.setattr(bench, "ROOT", _fake_root(tmp_path / "b", src + b" ", sha))
    value, why = bench.recorded_traffic("w")
    assert value is None and "changed" in why
    # no capture for this workload
    assert bench.recorded_traffic("other")[0] is None


def test_clock_sampler_parses_the_log(tmp_path):
    rows = [
        "0, GPU-1, 1965, 1965, 300.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, GPU-1, 1800, 1965, 990.1, 0x4, Not Active, Not Active, Not Active, Active",
        "0, GPU-1, 1790, 1965, 995.7, 0x4, Not Active, Not Active, Not Active, Active",
        "0, GPU-1, 1810, 1965, 992.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, GPU-1, 345, 1965, 90.0, 0x1, Not Active, Not Active, Not Active, Not Active",  # idle sample
    ]
    log = tmp_path / "clocks.csv"
    log.write_text("\n".join(rows) + "\n")
    s = bench.ClockSampler(0)
    s.path = str(log)
    s.proc = subprocess.Popen([sys.executable, "-c", "import time; time.sleep(30)"])
    clk = s.stop()
    assert clk["samples"] == 5
    assert clk["sm_max_mhz"] == 1965.0
    assert clk["sm_mhz"] == 1805.0          # median of the loaded samples (> half of max)
    assert clk["reasons"] == ["sw_power_cap"]


def test_reference_arm_prints_one_json_line_on_cpu():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "1"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [line for line in r.stdout.splitlines() if line.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "Mtokens/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["dtype"] == "f64"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "Mtokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("tiny")


def test_l2_note_states_the_size_relation():
    assert bench.l2_note(2.88e9).startswith("inputs larger than L2")
    assert bench.l2_note(90e6).startswith("inputs smaller than L2")
