"""The bench's reference arm (the oracle on the host cores) prints one JSON
line with the keys the driver reads; the CPU-side helpers of the device arm."""
import json
import os
import subprocess
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["warmup"] >= 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "tiny"


def test_max_over_ranks_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    v = torch.tensor([3.0, 1.0])
    assert bench.max_over_ranks(v, 1).tolist() == [3.0, 1.0]


def test_attention_traffic_only_for_recorded_source(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    assert bench.attention_traffic("no-such-workload") is None
    h = bench.attention_sources_hash()
    monkeypatch.setattr(bench, "ATTN_TRAFFIC", {"w": {"sources_sha256_16": h, "bytes": 123},
                                                "old": {"sources_sha256_16": "0" * 16, "bytes": 456}})
    assert bench.attention_traffic("w") == 123
    assert bench.attention_traffic("old") is None  # recorded for other attention sources


def test_default_workload_is_largest_single_gpu_config():
    sys.path.insert(0, ROOT)
    from video_dit_sparse_da2_b200.inputs import ALL
    src = open(os.path.join(ROOT, "bench.py")).read()
    largest = max(ALL, key=lambda w: 4 * w.B * w.H * w.N * w.N * w.d)
    assert f'ap.add_argument("--workload", default="{largest.name}")' in src
