"""Host-side checks of bench.py (no GPU): the algorithmic byte count behind
`roofline.achieved` for both decoder stacks, the guard that keeps a stale ncu
traffic record out of the JSON line, and the reference arm's JSON line (the
CPU oracle timed on a bounded sample, run here as a subprocess).
"""
import json
import os
import subprocess
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from dense_fp8_gemm_b200 import workloads  # noqa: E402


def test_algorithmic_bytes_by_hand():
    # One decode step of the 32B attention projections at M = 16, dense_frac 0.25 (tail).
    # Per weight row: a 2:4 column costs half a byte of values plus a quarter of a nibble of
    # metadata (0.625 B), a dense column one byte; plus fp32 row scales, the e4m3 activations
    # and their fp32 scales once per launch, and the bf16 output.
    M = 16
    # q/k/v grouped: N = 8192 + 1024 + 1024 rows over K = 5120 (3840 2:4 columns, 1280 dense)
    qkv = 10240 * 3840 // 2 + 10240 * 3840 // 8 + 10240 * 1280 + 4 * 10240 + M * 5120 + 4 * M + 2 * M * 10240
    # o_proj: N = 5120 rows over K = 8192 (6144 2:4 columns, 2048 dense)
    o = 5120 * 6144 // 2 + 5120 * 6144 // 8 + 5120 * 2048 + 4 * 5120 + M * 8192 + 4 * M + 2 * M * 5120
    assert qkv == 38133824 and o == 30462016
    assert workloads.group_algorithmic_bytes([(8192, 5120, 1280), (1024, 5120, 1280), (1024, 5120, 1280)], M) == qkv
    assert workloads.algorithmic_bytes(5120, 8192, 2048, M) == o
    args = types.SimpleNamespace(tokens=M, dense_frac=0.25, layers=1, workload="attn32b")
    assert bench.step_bytes(args) == qkv + o
    # the dense FP8 comparison moves every column as one byte
    dense_qkv = 10240 * 5120 + 4 * 10240 + M * 5120 + 4 * M + 2 * M * 10240
    dense_o = 5120 * 8192 + 4 * 5120 + M * 8192 + 4 * M + 2 * M * 5120
    assert bench.step_bytes(args, dense=True) == dense_qkv + dense_o


def test_chain36b_step_bytes_by_hand():
    # One decode step of the 36B chain at M = 16: 64 layers of q/k/v grouped (10240 + 1024 + 1024 rows,
    # K = 5120), o_proj (5120 x 10240), gate+up (55296 x 5120) and down (5120 x 27648), dense_frac 0.25.
    M = 16

    def launch(rows, K):
        Kd = K // 4
        Ks = K - Kd
        return sum(n * Ks // 2 + n * Ks // 8 + n * Kd + 4 * n + 2 * M * n for n in rows) + M * K + 4 * M

    layer = launch([10240, 1024, 1024], 5120) + launch([5120], 10240) + launch([55296], 5120) + \
        launch([5120], 27648)
    args = types.SimpleNamespace(tokens=M, dense_frac=0.25, layers=0, workload="chain36b")
    assert bench.step_bytes(args) == 64 * layer
    # 24.8 GB of packed weights per step (0.71875 of the dense FP8 bytes)
    weights = 64 * 0.71875 * (12288 * 5120 + 5120 * 10240 + 55296 * 5120 + 5120 * 27648)
    assert abs(weights - 24.8e9) < 0.05e9
    assert bench.step_bytes(args) > weights
    assert bench.sweep_tokens(types.SimpleNamespace(tokens=16, sweep=None, layers=0, workload="chain36b")) == \
        [1, 4, 64, 256]


def test_stale_traffic_record_is_not_reported(monkeypatch, tmp_path):
    args = types.SimpleNamespace(tokens=16, workload="chain36b")
    rec = {"kernel_source_sha256": "ab" * 32, "dram_bytes_per_launch_avg": 12345}
    path = tmp_path / "traffic.txt"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "traffic_path", lambda a: str(path))
    monkeypatch.setattr(bench, "kernel_source_sha256", lambda: rec["kernel_source_sha256"])
    assert bench.read_traffic(args) == 12345
    monkeypatch.setattr(bench, "kernel_source_sha256", lambda: "0" * 64)
    assert bench.read_traffic(args) is None


def test_reference_arm_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == "spense_fp8_weight_stream_GBps" and line["unit"] == "GB/s"
    assert line["higher_is_better"] is True and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"].startswith("chain36b")
