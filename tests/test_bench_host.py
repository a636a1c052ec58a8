"""Host-side checks of bench.py (no GPU): the algorithmic byte count behind
`roofline.achieved`, the guard that keeps a stale ncu traffic record out of
the JSON line, the L2 statement, and the reference arm's JSON line (the CPU
oracle timed on a bounded sample, run here as a subprocess).
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
    args = types.SimpleNamespace(tokens=M, dense_frac=0.25, layers=8)
    assert bench.step_bytes(args) == qkv + o
    # the dense FP8 comparison moves every column as one byte
    dense_qkv = 10240 * 5120 + 4 * 10240 + M * 5120 + 4 * M + 2 * M * 10240
    dense_o = 5120 * 8192 + 4 * 5120 + M * 8192 + 4 * M + 2 * M * 5120
    assert bench.step_bytes(args, dense=True) == dense_qkv + dense_o


def test_stale_traffic_record_is_not_reported(monkeypatch):
    path = os.path.join(ROOT, "profiles", "spense_gemm_attn32b_m16_traffic.txt")
    with open(path) as f:
        rec = json.load(f)
    per = rec["dram_bytes_per_launch"]
    assert rec["dram_bytes_per_launch_avg"] == sum(per.values()) // len(per)
    monkeypatch.setattr(bench, "kernel_source_sha256", lambda: rec["kernel_source_sha256"])
    assert bench.read_traffic() == rec["dram_bytes_per_launch_avg"]
    monkeypatch.setattr(bench, "kernel_source_sha256", lambda: "0" * 64)
    assert bench.read_traffic() is None


def test_l2_note():
    assert "larger than the 126 MB L2" in bench.l2_note(8, 549e6)
    assert "NOT larger" in bench.l2_note(1, 68e6)


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
    assert line["config"]["workload"].startswith("attn32b")
