"""The committed ncu summaries stay reproducible: each gives the command that
made it, every such command leaves the GPU clocks alone (`--clock-control
none`), and the program it profiles is a committed file of this repository
(a module of the package or a script at the root), run with options that
program accepts.
"""
import glob
import json
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUMMARIES = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))


def commands(path):
    text = open(path).read()
    blocks = re.findall(r"```\n(.*?)```", text, re.S)
    cmds = []
    for b in blocks:
        joined = re.sub(r"\\\n\s*", " ", b)
        cmds += [ln.strip() for ln in joined.splitlines() if ln.strip().startswith("ncu ")]
    return cmds


@pytest.mark.parametrize("path", SUMMARIES, ids=os.path.basename)
def test_summary_command_is_reproducible(path):
    cmds = commands(path)
    assert cmds, "no ncu command recorded"
    for cmd in cmds:
        assert "--clock-control none" in cmd
        m = re.search(r"\bpython (-m ([\w.]+)|([\w/]+\.py))(.*)$", cmd)
        assert m, cmd
        if m.group(2):
            target = os.path.join(ROOT, *m.group(2).split(".")) + ".py"
        else:
            target = os.path.join(ROOT, m.group(3))
        assert os.path.isfile(target), target
        source = open(target).read()
        for opt in re.findall(r"(--[a-z][\w-]*)", m.group(4)):
            assert f'"{opt}"' in source, f"{opt} is not an option of {os.path.basename(target)}"


TRAFFIC = sorted(glob.glob(os.path.join(ROOT, "profiles", "*_traffic.txt")))


@pytest.mark.parametrize("path", TRAFFIC, ids=os.path.basename)
def test_traffic_record_names_its_sources(path):
    rec = json.load(open(path))
    assert re.fullmatch(r"[0-9a-f]{64}", rec["kernel_source_sha256"])
    for name in rec["kernel_sources"]:
        assert os.path.isfile(os.path.join(ROOT, "dense_fp8_gemm_b200", "csrc", name)), name
    per = rec["dram_bytes_per_launch"]
    assert rec["dram_bytes_per_launch_avg"] == sum(per.values()) // len(per) > 0
    assert "--clock-control none" in rec["source"]


def test_bench_workloads_have_a_traffic_record():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    names = {os.path.basename(p) for p in TRAFFIC}
    for wl in bench.STACKS:
        assert f"spense_gemm_{wl}_m16_traffic.txt" in names
