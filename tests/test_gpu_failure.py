"""Failure detection on the GPU without a fault: every wait in the GEMM kernel
is bounded. The test build of the library (libspense_testhooks.so, selected by
SPENSE_TEST_HOOKS=1; the product library has no such hook) reads
SPENSE_TEST_STALL=1 and makes the loader warps wait on a workspace word that
nothing sets; the kernel must give up after its time limit, record the timeout
in the status word, leave no copy in flight and return, and the CUDA context
must stay usable. The knob is read once per process, so each check runs in a
child process.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import time, torch
from dense_fp8_gemm_b200 import spense, synth
W, s_w = synth.quantize_rows(synth.normal(3, 1, (256, 512), 0.02))
X, s_x = synth.quantize_rows(synth.normal(3, 2, (8, 512), 1.0))
pw = spense.pack(torch.from_numpy(W).cuda(), torch.from_numpy(s_w).cuda(), Kd=128)
ws = spense.new_workspace(spense.workspace_size(pw, 8))
t0 = time.time()
spense.gemm(pw, torch.from_numpy(X).cuda(), torch.from_numpy(s_x).cuda(), workspace=ws)
torch.cuda.synchronize()
elapsed = time.time() - t0
status = spense.workspace_status(ws)
again = spense.workspace_status(ws)          # reading clears it
usable = float((torch.ones(1024, device="cuda") * 2).sum().item())
print("RESULT", status, again, usable, round(elapsed, 2))
"""


def test_stalled_loaders_time_out_and_report():
    env = dict(os.environ, SPENSE_TEST_STALL="1", SPENSE_TEST_HOOKS="1")
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT")][-1].split()
    status, again, usable, elapsed = int(line[1]), int(line[2]), float(line[3]), float(line[4])
    assert status & 0x1, f"no producer timeout recorded (status {status:#x})"
    assert status & ~0x7 == 0
    assert again == 0
    assert usable == 2048.0
    assert elapsed < 60.0


CHILD_NOALLOC = r"""
import time, torch
from dense_fp8_gemm_b200 import spense, synth
W, s_w = synth.quantize_rows(synth.normal(3, 1, (256, 512), 0.02))
X, s_x = synth.quantize_rows(synth.normal(3, 2, (8, 512), 1.0))
pw = spense.pack(torch.from_numpy(W).cuda(), torch.from_numpy(s_w).cuda(), Kd=128)
Y = torch.empty((8, 256), dtype=torch.bfloat16, device="cuda")
before = spense.noalloc_status()
spense.gemm_noalloc(pw, torch.from_numpy(X).cuda(), torch.from_numpy(s_x).cuda(), Y)
torch.cuda.synchronize()
status = spense.noalloc_status()
again = spense.noalloc_status()              # reading clears it
usable = float((torch.ones(1024, device="cuda") * 2).sum().item())
print("RESULT", before, status, again, usable, spense.lib_path().endswith("libspense_testhooks.so"))
"""


def test_noalloc_timeout_is_reported():
    """A wait that gives up inside spense_gemm_noalloc is recorded in the
    scratch array's status word and read back by spense_noalloc_status."""
    env = dict(os.environ, SPENSE_TEST_STALL="1", SPENSE_TEST_HOOKS="1")
    r = subprocess.run([sys.executable, "-c", CHILD_NOALLOC], env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT")][-1].split()
    before, status, again, usable, hooked = int(line[1]), int(line[2]), int(line[3]), float(line[4]), line[5]
    assert hooked == "True"
    assert before == 0
    assert status & 0x1, f"no producer timeout recorded (status {status:#x})"
    assert status & ~0x7 == 0
    assert again == 0
    assert usable == 2048.0
