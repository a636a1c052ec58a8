"""The allocation-free entry point, spense_gemm_noalloc, against spense_gemm.

Some callers cannot allocate device memory when they run the GEMM (an engine
that owns every allocation and gives plugins none, or a serving loop that bans
cudaMalloc after start-up), so they cannot pass a workspace. spense_gemm_noalloc
uses the library's own fixed scratch array instead. This test calls it through
the C ABI twice in a row (the second call finds the first call's leftovers in
the shared array) and checks both outputs bit for bit against the workspace
entry point (the same plan and kernel) and against the oracle within the
parity tolerance, and that the calls leave the device's free memory
unchanged. It runs last so that a failure here never hides the result of
another test, and it works alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
from dense_fp8_gemm_b200 import spense, synth

pytestmark = pytest.mark.gpu

CASES = [
    # M, N, K, Kd, scattered
    (8, 256, 512, 128, False),
    (16, 8192, 5120, 1280, False),     # q_proj at decode: tiles shared by several CTAs
    (24, 8192, 5120, 1280, False),     # q_proj, 24 tokens: the largest plan of the 32B shapes
    (1, 1024, 5120, 1280, False),
    (24, 2048, 4096, 1024, True),      # SpenseGPT+ gather into the scratch
]


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("M,N,K,Kd,scattered", CASES)
def test_noalloc_matches_workspace_entry_point(M, N, K, Kd, scattered):
    X, s_x = synth.quantize_rows(synth.normal(900 + M, 1, (M, K), 1.0))
    W, s_w = synth.quantize_rows(synth.normal(900 + M, 2, (N, K), 0.02))
    idx = synth.scored_dense_idx(900 + M, 3, K, Kd) if scattered else None
    pw = spense.pack(_dev(W), _dev(s_w), Kd=Kd, dense_idx=idx)
    Xd, sxd = _dev(X), _dev(s_x)
    Y_ws = spense.gemm(pw, Xd, sxd)  # the existing entry point, with its own workspace
    keep = oracle.pack(W, dense_idx=idx, Kd=Kd)["keep"]
    yref, bound = oracle.gemm(X, s_x, W, s_w, keep=keep)
    assert oracle.within_tolerance(Y_ws.float().cpu().numpy(), yref, bound).all()
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    spense.gemm_noalloc(pw, Xd, sxd, Y)  # first call on this device: looks up the scratch address
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for call in range(2):
        Y.fill_(float("nan"))
        spense.gemm_noalloc(pw, Xd, sxd, Y)
        torch.cuda.synchronize()
        # the same plan and kernel as the workspace entry point: bit for bit the same output
        assert torch.equal(Y.view(torch.int16), Y_ws.view(torch.int16)), f"call {call}: differs from spense_gemm"
        y = Y.float().cpu().numpy().astype(np.float64)
        ok = oracle.within_tolerance(y, yref, bound)
        assert ok.all(), f"call {call}: {int((~ok).sum())} of {ok.size} outputs outside tolerance"
    assert torch.cuda.mem_get_info()[0] == free_before, "device memory was allocated by the noalloc calls"
    assert spense.noalloc_status() == 0
    pw.free()


def test_noalloc_rejects_work_beyond_its_scratch():
    N, K, Kd, M = 8192, 5120, 1280, 256   # fp32 partials for 256 tokens exceed the fixed scratch
    W, s_w = synth.quantize_rows(synth.normal(7, 2, (N, K), 0.02))
    X, s_x = synth.quantize_rows(synth.normal(7, 1, (M, K), 1.0))
    pw = spense.pack(_dev(W), _dev(s_w), Kd=Kd)
    assert spense.workspace_size(pw, M) > spense.NOALLOC_SCRATCH_BYTES
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(spense.SpenseError) as ei:
        spense.gemm_noalloc(pw, _dev(X), _dev(s_x), Y)
    assert ei.value.code == 7
    assert "scratch" in str(ei.value)
    pw.free()
