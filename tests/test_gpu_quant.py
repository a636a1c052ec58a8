"""GPU parity of spense_quantize (per-token FP8 quantisation with the packed
column order fused in) against the CPU oracle: codes and scales bit-exact.
The quantisation decides integers (codes) from floating point, so both sides
decide in the same precision (IEEE fp32, one rounding per operation)."""
import numpy as np
import pytest
import torch

import oracle
from dense_fp8_gemm_b200 import spense, synth

pytestmark = pytest.mark.gpu


def bf16_bits(x):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def activations(seed, M, K):
    g = np.random.default_rng(seed)
    x = g.standard_normal((M, K)).astype(np.float32) * np.float32(10.0) ** g.integers(-4, 5, size=(M, 1))
    if M > 2:
        x[1, :] = 0.0                                         # all-zero row
        x[2, g.integers(0, K)] = 3e4                          # one outlier sets the scale
    if M > 3:
        x[3, :] = np.float32(1e-36) * np.sign(x[3, :])        # subnormal codes and signed zeros
    return bf16_bits(x)


def run(bits, order=None):
    X = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    Xq, s = spense.quantize(X, order=order)
    torch.cuda.synchronize()
    return Xq.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("M,K", [(1, 16), (4, 512), (7, 1040), (16, 5120), (33, 8192), (300, 2048)])
def test_quantize_matches_oracle(M, K):
    bits = activations(M * 7 + K, M, K)
    q, s = run(bits)
    oq, os_ = oracle.quantize(bits)
    assert np.array_equal(s, os_)
    assert np.array_equal(q, oq)


def packed_with_dense_set(K, Kd, seed):
    W, s_w = synth.quantize_rows(synth.normal(seed, 1, (128, K), 0.02))
    dense_idx = np.sort(np.random.default_rng(seed).choice(K, Kd, replace=False)).astype(np.int32)
    pw = spense.pack(torch.from_numpy(W).cuda(), torch.from_numpy(s_w).cuda(), Kd=Kd, dense_idx=dense_idx)
    return pw, dense_idx, W, s_w


@pytest.mark.parametrize("M,K,Kd", [(5, 512, 128), (16, 5120, 1280), (32, 25600, 3200), (3, 65536, 16384)])
def test_quantize_in_packed_order_matches_oracle(M, K, Kd):
    pw, dense_idx, _, _ = packed_with_dense_set(K, Kd, 11)
    bits = activations(3 + M, M, K)
    q, s = run(bits, order=pw)
    oq, os_ = oracle.quantize(bits, dense_idx=dense_idx)
    assert np.array_equal(s, os_)
    assert np.array_equal(q, oq)
    pw.free()


def test_tail_order_is_the_identity():
    W, s_w = synth.quantize_rows(synth.normal(2, 1, (128, 1024), 0.02))
    pw = spense.pack(torch.from_numpy(W).cuda(), torch.from_numpy(s_w).cuda(), Kd=256)
    bits = activations(9, 6, 1024)
    q0, s0 = run(bits)
    q1, s1 = run(bits, order=pw)
    assert np.array_equal(q0, q1) and np.array_equal(s0, s1)
    pw.free()


def test_full_size_down_projection_sampled_rows():
    M, K = 256, 25600
    bits = activations(21, M, K)
    q, s = run(bits)
    rows = np.array([0, 1, 2, 3, 127, 128, 200, 255])
    oq, os_ = oracle.quantize(bits[rows])
    assert np.array_equal(s[rows], os_)
    assert np.array_equal(q[rows], oq)


def test_fused_order_feeds_the_gemm_without_its_gather():
    """quantize(order=W) + GEMM with SPENSE_GEMM_X_PACKED_ORDER gives bitwise the
    same Y as quantize() + the GEMM's own gather, and Y is within the tolerance
    of the oracle GEMM on the quantised input."""
    M, K, Kd = 16, 2048, 512
    pw, dense_idx, W, s_w = packed_with_dense_set(K, Kd, 4)
    bits = activations(5, M, K)
    X = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    Xq, sx = spense.quantize(X)
    Xo, sxo = spense.quantize(X, order=pw)
    ws = spense.new_workspace(spense.workspace_size(pw, M))
    Y1 = spense.gemm(pw, Xq, sx, workspace=ws)
    Y2 = spense.gemm_grouped([pw], Xo, sxo, workspace=ws, flags=spense.GEMM_X_PACKED_ORDER)[0]
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    assert spense.workspace_status(ws) == 0
    keep = oracle.pack(W, dense_idx=dense_idx)["keep"]
    yref, bound = oracle.gemm(Xq.cpu().numpy(), sx.cpu().numpy(), W, s_w, keep=keep)
    assert oracle.within_tolerance(Y1.float().cpu().numpy(), yref, bound).all()
    pw.free()


def test_empty_input_is_a_no_op():
    X = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    Xq, s = spense.quantize(X)
    assert Xq.shape == (0, 64) and s.shape == (0,)
