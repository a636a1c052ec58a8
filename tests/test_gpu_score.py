"""GPU parity of the SpenseGPT+ scorer (spense_score_glu) and the dense-set
selection (spense_select_dense) against the CPU oracle.

Scores are sums of thousands of fp32 terms, so they are compared within a
relative tolerance (the oracle sums in float64). The selection is an integer
decision: run on the GPU's own scores it must equal the oracle's selection on
those same scores exactly; against the oracle's float64 scores it must be a
valid top-Kd (no unselected index scores clearly above a selected one).
"""
import numpy as np
import pytest
import torch

import oracle
from dense_fp8_gemm_b200 import spense, synth

pytestmark = pytest.mark.gpu

RTOL = 5e-5  # fp32 accumulation of up to ~2 x 25600 positive terms


def mlp(seed, I, H, gate=True, up=True):
    g = np.random.default_rng(seed)
    out = {}
    if gate:
        out["gate"], out["s_gate"] = synth.quantize_rows(synth.normal(seed, 1, (I, H), 0.02))
    if up:
        out["up"], out["s_up"] = synth.quantize_rows(synth.normal(seed, 2, (I, H), 0.02))
    out["down"], out["s_down"] = synth.quantize_rows(synth.normal(seed, 3, (H, I), 0.02))
    # synthetic Hessian diagonals: sums of squares of seeded calibration activations
    out["h_in"] = (g.standard_normal((8, H)).astype(np.float32) ** 2).sum(0) * np.float32(1.0 + g.random())
    out["h_mid"] = (g.standard_normal((8, I)).astype(np.float32) ** 2).sum(0)
    return out


def gpu_scores(m):
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in m.items()}
    sc = spense.score_glu(t["down"], t["s_down"], t["h_in"], t["h_mid"], gate=t.get("gate"), s_gate=t.get("s_gate"),
                          up=t.get("up"), s_up=t.get("s_up"))
    torch.cuda.synchronize()
    return sc


def oracle_scores(m):
    return oracle.score_glu(m["down"], m["s_down"], m["h_in"], m["h_mid"], gate=m.get("gate"),
                            s_gate=m.get("s_gate"), up=m.get("up"), s_up=m.get("s_up"))


@pytest.mark.parametrize("I,H,gate,up", [(64, 32, True, True), (256, 128, True, True), (1040, 512, True, False),
                                         (512, 256, False, True), (4096, 1024, False, False),
                                         (25600, 5120, True, True)])
def test_scores_match_oracle(I, H, gate, up):
    m = mlp(I + H, I, H, gate, up)
    got = gpu_scores(m).cpu().numpy().astype(np.float64)
    ref = oracle_scores(m)
    rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
    assert rel.max() <= RTOL, (rel.max(), int(rel.argmax()))


def test_scores_are_repeatable_bit_for_bit():
    m = mlp(7, 2048, 1024)
    a = gpu_scores(m)
    b = gpu_scores(m)
    assert torch.equal(a, b)


@pytest.mark.parametrize("I,frac", [(25600, 0.25), (27648, 0.125), (1040, 0.5), (2000, 1.0), (16, 0.0)])
def test_selection_of_gpu_scores_equals_oracle_selection(I, frac):
    H = 512 if I > 5000 else 256
    m = mlp(I, I, H)
    sc = gpu_scores(m)
    Kd = int(round(frac * I))
    got = spense.select_dense(sc, Kd).cpu().numpy()
    sc64 = sc.cpu().numpy().astype(np.float64)
    assert np.array_equal(got, oracle.select_top(sc64, Kd))
    # valid against the oracle's own float64 scores: no unselected index above a selected one beyond tolerance
    ref = oracle_scores(m)
    if 0 < Kd < I:
        sel = np.zeros(I, bool)
        sel[got] = True
        assert ref[sel].min() >= ref[~sel].max() * (1 - 2 * RTOL)


@pytest.mark.parametrize("I,Kd", [(1, 1), (1000, 333), (4097, 4096), (3000, 1500), (60000, 15000)])
def test_selection_with_ties_and_ragged_sizes(I, Kd):
    g = np.random.default_rng(I)
    sc = g.integers(0, 7, size=I).astype(np.float32)      # heavy ties
    got = spense.select_dense(torch.from_numpy(sc).cuda(), Kd).cpu().numpy()
    assert np.array_equal(got, oracle.select_top(sc.astype(np.float64), Kd))


def test_selected_set_drives_a_spenseplus_gemm():
    """The GPU-selected dense set packs and runs: Y matches the oracle GEMM."""
    I, H, M = 2048, 512, 8
    m = mlp(3, I, H)
    Kd = I // 4
    dense_idx = spense.select_dense(gpu_scores(m), Kd).cpu().numpy()
    W, s_w = m["down"], m["s_down"]
    pw = spense.pack(torch.from_numpy(W).cuda(), torch.from_numpy(s_w).cuda(), Kd=Kd, dense_idx=dense_idx)
    X, s_x = synth.quantize_rows(synth.normal(3, 9, (M, I), 1.0))
    Y = spense.gemm(pw, torch.from_numpy(X).cuda(), torch.from_numpy(s_x).cuda())
    torch.cuda.synchronize()
    keep = oracle.pack(W, dense_idx=dense_idx)["keep"]
    yref, bound = oracle.gemm(X, s_x, W, s_w, keep=keep)
    assert oracle.within_tolerance(Y.float().cpu().numpy(), yref, bound).all()
    pw.free()
