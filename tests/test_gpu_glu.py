"""GPU parity of the output-split execution and of the GLU policy with the
SpenseGPT+ permutation folded upstream (Technical Summary §2A, §2B).

- Output-split: the 2:4 rows (packed with Kd = 0) and the dense rows (Kd = K)
  of a weight run as members of one launch, writing column slices of one Y;
  Y equals the oracle's output-split GEMM element by element (tolerance).
- GLU policy: gate and up output-split (four members, one launch), down
  input-split with a scattered dense set. Folding the permutation: gate and
  up rows are packed in the GLU order (sparse indices, then dense ones), so
  their outputs arrive permuted and down runs without its gather. The order
  comes from the library (spense_glu_order); the oracle only checks results.
"""
import numpy as np
import pytest
import torch

import oracle
from dense_fp8_gemm_b200 import spense, synth

pytestmark = pytest.mark.gpu


def check(Y, X, s_x, W, s_w, keep):
    yref, bound = oracle.gemm(X, s_x, W, s_w, keep=keep)
    ok = oracle.within_tolerance(Y, yref, bound)
    assert ok.all(), f"{(~ok).sum()} of {ok.size} outside the tolerance"


def dense_rows_for(N, frac, seed):
    nd = int(round(frac * N / 8)) * 8
    return np.sort(np.random.default_rng(seed).choice(N, nd, replace=False))


@pytest.mark.parametrize("N,K,M,frac", [(256, 512, 8, 0.25), (1000, 1024, 5, 0.5), (4096, 2048, 16, 0.25),
                                        (51200, 1024, 16, 0.25), (384, 768, 300, 0.125)])
def test_output_split_matches_oracle(N, K, M, frac):
    W, s_w = synth.quantize_rows(synth.normal(N, 1, (N, K), 0.02))
    X, s_x = synth.quantize_rows(synth.normal(N, 2, (M, K), 1.0))
    dense_rows = dense_rows_for(N, frac, N)
    order = spense.glu_order(N, dense_rows)           # sparse rows, then dense rows (the library's order)
    Ns = N - dense_rows.size
    Wd, sd = torch.from_numpy(W).cuda(), torch.from_numpy(s_w).cuda()
    sp = spense.pack(Wd, sd, Kd=0, rows=order[:Ns])
    dn = spense.pack(Wd, sd, Kd=K, rows=order[Ns:])
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    spense.gemm_grouped([sp, dn], torch.from_numpy(X).cuda(), torch.from_numpy(s_x).cuda(), Ys=[Y[:, :Ns], Y[:, Ns:]])
    torch.cuda.synchronize()
    y = np.empty((M, N))
    y[:, order] = Y.float().cpu().numpy()              # back to the original row order
    check(y, X, s_x, W, s_w, oracle.output_split_keep(W, dense_rows))
    sp.free()
    dn.free()


def test_misaligned_output_slice_is_rejected():
    W, s_w = synth.quantize_rows(synth.normal(1, 1, (64, 256), 0.02))
    Wd, sd = torch.from_numpy(W).cuda(), torch.from_numpy(s_w).cuda()
    a = spense.pack(Wd, sd, Kd=0, rows=np.arange(60))
    b = spense.pack(Wd, sd, Kd=256, rows=np.arange(60, 64))
    X, s_x = synth.quantize_rows(synth.normal(1, 2, (4, 256), 1.0))
    Y = torch.empty((4, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(spense.SpenseError):
        # the dense slice starts 60 bf16 = 120 bytes in: not 16-byte aligned
        spense.gemm_grouped([a, b], torch.from_numpy(X).cuda(), torch.from_numpy(s_x).cuda(),
                            Ys=[Y[:, :60], Y[:, 60:]])
    a.free()
    b.free()


@pytest.mark.parametrize("I,H,M", [(2048, 512, 16), (25600, 5120, 16)])
def test_glu_policy_with_the_permutation_folded_upstream(I, H, M):
    g = np.random.default_rng(I)
    gate, s_gate = synth.quantize_rows(synth.normal(7, 1, (I, H), 0.02))
    up, s_up = synth.quantize_rows(synth.normal(7, 2, (I, H), 0.02))
    down, s_down = synth.quantize_rows(synth.normal(7, 3, (H, I), 0.02))
    x, s_x = synth.quantize_rows(synth.normal(7, 4, (M, H), 1.0))
    Nd = I // 4
    D = np.sort(g.choice(I, Nd, replace=False)).astype(np.int32)   # the SpenseGPT+ dense set
    pi = spense.glu_order(I, D)                      # the library's GLU order
    Ns = I - Nd
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    # gate and up: output-split, rows in the GLU order (dense rows last); one launch of four members
    mem = [spense.pack(dev(gate), dev(s_gate), Kd=0, rows=pi[:Ns]), spense.pack(dev(gate), dev(s_gate), Kd=H, rows=pi[Ns:]),
           spense.pack(dev(up), dev(s_up), Kd=0, rows=pi[:Ns]), spense.pack(dev(up), dev(s_up), Kd=H, rows=pi[Ns:])]
    G = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    U = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    spense.gemm_grouped(mem, dev(x), dev(s_x), Ys=[G[:, :Ns], G[:, Ns:], U[:, :Ns], U[:, Ns:]])
    torch.cuda.synchronize()
    # stage 1 against the oracle (output-split on the original row order)
    for Yp, W, s in ((G, gate, s_gate), (U, up, s_up)):
        y = np.empty((M, I))
        y[:, pi] = Yp.float().cpu().numpy()
        check(y, x, s_x, W, s, oracle.output_split_keep(W, D))
    # the activation between the GEMMs (outside this library), then the fused quantisation
    h = (torch.nn.functional.silu(G.float()) * U.float()).to(torch.bfloat16)     # already in GLU order
    hq, sh = spense.quantize(h)
    # down: input-split with the dense set D; its packed column order is pi, which is the order h arrives in,
    # so the GEMM skips its gather
    dn = spense.pack(dev(down), dev(s_down), Kd=Nd, dense_idx=D)
    Yd = spense.gemm_grouped([dn], hq, sh, flags=spense.GEMM_X_PACKED_ORDER)[0]
    torch.cuda.synchronize()
    h_orig = np.empty((M, I), np.uint8)
    h_orig[:, pi] = hq.cpu().numpy()                  # the same codes in the original index order
    keep = oracle.pack(down, dense_idx=D)["keep"]
    check(Yd.float().cpu().numpy(), h_orig, sh.cpu().numpy(), down, s_down, keep)
    for p in mem + [dn]:
        p.free()
