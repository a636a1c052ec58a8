"""Pins for the oracle's output-split keep mask and GLU index order (CPU only).

Fixed independently of the oracle's code:
- an output-split weight with every row dense is a plain dense GEMM, and with
  no dense row it is the pure 2:4 GEMM over all columns;
- the rows are independent: a dense row keeps all K entries, a sparse row keeps
  exactly two of every four and the same two as when it is packed alone;
- the GLU order is a permutation that puts the dense indices last, and
  permuting the intermediate indices of gate/up rows and down columns together
  leaves the MLP output unchanged (checked with float64 matmuls on the decoded
  tensors and an elementwise activation).
"""
import numpy as np
import pytest

import oracle
from dense_fp8_gemm_b200 import synth


def weights(seed, N, K):
    W, s = synth.quantize_rows(synth.normal(seed, 1, (N, K), 0.02))
    return W, s


def test_all_dense_rows_is_a_dense_gemm_and_no_dense_row_is_pure_24():
    W, s_w = weights(1, 24, 64)
    X, s_x = synth.quantize_rows(synth.normal(1, 2, (3, 64), 1.0))
    keep_all = oracle.output_split_keep(W, np.arange(24))
    assert keep_all.all()
    y_dense, _ = oracle.gemm(X, s_x, W, s_w)
    y_split, _ = oracle.gemm(X, s_x, W, s_w, keep=keep_all)
    assert np.array_equal(y_dense, y_split)
    keep_none = oracle.output_split_keep(W, np.array([], np.int64))
    assert np.array_equal(keep_none, oracle.pack(W, Kd=0)["keep"])


def test_rows_are_independent():
    W, _ = weights(2, 40, 128)
    dense_rows = np.array([0, 7, 8, 31, 39])
    keep = oracle.output_split_keep(W, dense_rows)
    for n in range(40):
        if n in dense_rows:
            assert keep[n].all()
        else:
            assert (keep[n].reshape(-1, 4).sum(1) == 2).all()
            assert np.array_equal(keep[n], oracle.pack(W[n:n + 1], Kd=0)["keep"][0])


def test_glu_order_and_invariance():
    I, H, M = 48, 32, 4
    d = np.array([3, 10, 11, 40, 47])
    pi = oracle.glu_order(I, d)
    assert sorted(pi.tolist()) == list(range(I))
    assert pi[-len(d):].tolist() == d.tolist()
    assert np.all(np.diff(pi[:-len(d)]) > 0)
    g = np.random.default_rng(0)
    table = oracle.e4m3_table()
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    dec = lambda a: table[a]
    gate, up = dec(g.choice(finite, (I, H))), dec(g.choice(finite, (I, H)))
    down = dec(g.choice(finite, (H, I)))
    x = g.standard_normal((M, H))
    act = lambda a, b: a / (1 + np.exp(-np.clip(a, -50, 50))) * b
    y = act(x @ gate.T, x @ up.T) @ down.T
    y_perm = act(x @ gate[pi].T, x @ up[pi].T) @ down[:, pi].T
    assert np.allclose(y, y_perm, rtol=1e-12, atol=1e-9 * np.abs(y).max())
