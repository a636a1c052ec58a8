"""Pins for the CPU oracle: each test ties the oracle to something other than
itself — values worked by hand from the page, a library routine, brute force
over every small case, or an invariant the method guarantees.

Page: "SpenseGPT: Practical One-shot Pruning Enabling Sparse and Dense GEMMs for
LLM Inference" (gist.science technical summary), Technical Summary §1 (2:4),
§2A (the Spense split and input-split accumulation), §2B (tail and
score-selected dense sets, permutation invariance), §4 (FP8).
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle
from dense_fp8_gemm_b200 import synth


def _torch_decode(b):
    return torch.from_numpy(np.asarray(b, np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


# --------------------------------------------------------------------------- e4m3


def test_e4m3_table_matches_torch_float8():
    """Decode of all 256 bytes equals torch.float8_e4m3fn (OCP E4M3)."""
    ours = oracle.e4m3_table()
    ref = _torch_decode(np.arange(256, dtype=np.uint8))
    nan_ours = np.isnan(ours)
    np.testing.assert_array_equal(nan_ours, np.isnan(ref))
    np.testing.assert_array_equal(ours[~nan_ours], ref[~nan_ours])
    assert set(np.nonzero(nan_ours)[0].tolist()) == {0x7F, 0xFF}


def test_e4m3_textbook_values():
    t = oracle.e4m3_table()
    assert t[0x00] == 0.0 and np.signbit(t[0x80])
    assert t[0x38] == 1.0 and t[0xB8] == -1.0
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x01] == 2.0 ** -9  # smallest subnormal
    assert t[0x08] == 2.0 ** -6  # smallest normal
    assert t[0x07] == 7 * 2.0 ** -9  # largest subnormal


# --------------------------------------------------------------------------- hand-worked K = 8


@pytest.fixture(scope="module")
def k8(golden_dir):
    with open(os.path.join(golden_dir, "k8_hand.json")) as f:
        return json.load(f)


def test_k8_top2_by_hand(k8):
    c = k8["top2"]
    W = np.array(c["W"], np.uint8)
    X = np.array(c["X"], np.uint8)
    np.testing.assert_array_equal(oracle.decode(W), np.array(c["W_values"]))
    np.testing.assert_array_equal(oracle.decode(X), np.array(c["X_values"]))
    p = oracle.pack(W, Kd=c["Kd"])
    np.testing.assert_array_equal(p["Vs"], np.array(c["Vs"], np.uint8))
    np.testing.assert_array_equal(p["E"], np.array(c["E"], np.uint8))
    np.testing.assert_array_equal(p["Wd"], np.array(c["Wd"], np.uint8))
    for n, (i0, i1) in enumerate(c["kept_sparse_indices"]):
        kept = np.nonzero(p["keep"][n, :4])[0].tolist()
        assert kept == [i0, i1]
    y, b = oracle.gemm(X, np.array(c["s_x"], np.float32), W, np.array(c["s_w"], np.float32),
                       keep=p["keep"])
    np.testing.assert_array_equal(y, np.array(c["y"]))
    np.testing.assert_array_equal(b, np.array(c["bound"]))


def test_k8_mask_by_hand(k8):
    c, m = k8["top2"], k8["mask"]
    W = np.array(c["W"], np.uint8)
    X = np.array(c["X"], np.uint8)
    mask = np.ones_like(W)
    mask[:, :4] = np.array(m["mask_sparse"], np.uint8)
    p = oracle.pack(W, mask=mask, Kd=c["Kd"])
    np.testing.assert_array_equal(p["Vs"], np.array(m["Vs"], np.uint8))
    np.testing.assert_array_equal(p["E"], np.array(m["E"], np.uint8))
    y, b = oracle.gemm(X, np.array(c["s_x"], np.float32), W, np.array(c["s_w"], np.float32),
                       keep=p["keep"])
    np.testing.assert_array_equal(y, np.array(m["y"]))
    np.testing.assert_array_equal(b, np.array(m["bound"]))


# --------------------------------------------------------------------------- selection, brute force

CLASSES = [0x00, 0x38, 0xB8, 0x40, 0x7E]  # 0, 1, -1 (ties with 1), 2, 448


def test_top2_all_magnitude_patterns():
    """All 5^4 patterns: the kept pair is the unique pair that beats every
    dropped entry on (magnitude desc, index asc)."""
    pats = np.array(list(itertools.product(CLASSES, repeat=4)), np.uint8)  # [625, 4]
    p = oracle.pack(pats, Kd=0)
    mag = oracle.decode(pats).__abs__()
    for r in range(pats.shape[0]):
        winners = []
        for pair in itertools.combinations(range(4), 2):
            rest = [j for j in range(4) if j not in pair]
            if all((mag[r, i] > mag[r, j]) or (mag[r, i] == mag[r, j] and i < j)
                   for i in pair for j in rest):
                winners.append(pair)
        assert len(winners) == 1
        assert tuple(np.nonzero(p["keep"][r])[0]) == winners[0]
        i0, i1 = winners[0]
        assert p["E"][r, 0] & 0xF == i0 | (i1 << 2)
        assert p["Vs"][r].tolist() == [pats[r, i0], pats[r, i1]]


def test_every_mask_pattern():
    """All 16 keep patterns of one group: <= 2 kept are stored (padded with the
    lowest unkept index, value 0x00); 3 or 4 kept is rejected."""
    w = np.array([[0x38, 0x40, 0x44, 0x48]], np.uint8)
    for bits in range(16):
        kept = [i for i in range(4) if bits >> i & 1]
        mask = np.array([[bits >> i & 1 for i in range(4)]], np.uint8)
        if len(kept) > 2:
            with pytest.raises(oracle.OracleError) as ei:
                oracle.pack(w, mask=mask, Kd=0)
            assert ei.value.code == oracle.OR_ERR_MASK
            continue
        p = oracle.pack(w, mask=mask, Kd=0)
        pad = [i for i in range(4) if i not in kept][: 2 - len(kept)]
        pair = sorted(kept + pad)
        assert p["E"][0, 0] & 0xF == pair[0] | (pair[1] << 2)
        assert p["Vs"][0].tolist() == [w[0, i] if i in kept else 0 for i in pair]
        assert np.nonzero(p["keep"][0])[0].tolist() == kept


def test_negative_zero_ranks_with_zero():
    w = np.array([[0x80, 0x00, 0x80, 0x00]], np.uint8)
    p = oracle.pack(w, Kd=0)
    assert np.nonzero(p["keep"][0])[0].tolist() == [0, 1]


# --------------------------------------------------------------------------- pack invariants


def _rand_w(seed, N, K):
    q, s = synth.quantize_rows(synth.normal(seed, 1, (N, K), 0.02))
    return q, s


@pytest.mark.parametrize("scattered", [False, True])
@pytest.mark.parametrize("use_mask", [False, True])
def test_unpack_of_pack_is_masked_w(scattered, use_mask):
    N, K, Kd = 24, 96, 32
    W, _ = _rand_w(7, N, K)
    idx = synth.scored_dense_idx(7, 2, K, Kd) if scattered else None
    sparse_cols = np.setdiff1d(np.arange(K), idx) if scattered else np.arange(K - Kd)
    mask = synth.random_mask(7, 3, N, K, (0, 1, 2), sparse_cols) if use_mask else None
    p = oracle.pack(W, mask=mask, dense_idx=idx, Kd=Kd)
    Wm = oracle.unpack(p["Vs"], p["E"], p["Wd"], K, dense_idx=idx)
    np.testing.assert_array_equal(Wm, np.where(p["keep"] != 0, W, 0).astype(np.uint8))
    dense_cols = idx if scattered else np.arange(K - Kd, K)
    assert np.all(p["keep"][:, dense_cols] == 1)
    groups = p["keep"][:, sparse_cols].reshape(N, -1, 4).sum(axis=2)
    if use_mask:
        np.testing.assert_array_equal(p["keep"][:, sparse_cols], mask[:, sparse_cols])
        assert groups.max() <= 2
    else:
        assert np.all(groups == 2)
    # every 4-group of the unpacked sparse region has at most two nonzeros
    nz = (Wm[:, sparse_cols] & 0x7F) != 0
    assert nz.reshape(N, -1, 4).sum(axis=2).max() <= 2
    # metadata nibbles are valid ordered pairs
    nib = np.stack([p["E"] & 0xF, p["E"] >> 4], axis=2).reshape(N, -1)
    assert set(np.unique(nib).tolist()) <= {0x4, 0x8, 0xC, 0x9, 0xD, 0xE}


def test_tail_index_list_equals_default():
    """SpenseGPT+ with the tail as its index set is SpenseGPT (§2B)."""
    N, K, Kd = 16, 64, 16
    W, _ = _rand_w(8, N, K)
    a = oracle.pack(W, Kd=Kd)
    b = oracle.pack(W, dense_idx=np.arange(K - Kd, K), Kd=Kd)
    for key in ("Vs", "E", "Wd", "keep"):
        np.testing.assert_array_equal(a[key], b[key])


def test_dense_idx_rejected():
    W, _ = _rand_w(9, 4, 32)
    for bad in ([3, 2, 5, 6], [1, 1, 2, 3], [0, 1, 2, 32], [-1, 0, 1, 2]):
        with pytest.raises(oracle.OracleError) as ei:
            oracle.pack(W, dense_idx=np.array(bad), Kd=4)
        assert ei.value.code == oracle.OR_ERR_DENSE_IDX


def test_nan_rejected():
    W, _ = _rand_w(10, 4, 32)
    W[2, 5] = 0x7F
    with pytest.raises(oracle.OracleError) as ei:
        oracle.pack(W, Kd=8)
    assert ei.value.code == oracle.OR_ERR_NONFINITE


# --------------------------------------------------------------------------- tiled storage


def test_tile_is_a_bijection_with_defined_padding():
    """Every canonical byte appears exactly once in the tiled arrays, padding
    holds the defined fill, and each 8-row x 128-byte swizzle atom permutes the
    16-byte chunks of a row by XOR with the row index."""
    N, K, Kd = 200, 640, 160  # ragged N (2 tiles), ragged sparse (480 -> 2 blocks) and dense (160 -> 2 blocks)
    Ks = K - Kd
    W, _ = _rand_w(11, N, K)
    p = oracle.pack(W, Kd=Kd)
    t = oracle.tile(p["Vs"], p["E"], p["Wd"], N, Ks, Kd)
    nt, nsb, ndb = 2, 2, 2
    vs = t["Vs_t"].reshape(nt, nsb, 128, 8, 16)
    # undo the swizzle by chunk index arithmetic (XOR is its own inverse)
    r = np.arange(128)[:, None]
    c = np.arange(8)[None, :]
    phys = c ^ (r % 8)
    un = vs[:, :, r, phys, :]  # [nt, nsb, 128, 8, 16] logical order
    rows = un.transpose(0, 2, 1, 3, 4).reshape(nt * 128, nsb * 128)
    np.testing.assert_array_equal(rows[:N, : Ks // 2], p["Vs"])
    assert np.all(rows[N:] == 0) and np.all(rows[:, Ks // 2:] == 0)
    e = t["E_t"].reshape(nt, nsb, 2, 128, 16).transpose(0, 3, 1, 2, 4).reshape(nt * 128, nsb * 32)
    np.testing.assert_array_equal(e[:N, : Ks // 8], p["E"])
    assert np.all(e[N:] == 0x44) and np.all(e[:, Ks // 8:] == 0x44)
    wd = t["Wd_t"].reshape(nt, ndb, 128, 8, 16)[:, :, r, phys, :]
    wd = wd.transpose(0, 2, 1, 3, 4).reshape(nt * 128, ndb * 128)
    np.testing.assert_array_equal(wd[:N, :Kd], p["Wd"])
    assert np.all(wd[N:] == 0) and np.all(wd[:, Kd:] == 0)


# --------------------------------------------------------------------------- GEMM


def _case(seed, M, N, K):
    X, s_x = synth.quantize_rows(synth.normal(seed, 20, (M, K), 1.0))
    W, s_w = synth.quantize_rows(synth.normal(seed, 21, (N, K), 0.02))
    return X, s_x, W, s_w


def _matmul_ref(X, s_x, Wm, s_w):
    xd = torch.from_numpy(_torch_decode(X))
    wd = torch.from_numpy(_torch_decode(Wm))
    y = (xd @ wd.T) * torch.from_numpy(s_x.astype(np.float64))[:, None] \
        * torch.from_numpy(s_w.astype(np.float64))[None, :]
    return y.numpy()


def test_dense_frac_one_is_plain_dense_gemm():
    X, s_x, W, s_w = _case(12, 5, 40, 256)
    p = oracle.pack(W, Kd=256)
    assert np.all(p["keep"] == 1)
    y, _ = oracle.gemm(X, s_x, W, s_w, keep=p["keep"])
    np.testing.assert_allclose(y, _matmul_ref(X, s_x, W, s_w), rtol=1e-12, atol=1e-12)


def test_dense_frac_zero_is_pure_24_gemm():
    X, s_x, W, s_w = _case(13, 3, 32, 256)
    p = oracle.pack(W, Kd=0)
    assert np.all(p["keep"].reshape(32, 64, 4).sum(axis=2) == 2)
    Wm = oracle.unpack(p["Vs"], p["E"], p["Wd"], 256)
    y, _ = oracle.gemm(X, s_x, W, s_w, keep=p["keep"])
    np.testing.assert_allclose(y, _matmul_ref(X, s_x, Wm, s_w), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("scattered", [False, True])
def test_hybrid_equals_dense_gemm_on_masked_matrix(scattered):
    M, N, K, Kd = 7, 48, 320, 80
    X, s_x, W, s_w = _case(14, M, N, K)
    idx = synth.scored_dense_idx(14, 3, K, Kd) if scattered else None
    p = oracle.pack(W, dense_idx=idx, Kd=Kd)
    Wm = oracle.unpack(p["Vs"], p["E"], p["Wd"], K, dense_idx=idx)
    y, b = oracle.gemm(X, s_x, W, s_w, keep=p["keep"])
    np.testing.assert_allclose(y, _matmul_ref(X, s_x, Wm, s_w), rtol=1e-12, atol=1e-12)
    # the bound is the same sum over absolute products
    babs = np.abs(_torch_decode(X)) @ np.abs(_torch_decode(Wm)).T * np.abs(s_x)[:, None] * np.abs(s_w)[None, :]
    np.testing.assert_allclose(b, babs, rtol=1e-12, atol=1e-12)


def test_permuting_columns_leaves_output_unchanged():
    """§2B: permuting the intermediate indices of W and X together does not
    change Y."""
    M, N, K, Kd = 4, 24, 128, 32
    X, s_x, W, s_w = _case(15, M, N, K)
    p = oracle.pack(W, Kd=Kd)
    perm = synth.rng(15, 9).permutation(K)
    y0, _ = oracle.gemm(X, s_x, W, s_w, keep=p["keep"])
    y1, _ = oracle.gemm(X[:, perm], s_x, W[:, perm], s_w, keep=p["keep"][:, perm])
    np.testing.assert_allclose(y1, y0, rtol=1e-12, atol=1e-14)


def test_row_subset_and_threads_agree():
    M, N, K = 3, 64, 256
    X, s_x, W, s_w = _case(16, M, N, K)
    keep = oracle.pack(W, Kd=64)["keep"]
    y_all, b_all = oracle.gemm(X, s_x, W, s_w, keep=keep, nthreads=1)
    rows = np.array([63, 0, 17, 17, 40])
    y_sub, b_sub = oracle.gemm(X, s_x, W, s_w, keep=keep, rows=rows, nthreads=4)
    np.testing.assert_array_equal(y_sub, y_all[:, rows])
    np.testing.assert_array_equal(b_sub, b_all[:, rows])


def test_tolerance_rule_accepts_bf16_rounding_and_rejects_a_dropped_term():
    """The acceptance rule admits bf16 rounding of the exact result and flags
    the loss of one product."""
    M, N, K, Kd = 4, 32, 256, 64
    X, s_x, W, s_w = _case(17, M, N, K)
    p = oracle.pack(W, Kd=Kd)
    y, b = oracle.gemm(X, s_x, W, s_w, keep=p["keep"])
    ybf = torch.from_numpy(y).to(torch.bfloat16).to(torch.float64).numpy()
    assert oracle.within_tolerance(ybf, y, b).all()
    keep2 = p["keep"].copy()
    keep2[:, K - 1] = 0  # drop the last dense column
    y2, _ = oracle.gemm(X, s_x, W, s_w, keep=keep2)
    assert not oracle.within_tolerance(y2, y, b).all()
