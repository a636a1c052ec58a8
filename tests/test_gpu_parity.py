"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Packing is compared byte for byte (tiled storage and canonical arrays); the
GEMM output must satisfy |y - y_ref| <= 4e-3 |y_ref| + 1e-5 sum_k |w_k x_k|
on every element the oracle computes (all of them for small cases, sampled
rows spanning every region of the tile grid for the full-size workloads).
"""
import numpy as np
import pytest
import torch

import oracle
from dense_fp8_gemm_b200 import spense, synth, workloads

pytestmark = pytest.mark.gpu

REL, ABS = 4e-3, 1e-5


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.cuda() if dtype is None else t.to(dtype).cuda()


def _assert_close(y_gpu, yref, bound, what=""):
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    ok = oracle.within_tolerance(y, yref, bound, REL, ABS)
    if not ok.all():
        bad = np.argwhere(~ok)
        i, j = bad[0]
        raise AssertionError(
            f"{what}: {len(bad)} of {ok.size} outside tolerance; first at {tuple(bad[0])}: "
            f"gpu {y[i, j]!r} ref {yref[i, j]!r} bound {bound[i, j]!r}")


def _make(seed, M, N, K, Kd, scattered=False, w_std=0.02):
    X, s_x = synth.quantize_rows(synth.normal(seed, 1, (M, K), 1.0))
    W, s_w = synth.quantize_rows(synth.normal(seed, 2, (N, K), w_std))
    idx = synth.scored_dense_idx(seed, 3, K, Kd) if scattered else None
    return X, s_x, W, s_w, idx


def _run(pw, X, s_x):
    Xd, sxd = _dev(X), _dev(s_x)
    ws = spense.new_workspace(spense.workspace_size(pw, X.shape[0]))
    Y = spense.gemm(pw, Xd, sxd, workspace=ws)
    torch.cuda.synchronize()
    assert spense.workspace_status(ws) == 0
    return Y, ws


# --------------------------------------------------------------------------- packing, bit-exact

PACK_CASES = [
    # N, K, Kd, scattered, mask
    (256, 512, 128, False, None),          # the tiny workload
    (200, 640, 160, False, None),          # ragged rows, ragged sparse and dense blocks
    (130, 1024, 0, False, None),           # pure 2:4
    (64, 512, 512, False, None),           # pure dense
    (256, 1024, 336, True, None),          # SpenseGPT+ scattered dense set
    (192, 768, 256, False, (0, 1, 2)),     # explicit masks with 0, 1 or 2 kept
    (160, 896, 224, True, (1, 2)),         # masks over a scattered sparse region
]


@pytest.mark.parametrize("N,K,Kd,scattered,keeps", PACK_CASES)
def test_pack_bit_exact(N, K, Kd, scattered, keeps):
    _, _, W, s_w, idx = _make(100 + N, 1, N, K, Kd, scattered)
    mask = None
    if keeps is not None:
        sparse_cols = np.setdiff1d(np.arange(K), idx) if scattered else np.arange(K - Kd)
        mask = synth.random_mask(100 + N, 7, N, K, keeps, sparse_cols)
    ref = oracle.pack(W, mask=mask, dense_idx=idx, Kd=Kd)
    Ks = K - Kd
    tref = oracle.tile(ref["Vs"], ref["E"], ref["Wd"], N, Ks, Kd)
    pw = spense.pack(_dev(W), _dev(s_w), Kd=Kd, mask=None if mask is None else _dev(mask), dense_idx=idx,
                     keep_canonical=True)
    torch.cuda.synchronize()
    for name, key in (("Vs_t", "Vs_t"), ("E_t", "E_t"), ("Wd_t", "Wd_t")):
        v = pw.view(name)
        got = np.zeros(0, np.uint8) if v is None else v.cpu().numpy()
        np.testing.assert_array_equal(got, tref[key], err_msg=name)
    for name in ("Vs", "E", "Wd"):
        v = pw.view(name)
        got = np.zeros(ref[name].shape, np.uint8) if v is None else v.cpu().numpy()
        np.testing.assert_array_equal(got, ref[name], err_msg=name)
    np.testing.assert_array_equal(pw.view("w_scale").cpu().numpy(), s_w)
    pw.free()


def test_pack_rejects_bad_mask_and_nan():
    N, K, Kd = 128, 256, 64
    _, _, W, s_w, _ = _make(5, 1, N, K, Kd)
    mask = np.ones((N, K), np.uint8)
    mask[:, :K - Kd] = synth.random_mask(5, 9, N, K - Kd, (2,))
    mask[17, 8:11] = 1  # three kept in group 2 of row 17
    mask[17, 11] = 0
    with pytest.raises(spense.SpenseError) as ei:
        spense.pack(_dev(W), _dev(s_w), Kd=Kd, mask=_dev(mask))
    assert ei.value.code == 4
    W2 = W.copy()
    W2[3, 200] = 0xFF
    with pytest.raises(spense.SpenseError) as ei:
        spense.pack(_dev(W2), _dev(s_w), Kd=Kd)
    assert ei.value.code == 6


# --------------------------------------------------------------------------- GEMM, all elements

SMALL = [
    # M, N, K, Kd, scattered
    (8, 256, 512, 128, False),     # the tiny workload shape
    (1, 384, 1024, 256, False),
    (5, 200, 640, 160, False),     # ragged rows and blocks
    (16, 512, 2048, 512, False),
    (17, 256, 1024, 256, False),   # tokens just past one MMA N step
    (40, 384, 768, 0, False),      # pure 2:4
    (33, 256, 768, 768, False),    # pure dense
    (24, 320, 1536, 384, True),    # SpenseGPT+ gather
    (64, 1024, 512, 128, False),
    (128, 256, 512, 128, False),
    (200, 256, 512, 128, False),
    (256, 384, 512, 128, False),
    (300, 256, 512, 128, False),   # two token tiles
    (600, 128, 256, 64, True),     # three token tiles with a gather
]


@pytest.mark.parametrize("M,N,K,Kd,scattered", SMALL)
def test_gemm_matches_oracle(M, N, K, Kd, scattered):
    X, s_x, W, s_w, idx = _make(M * 7 + N, M, N, K, Kd, scattered)
    ref = oracle.pack(W, dense_idx=idx, Kd=Kd)
    yref, bound = oracle.gemm(X, s_x, W, s_w, keep=ref["keep"])
    pw = spense.pack(_dev(W), _dev(s_w), Kd=Kd, dense_idx=idx)
    Y, _ = _run(pw, X, s_x)
    _assert_close(Y, yref, bound, f"M={M} N={N} K={K} Kd={Kd}")


@pytest.mark.parametrize("pad", [3, 4, 8])
def test_strided_outputs_keep_their_padding(pad):
    # Outputs as column slices of a wider buffer (row stride N + pad elements), a ragged last row tile and
    # token counts with whole and shared stream-K tiles: whole tiles go out as 16-byte stores only when the
    # stride is a multiple of 8 elements and a warp's 32 rows are all in range, else as 2-byte stores; the
    # padding columns must stay untouched either way.
    # N = 40 x 128 + 104: 70 tokens split tiles over clusters of 2, 200 and 300 tokens run stream-K
    N, K, Kd = 5224, 1024, 256
    X0, s_x0, W, s_w, _ = _make(4242 + pad, 300, N, K, Kd)
    ref = oracle.pack(W, Kd=Kd)
    pw = spense.pack(_dev(W), _dev(s_w), Kd=Kd)
    for M in (70, 200, 300):
        X, s_x = X0[:M], s_x0[:M]
        yref, bound = oracle.gemm(X, s_x, W, s_w, keep=ref["keep"])
        big = torch.full((M, N + pad), float("nan"), dtype=torch.bfloat16, device="cuda")
        ws = spense.new_workspace(spense.grouped_workspace_size([pw], M))
        spense.gemm_grouped([pw], _dev(X), _dev(s_x), Ys=[big[:, :N]], workspace=ws)
        torch.cuda.synchronize()
        assert spense.workspace_status(ws) == 0
        _assert_close(big[:, :N], yref, bound, f"ldy={N + pad} M={M}")
        assert torch.isnan(big[:, N:]).all(), "a store reached the padding columns"
    pw.free()


def test_gemm_with_explicit_mask():
    M, N, K, Kd = 12, 384, 1024, 256
    X, s_x, W, s_w, _ = _make(21, M, N, K, Kd)
    mask = synth.random_mask(21, 8, N, K, (0, 1, 2), np.arange(K - Kd))
    ref = oracle.pack(W, mask=mask, Kd=Kd)
    yref, bound = oracle.gemm(X, s_x, W, s_w, keep=ref["keep"])
    pw = spense.pack(_dev(W), _dev(s_w), Kd=Kd, mask=_dev(mask))
    Y, _ = _run(pw, X, s_x)
    _assert_close(Y, yref, bound, "mask")


def test_gemm_is_deterministic_and_host_path_agrees():
    M, N, K, Kd = 16, 1024, 4096, 1024  # several CTAs share each tile
    X, s_x, W, s_w, _ = _make(31, M, N, K, Kd)
    pw = spense.pack(_dev(W), _dev(s_w), Kd=Kd)
    Y1, ws = _run(pw, X, s_x)
    Y2 = spense.gemm(pw, _dev(X), _dev(s_x), workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    hws = spense.new_workspace(spense.host_workspace_size(pw, M))
    Yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    spense.gemm_host(pw, torch.from_numpy(X).pin_memory(), torch.from_numpy(s_x).pin_memory(), Yh, hws)
    assert torch.equal(Yh.view(torch.int16), Y1.cpu().view(torch.int16))


@pytest.mark.parametrize("flags", ["x", "y", "xy", "none"])
def test_grouped_host_entry_point_equals_the_device_path(flags):
    """spense_gemm_grouped_host with the input in host memory (GEMM_HOST_X), the
    outputs in host memory (GEMM_HOST_Y), both, or neither: the same launch as
    spense_gemm_grouped on device buffers, so the outputs are equal bit for bit;
    the copies run inside the call (a decode step issued from host buffers)."""
    M, K, Kd = 16, 1024, 256
    Ns = (384, 128, 128)
    X, s_x = synth.quantize_rows(synth.normal(61, 1, (M, K), 1.0))
    pws = []
    for i, N in enumerate(Ns):
        W, s_w = synth.quantize_rows(synth.normal(61, 10 + i, (N, K), 0.02))
        pws.append(spense.pack(_dev(W), _dev(s_w), Kd=Kd))
    Xd, sxd = _dev(X), _dev(s_x)
    ref = spense.gemm_grouped(pws, Xd, sxd)
    f = (spense.GEMM_HOST_X if "x" in flags else 0) | (spense.GEMM_HOST_Y if "y" in flags else 0)
    ws = spense.new_workspace(spense.grouped_host_workspace_size(pws, M))
    xin = torch.from_numpy(X).pin_memory() if "x" in flags else Xd
    sin = torch.from_numpy(s_x).pin_memory() if "x" in flags else sxd
    if "y" in flags:
        Ys = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for N in Ns]
    else:
        Ys = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for N in Ns]
    for _ in range(2):  # twice: the second call reuses the cached launch and the staging areas
        for Y in Ys:
            Y.fill_(float("nan"))
        spense.gemm_grouped_host(pws, xin, sin, Ys, ws, f)
        torch.cuda.synchronize()
        for Y, R in zip(Ys, ref):
            assert torch.equal(Y.cpu().view(torch.int16), R.cpu().view(torch.int16)), flags
    assert spense.workspace_status(ws) == 0
    for pw in pws:
        pw.free()


def test_spenseplus_with_tail_list_equals_spensegpt():
    M, N, K, Kd = 8, 256, 1024, 256
    X, s_x, W, s_w, _ = _make(41, M, N, K, Kd)
    a = spense.pack(_dev(W), _dev(s_w), Kd=Kd)
    b = spense.pack(_dev(W), _dev(s_w), dense_idx=np.arange(K - Kd, K))
    Ya, _ = _run(a, X, s_x)
    Yb, _ = _run(b, X, s_x)
    assert torch.equal(Ya.view(torch.int16), Yb.view(torch.int16))


# --------------------------------------------------------------------------- full-size workloads, sampled rows


def _sample_rows(N, count=96, seed=0):
    g = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, N // 2, N - 129, N - 128, N - 1]
    rows = np.unique(np.concatenate([np.array([r for r in fixed if 0 <= r < N]),
                                     g.choice(N, size=min(count, N), replace=False)]))
    return rows


def _check_workload_shape(wl, i, batches, dense_frac=None):
    w = workloads.make_weight(wl, i, dense_frac)
    pw = spense.pack(_dev(w.W), _dev(w.s_w), Kd=w.Kd, dense_idx=w.dense_idx)
    rows = _sample_rows(w.N, seed=i)
    keep = oracle.pack(w.W[rows], dense_idx=w.dense_idx, Kd=w.Kd)["keep"]
    for M in batches:
        X, s_x = workloads.make_activations(wl, i, M)
        yref, bound = oracle.gemm(X, s_x, w.W[rows], w.s_w[rows], keep=keep)
        Y, _ = _run(pw, X, s_x)
        _assert_close(Y[:, torch.from_numpy(rows).cuda()], yref, bound,
                      f"{wl.name}/{w.label} M={M} df={dense_frac}")
    pw.free()


def test_tiny_workload_all_elements():
    wl = workloads.TINY
    w = workloads.make_weight(wl, 0)
    X, s_x = workloads.make_activations(wl, 0, 8)
    ref = oracle.pack(w.W, Kd=w.Kd)
    yref, bound = oracle.gemm(X, s_x, w.W, w.s_w, keep=ref["keep"])
    pw = spense.pack(_dev(w.W), _dev(w.s_w), Kd=w.Kd)
    Y, _ = _run(pw, X, s_x)
    _assert_close(Y, yref, bound, "tiny")


@pytest.mark.parametrize("i", range(4))
def test_attn32b(i):
    _check_workload_shape(workloads.ATTN32B, i, workloads.ATTN32B.batches)


@pytest.mark.parametrize("i", range(2))
def test_ffn32b(i):
    _check_workload_shape(workloads.FFN32B, i, workloads.FFN32B.batches)


@pytest.mark.parametrize("df", workloads.SPENSE_PLUS.dense_fracs)
def test_spensegpt_plus_sweep(df):
    _check_workload_shape(workloads.SPENSE_PLUS, 0, workloads.SPENSE_PLUS.batches, dense_frac=df)


@pytest.mark.parametrize("i", range(6))
def test_chain36b_layer(i):
    _check_workload_shape(workloads.CHAIN36B, i, workloads.CHAIN36B.batches)


# --------------------------------------------------------------------------- grouped launches


@pytest.mark.parametrize("M,Ns,K,Kd,scattered", [
    (16, (384, 128, 128), 1024, 256, False),
    (5, (200, 72, 330), 640, 160, False),       # ragged row counts in every member
    (40, (256, 256), 768, 256, True),            # shared SpenseGPT+ dense set
    (300, (128, 256, 128, 128), 512, 128, False),
])
def test_grouped_matches_oracle(M, Ns, K, Kd, scattered):
    X, s_x = synth.quantize_rows(synth.normal(55 + M, 1, (M, K), 1.0))
    idx = synth.scored_dense_idx(55, 3, K, Kd) if scattered else None
    pws, refs = [], []
    for i, N in enumerate(Ns):
        W, s_w = synth.quantize_rows(synth.normal(55 + M, 10 + i, (N, K), 0.02))
        keep = oracle.pack(W, dense_idx=idx, Kd=Kd)["keep"]
        refs.append(oracle.gemm(X, s_x, W, s_w, keep=keep))
        pws.append(spense.pack(_dev(W), _dev(s_w), Kd=Kd, dense_idx=idx))
    ws = spense.new_workspace(spense.grouped_workspace_size(pws, M))
    Ys = spense.gemm_grouped(pws, _dev(X), _dev(s_x), workspace=ws)
    torch.cuda.synchronize()
    assert spense.workspace_status(ws) == 0
    for i, (Y, (yref, bound)) in enumerate(zip(Ys, refs)):
        _assert_close(Y, yref, bound, f"member {i}")


@pytest.mark.parametrize("M", [1, 16])
def test_grouped_attn32b_qkv(M):
    wl = workloads.ATTN32B
    X, s_x = workloads.make_activations(wl, 0, M)
    pws, checks = [], []
    for i in range(3):  # q, k, v share the input of the layer
        w = workloads.make_weight(wl, i)
        rows = _sample_rows(w.N, seed=i)
        keep = oracle.pack(w.W[rows], Kd=w.Kd)["keep"]
        checks.append((rows, oracle.gemm(X, s_x, w.W[rows], w.s_w[rows], keep=keep)))
        pws.append(spense.pack(_dev(w.W), _dev(w.s_w), Kd=w.Kd))
    Ys = spense.gemm_grouped(pws, _dev(X), _dev(s_x))
    torch.cuda.synchronize()
    for i, (Y, (rows, (yref, bound))) in enumerate(zip(Ys, checks)):
        _assert_close(Y[:, torch.from_numpy(rows).cuda()], yref, bound, f"qkv member {i} M={M}")


def test_grouped_layout_rules():
    """Members with tail dense sets may differ in Kd (each output is its own
    GEMM); a different K or a different scattered dense set cannot share X."""
    K = 512
    W, s_w = synth.quantize_rows(synth.normal(77, 1, (128, K), 0.02))
    X, s_x = synth.quantize_rows(synth.normal(77, 2, (4, K), 1.0))
    a = spense.pack(_dev(W), _dev(s_w), Kd=128)
    b = spense.pack(_dev(W), _dev(s_w), Kd=256)
    Ya, Yb = spense.gemm_grouped([a, b], _dev(X), _dev(s_x), workspace=spense.new_workspace(1 << 20))
    torch.cuda.synchronize()
    for Y, Kd in ((Ya, 128), (Yb, 256)):
        keep = oracle.pack(W, Kd=Kd)["keep"]
        yref, bound = oracle.gemm(X, s_x, W, s_w, keep=keep)
        assert oracle.within_tolerance(Y.float().cpu().numpy(), yref, bound).all()
    W2, s2 = synth.quantize_rows(synth.normal(77, 3, (128, K + 16), 0.02))
    c = spense.pack(_dev(W2), _dev(s2), Kd=128)
    d1 = spense.pack(_dev(W), _dev(s_w), dense_idx=np.arange(0, 256, 2, dtype=np.int32))
    d2 = spense.pack(_dev(W), _dev(s_w), dense_idx=np.arange(1, 256, 2, dtype=np.int32))
    for grp in ([a, c], [d1, d2], [a, d1]):
        with pytest.raises(spense.SpenseError) as ei:
            spense.gemm_grouped(grp, _dev(X), _dev(s_x), workspace=spense.new_workspace(1 << 20))
        assert ei.value.code == 1


def test_gemm_rejects_small_workspace_and_bad_token_count():
    M, N, K, Kd = 4, 256, 512, 128
    X, s_x, W, s_w, _ = _make(88, M, N, K, Kd)
    pw = spense.pack(_dev(W), _dev(s_w), Kd=Kd)
    need = spense.workspace_size(pw, M)
    small = spense.new_workspace(need - 256)
    with pytest.raises(spense.SpenseError) as ei:
        spense.gemm(pw, _dev(X), _dev(s_x), workspace=small)
    assert ei.value.code == 7
    empty = torch.empty((0, K), dtype=torch.uint8, device="cuda")
    with pytest.raises(spense.SpenseError) as ei:
        spense.gemm(pw, empty, _dev(s_x[:0]), Y=torch.empty((1, N), dtype=torch.bfloat16, device="cuda"),
                    workspace=spense.new_workspace(need))
    assert ei.value.code == 2


def test_launch_cache_follows_handles_and_buffers():
    """Repeated calls reuse a cached launch; a freed and re-packed weight (which
    may land at the same address) and changed outputs are never served from a
    stale entry."""
    M, N, K, Kd = 8, 256, 512, 128
    X, s_x, W1, s_w1, _ = _make(61, M, N, K, Kd)
    _, _, W2, s_w2, _ = _make(62, M, N, K, Kd)
    Xd, sxd = _dev(X), _dev(s_x)
    ws = spense.new_workspace(1 << 22)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for W, s_w in ((W1, s_w1), (W2, s_w2), (W1, s_w1)):
        pw = spense.pack(_dev(W), _dev(s_w), Kd=Kd)
        for _ in range(3):
            spense.gemm_grouped([pw], Xd, sxd, [Y], ws)
        torch.cuda.synchronize()
        yref, bound = oracle.gemm(X, s_x, W, s_w, keep=oracle.pack(W, Kd=Kd)["keep"])
        _assert_close(Y, yref, bound, "cached launch")
        Y2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        spense.gemm_grouped([pw], Xd, sxd, [Y2], ws)
        torch.cuda.synchronize()
        assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
        pw.free()
    assert spense.workspace_status(ws) == 0
