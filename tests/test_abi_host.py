"""Host-only checks of the C ABI: the library loads, exports every entry point
include/spense.h declares, and rejects bad arguments with status codes before
touching a device. No GPU is needed."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import dense_fp8_gemm_b200.build as build_mod
from dense_fp8_gemm_b200 import spense

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spense.h")


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return spense.lib()


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"SPENSE_API\s+[\w\s\*]*?\b(spense_\w+)\s*\(", text)


def test_header_declares_the_binding_symbols():
    assert sorted(declared_symbols()) == sorted(spense.SYMBOLS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", build_mod.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(declared_symbols()) <= exported
    # nothing else leaks out under the spense_ prefix
    assert {s for s in exported if s.startswith("spense_")} == set(declared_symbols())


def test_version(L):
    assert re.fullmatch(r"\d+\.\d+\.\d+", spense.version())


def _pack_raw(L, W=0x1000, w_scale=0x2000, N=128, K=256, mask=None, dense_idx=None, Kd=64, flags=0):
    out = ctypes.c_void_p(0x1234)
    code = L.spense_pack(ctypes.c_void_p(W) if W else None, ctypes.c_void_p(w_scale) if w_scale else None,
                         N, K, ctypes.c_void_p(mask) if mask else None, dense_idx, Kd, flags, None,
                         ctypes.byref(out))
    return code, out


def test_pack_rejects_null_and_flags(L):
    code, out = _pack_raw(L, W=0)
    assert code == 1 and out.value is None
    assert b"NULL" in L.spense_last_error()
    code, _ = _pack_raw(L, flags=0x10)
    assert code == 1
    code = L.spense_pack(ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000), 128, 256, None, None, 64, 0, None,
                         None)
    assert code == 1


@pytest.mark.parametrize("N,K,Kd", [(0, 256, 64), (128, 8, 0), (128, 250, 64), (128, 256, 72),
                                    (128, 256, 272), (128, 256, -16), (1 << 21, 256, 0)])
def test_pack_rejects_shapes(L, N, K, Kd):
    code, _ = _pack_raw(L, N=N, K=K, Kd=Kd)
    assert code == 2, L.spense_last_error()


def test_pack_rejects_misalignment(L):
    assert _pack_raw(L, W=0x1001)[0] == 3
    assert _pack_raw(L, mask=0x3008)[0] == 3
    assert _pack_raw(L, w_scale=0x2002)[0] == 3


@pytest.mark.parametrize("idx", [[3, 2], [1, 1], [0, 256], [-1, 5]])
def test_pack_rejects_dense_idx(L, idx):
    arr = np.zeros(16, np.int32)
    arr[:] = np.arange(16) * 2
    arr[: len(idx)] = idx
    if idx == [0, 256]:
        arr = np.arange(16, dtype=np.int32)
        arr[-1] = 256
    code, _ = _pack_raw(L, dense_idx=arr.ctypes.data_as(ctypes.c_void_p), Kd=16)
    assert code == 5, L.spense_last_error()


def test_gemm_rejects_null(L):
    code = L.spense_gemm(None, ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000), 1, ctypes.c_void_p(0x3000),
                         ctypes.c_void_p(0x4000), 1 << 20, None)
    assert code == 1
    code = L.spense_gemm(ctypes.c_void_p(0x10), None, ctypes.c_void_p(0x2000), 1, ctypes.c_void_p(0x3000),
                         ctypes.c_void_p(0x4000), 1 << 20, None)
    assert code == 1
    code = L.spense_gemm(ctypes.c_void_p(0x10), ctypes.c_void_p(0x1008), ctypes.c_void_p(0x2000), 1,
                         ctypes.c_void_p(0x3000), ctypes.c_void_p(0x4000), 1 << 20, None)
    assert code == 3
    assert L.spense_gemm_workspace_size(None, 4) == 0
    assert L.spense_gemm_host_workspace_size(None, 4) == 0
    assert L.spense_get_info(None, None) == 1
    assert L.spense_free(None) == 0


def test_valid_arguments_without_a_device_report_unsupported(L):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if has_gpu:
        pytest.skip("a GPU is present")
    code, out = _pack_raw(L)
    assert code == 11 and out.value is None


def _quant_raw(L, X=0x1000, M=4, K=256, order=None, Xq=0x8000, s=0x9000):
    v = lambda a: ctypes.c_void_p(a) if a else None
    return L.spense_quantize(v(X), M, K, v(order), v(Xq), v(s), None)


def test_quantize_rejects_bad_arguments(L):
    assert _quant_raw(L, X=0) == 1
    assert _quant_raw(L, Xq=0) == 1
    assert _quant_raw(L, s=0) == 1
    for M, K in [(-1, 256), (65536, 256), (4, 8), (4, 264 - 4), (4, 0), (4, (1 << 20) + 16)]:
        assert _quant_raw(L, M=M, K=K) == 2, (M, K)
    assert _quant_raw(L, X=0x1008) == 3
    assert _quant_raw(L, Xq=0x8004) == 3
    assert _quant_raw(L, s=0x9002) == 3


def test_gemm_ex_rejects_unknown_flags(L):
    h = (ctypes.c_void_p * 1)(0x10)
    y = (ctypes.c_void_p * 1)(0x3000)
    code = L.spense_gemm_grouped_ex(h, 1, ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000), 1, y, None,
                                    ctypes.c_void_p(0x4000), 1 << 20, 0x2, None)
    assert code == 1 and b"flags" in L.spense_last_error()


def test_quantize_without_a_device_reports_unsupported(L):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if has_gpu:
        pytest.skip("a GPU is present")
    assert _quant_raw(L) == 11


def test_score_and_select_reject_bad_arguments(L):
    v = lambda a: ctypes.c_void_p(a) if a else None
    def score(gate=0x1000, s_gate=0x2000, I=64, H=32, down=0x3000, s_down=0x4000, h_in=0x5000, h_mid=0x6000,
              out=0x7000, ws=0x8000, ws_bytes=1 << 20):
        return L.spense_score_glu(v(gate), v(s_gate), None, None, I, H, v(down), v(s_down), v(h_in), v(h_mid),
                                  v(out), v(ws), ws_bytes, None)
    assert score(down=0) == 1
    assert score(s_gate=0) == 1                  # gate without its scales
    assert score(I=60) == 2 and score(H=8) == 2
    assert score(gate=0x1008) == 3 and score(h_in=0x5002) == 3
    assert score(ws=0) == 7 and score(ws_bytes=16) == 7
    assert score(ws=0x8010) == 3
    assert L.spense_score_workspace_size(64, 32) >= 32 * 64 * 4
    assert L.spense_score_workspace_size(60, 32) == 0
    assert L.spense_select_dense(v(0x1000), 0, 0, v(0x2000), None) == 2
    assert L.spense_select_dense(v(0x1000), 10, 11, v(0x2000), None) == 2
    assert L.spense_select_dense(None, 10, 3, v(0x2000), None) == 1
    assert L.spense_select_dense(v(0x1002), 10, 3, v(0x2000), None) == 3


def test_pack_rows_rejects_bad_arguments(L):
    out = ctypes.c_void_p(0x1234)
    rows = (ctypes.c_int32 * 3)(0, 5, 2)
    v = lambda a: ctypes.c_void_p(a) if a else None
    def call(W=0x1000, s=0x2000, N_src=4, K=256, r=rows, N=3):
        return L.spense_pack_rows(v(W), v(s), N_src, K, r, N, None, None, 0, 0, None, ctypes.byref(out))
    assert call(W=0) == 1 and out.value is None
    assert call(r=None) == 1
    assert call(N_src=0) == 2 and call(N=0) == 2 and call(K=250) == 2
    assert call(W=0x1004) == 3
    assert call() == 1  # rows[1] = 5 is outside [0, 4)
    assert b"rows[1]" in L.spense_last_error()


def test_glu_order_matches_the_oracle_reading():
    """spense_glu_order (host only) against the oracle's independent restatement
    of the SpenseGPT+ layout: the other indices ascending, then the dense set."""
    import oracle
    rng = np.random.default_rng(11)
    for I, kd in ((1, 0), (1, 1), (10, 3), (4096, 1024), (25600, 6400), (27648, 0), (64, 64)):
        d = np.sort(rng.choice(I, kd, replace=False)).astype(np.int32)
        got = spense.glu_order(I, d)
        assert got.dtype == np.int32
        assert np.array_equal(got, oracle.glu_order(I, d))


def test_glu_order_rejects_bad_sets(L):
    for I, d, code in ((8, [3, 3], 5), (8, [5, 2], 5), (8, [8], 5), (8, [-1], 5), (0, [], 2),
                       (4, [0, 1, 2, 3, 3], 2)):
        with pytest.raises(spense.SpenseError) as e:
            spense.glu_order(I, d)
        assert e.value.code == code, (I, d, e.value)


def test_grouped_host_rejects_bad_arguments(L):
    """spense_gemm_grouped_host checks its flags and pointers before any device
    work: unknown flags, NULL input or output, and (for device-side buffers)
    misalignment come back as status codes."""
    v = lambda a: ctypes.c_void_p(a) if a else None
    h = (ctypes.c_void_p * 1)(0x10)
    y = (ctypes.c_void_p * 1)(0x3000)
    def call(X=0x1000, sx=0x2000, Ys=y, ws=0x4000, flags=0):
        return L.spense_gemm_grouped_host(h, 1, v(X), v(sx), 4, Ys, v(ws), 1 << 20, flags, None)
    assert call(flags=0x8) == 1 and b"flags" in L.spense_last_error()
    assert call(X=0) == 1 and call(sx=0) == 1 and call(Ys=None) == 1
    assert call(X=0x1004) == 3                       # a device X must be 16-byte aligned
    assert call(sx=0x2002) == 3
    assert call(ws=0) == 7                           # no workspace
    assert L.spense_gemm_grouped_host_workspace_size(None, 1, 4) == 0
