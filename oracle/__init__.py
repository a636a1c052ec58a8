"""CPU oracle for the Spense hybrid 2:4-sparse + dense FP8 GEMM.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product library
(``dense_fp8_gemm_b200``) never imports it and shares no code with it.

The arithmetic lives in ``spense_oracle.cpp`` (plain C++, double precision);
this module only marshals numpy arrays through ``ctypes``. Every function cites
the passage of "SpenseGPT: Practical One-shot Pruning Enabling Sparse and Dense
GEMMs for LLM Inference" (gist.science technical summary) that it follows; the
readings taken where that page is silent are listed at the top of the C++ file.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build as _build, LIB_PATH

_lib = None

OR_OK = 0
OR_ERR_ARG = 1
OR_ERR_SHAPE = 2
OR_ERR_MASK = 4
OR_ERR_DENSE_IDX = 5
OR_ERR_NONFINITE = 6


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what} failed with status {code}")
        self.code = code


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        _build()
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.oracle_e4m3_table.argtypes = [P]
    lib.oracle_e4m3_table.restype = None
    lib.oracle_pack.argtypes = [P, I64, I64, P, P, I64, P, P, P, P]
    lib.oracle_pack.restype = ctypes.c_int
    lib.oracle_unpack.argtypes = [P, P, P, I64, I64, P, I64, P]
    lib.oracle_unpack.restype = ctypes.c_int
    lib.oracle_tile.argtypes = [P, P, P, I64, I64, I64, P, P, P]
    lib.oracle_tile.restype = ctypes.c_int
    lib.oracle_gemm.argtypes = [P, P, I64, P, P, I64, I64, P, P, I64, P, P, ctypes.c_int]
    lib.oracle_gemm.restype = ctypes.c_int
    lib.oracle_quantize.argtypes = [P, I64, I64, P, I64, P, P]
    lib.oracle_quantize.restype = ctypes.c_int
    lib.oracle_score_glu.argtypes = [P, P, P, P, I64, I64, P, P, P, P, P]
    lib.oracle_score_glu.restype = ctypes.c_int
    lib.oracle_select_top.argtypes = [P, I64, I64, P]
    lib.oracle_select_top.restype = ctypes.c_int
    lib.oracle_hardware_concurrency.argtypes = []
    lib.oracle_hardware_concurrency.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u8(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.uint8)


def _idx(dense_idx):
    return None if dense_idx is None else np.ascontiguousarray(dense_idx, dtype=np.int32)


def e4m3_table() -> np.ndarray:
    """All 256 e4m3fn byte values decoded to float64 (OCP FP8 E4M3; the pages
    say only "FP8 precision on B200", Technical Summary §4)."""
    out = np.empty(256, dtype=np.float64)
    _load().oracle_e4m3_table(_ptr(out))
    return out


def decode(b: np.ndarray) -> np.ndarray:
    return e4m3_table()[np.asarray(b, dtype=np.uint8)]


def pack(W, mask=None, dense_idx=None, Kd=None):
    """Canonical Spense pack (Technical Summary §2A split into a dense region and
    a 2:4 region; §2B tail or index-set dense selection; §1 2:4 definition).

    Returns dict(Vs [N,Ks/2], E [N,ceil(Ks/8)], Wd [N,Kd], keep [N,K]) of uint8.
    """
    W = _u8(W)
    N, K = W.shape
    di = _idx(dense_idx)
    if di is not None:
        Kd = di.shape[0]
    assert Kd is not None
    Ks = K - Kd
    Vs = np.zeros((N, Ks // 2), np.uint8)
    E = np.zeros((N, (Ks + 7) // 8), np.uint8)
    Wd = np.zeros((N, Kd), np.uint8)
    keep = np.zeros((N, K), np.uint8)
    m = _u8(mask)
    st = _load().oracle_pack(_ptr(W), N, K, _ptr(m), _ptr(di), Kd, _ptr(Vs), _ptr(E), _ptr(Wd),
                             _ptr(keep))
    if st != OR_OK:
        raise OracleError(st, "pack")
    return {"Vs": Vs, "E": E, "Wd": Wd, "keep": keep, "Ks": Ks, "Kd": Kd}


def unpack(Vs, E, Wd, K, dense_idx=None):
    """Masked matrix in original column order from the canonical pack."""
    Vs, E, Wd = _u8(Vs), _u8(E), _u8(Wd)
    N = Vs.shape[0]
    Kd = Wd.shape[1]
    out = np.zeros((N, K), np.uint8)
    st = _load().oracle_unpack(_ptr(Vs), _ptr(E), _ptr(Wd), N, K, _ptr(_idx(dense_idx)), Kd,
                               _ptr(out))
    if st != OR_OK:
        raise OracleError(st, "unpack")
    return out


def tile(Vs, E, Wd, N, Ks, Kd):
    """The library's MMA-tiled storage restated from its definition."""
    nt = (N + 127) // 128
    nsb = (Ks + 255) // 256
    ndb = (Kd + 127) // 128
    Vs_t = np.zeros(nt * nsb * 16384, np.uint8)
    E_t = np.zeros(nt * nsb * 4096, np.uint8)
    Wd_t = np.zeros(nt * ndb * 16384, np.uint8)
    st = _load().oracle_tile(_ptr(_u8(Vs)), _ptr(_u8(E)), _ptr(_u8(Wd)), N, Ks, Kd, _ptr(Vs_t),
                             _ptr(E_t), _ptr(Wd_t))
    if st != OR_OK:
        raise OracleError(st, "tile")
    return {"Vs_t": Vs_t, "E_t": E_t, "Wd_t": Wd_t}


def gemm(X, s_x, W, s_w, keep=None, rows=None, nthreads=None):
    """y_ref and the tolerance bound of Y = X * (keep . W)^T with scales, in
    float64 (Technical Summary §2A input-split: sparse GEMM plus dense GEMM
    with accumulation equals one GEMM over the masked matrix; §2B the dense
    permutation leaves the output unchanged).

    Returns (yref [M,R], bound [M,R]) where R = len(rows) or N.
    """
    X = _u8(X)
    W = _u8(W)
    M, K = X.shape
    N, K2 = W.shape
    assert K == K2
    s_x = np.ascontiguousarray(s_x, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    kp = _u8(keep)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    R = N if r is None else r.shape[0]
    y = np.zeros((M, R), np.float64)
    b = np.zeros((M, R), np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    st = _load().oracle_gemm(_ptr(X), _ptr(s_x), M, _ptr(W), _ptr(s_w), N, K, _ptr(kp), _ptr(r),
                             R, _ptr(y), _ptr(b), int(nthreads))
    if st != OR_OK:
        raise OracleError(st, "gemm")
    return y, b


def quantize(X_bf16, dense_idx=None):
    """Per-token FP8 quantisation of bf16 activations with the packed column
    order fused in: s[m] = fp32(absmax / 448) (1 for a zero row), Xq[m][j] =
    e4m3 round-to-nearest-even, saturating, of fp32(x[m][c(j)] / s[m]), where c
    is sparse columns ascending then `dense_idx` (identity when None).
    (Technical Summary §2B: the dense indices are permuted into a contiguous
    block; the SlideSparse page, Activation Lifting: the rearrangement is
    folded into per-token quantisation.)

    X_bf16: uint16 bit patterns [M, K]. Returns (Xq uint8 [M, K], s float32 [M]).
    """
    X = np.ascontiguousarray(X_bf16, dtype=np.uint16)
    M, K = X.shape
    di = _idx(dense_idx)
    Kd = 0 if di is None else di.shape[0]
    Xq = np.zeros((M, K), np.uint8)
    s = np.zeros(M, np.float32)
    st = _load().oracle_quantize(_ptr(X), M, K, _ptr(di), Kd, _ptr(Xq), _ptr(s))
    if st != OR_OK:
        raise OracleError(st, "quantize")
    return Xq, s


def score_glu(down, s_down, h_in, h_mid, gate=None, s_gate=None, up=None, s_up=None):
    """SpenseGPT+ importance of every intermediate index of a GLU MLP, float64
    (Technical Summary §2B: S_ij = |W_ij| sqrt(H_jj) aggregated over gate, up
    and down). gate/up: e4m3 [I, H] with fp32 row scales [I]; down: e4m3 [H, I]
    with row scales [H]; h_in [H], h_mid [I]: Hessian diagonals. Returns [I]."""
    down = _u8(down)
    H, I = down.shape
    f32 = lambda a: None if a is None else np.ascontiguousarray(a, dtype=np.float32)
    g, u = _u8(gate), _u8(up)
    out = np.zeros(I, np.float64)
    st = _load().oracle_score_glu(_ptr(g), _ptr(f32(s_gate)), _ptr(u), _ptr(f32(s_up)), I, H, _ptr(down),
                                  _ptr(f32(s_down)), _ptr(f32(h_in)), _ptr(f32(h_mid)), _ptr(out))
    if st != OR_OK:
        raise OracleError(st, "score_glu")
    return out


def select_top(score, Kd):
    """The Kd largest scores (ties to the lower index), ascending indices
    (Technical Summary §2B: the top-scoring indices stay dense)."""
    sc = np.ascontiguousarray(score, dtype=np.float64)
    out = np.zeros(Kd, np.int32)
    st = _load().oracle_select_top(_ptr(sc), sc.shape[0], int(Kd), _ptr(out))
    if st != OR_OK:
        raise OracleError(st, "select_top")
    return out


def output_split_keep(W, dense_rows):
    """Keep mask [N, K] of an output-split weight (Technical Summary §2A:
    output-split splits the output tensor, a sparse GEMM for one part and a
    dense GEMM for the other): the rows in `dense_rows` keep every entry, every
    other row is 2:4 over all K columns (its top two per group of four, as
    `pack` with Kd = 0 selects them). Y = gemm(X, s_x, W, s_w, keep=...)."""
    W = _u8(W)
    N, K = W.shape
    dense = np.zeros(N, bool)
    dense[np.asarray(dense_rows, dtype=np.int64)] = True
    keep = np.ones((N, K), np.uint8)
    sparse_rows = np.flatnonzero(~dense)
    if sparse_rows.size:
        keep[sparse_rows] = pack(W[sparse_rows], Kd=0)["keep"]
    return keep


def glu_order(I, dense_idx):
    """The order of the intermediate indices of a GLU MLP after its dense
    indices are permuted into one contiguous block at the end (Technical
    Summary §2B): the other indices ascending, then `dense_idx` ascending."""
    d = np.asarray(dense_idx, dtype=np.int64)
    rest = np.setdiff1d(np.arange(I, dtype=np.int64), d)
    return np.concatenate([rest, np.sort(d)])


def hardware_concurrency() -> int:
    """std::thread::hardware_concurrency() of the host the oracle runs on."""
    return int(_load().oracle_hardware_concurrency())


def within_tolerance(y, yref, bound, rel=4e-3, absb=1e-5):
    """The acceptance rule |y - y_ref| <= 4e-3 |y_ref| + 1e-5 sum_k |w_k x_k|."""
    y = np.asarray(y, dtype=np.float64)
    return np.abs(y - yref) <= rel * np.abs(yref) + absb * bound
