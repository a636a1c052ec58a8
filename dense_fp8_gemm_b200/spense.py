"""Python binding of the Spense C ABI (include/spense.h): argument marshalling
only. Every step of the GEMM path runs in the CUDA library ``libspense.so``;
there is no CPU or PyTorch fallback — if the library cannot be loaded or no
sm_100 device is present, calls raise.

PyTorch supplies device memory and streams; tensors are passed by address.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from .build import LIB_PATH, TEST_LIB_PATH

SPENSE_OK = 0
STATUS_NAMES = {
    0: "OK", 1: "ERR_ARG", 2: "ERR_SHAPE", 3: "ERR_ALIGN", 4: "ERR_MASK", 5: "ERR_DENSE_IDX",
    6: "ERR_NONFINITE", 7: "ERR_WORKSPACE", 8: "ERR_OOM", 9: "ERR_CUDA", 10: "ERR_TIMEOUT",
    11: "ERR_UNSUPPORTED",
}
PACK_KEEP_CANONICAL = 1

# Exported symbols, in header order.
SYMBOLS = (
    "spense_pack", "spense_gemm", "spense_gemm_workspace_size", "spense_gemm_host",
    "spense_gemm_host_workspace_size", "spense_free", "spense_get_info",
    "spense_workspace_status", "spense_last_error", "spense_version", "spense_gemm_noalloc",
    "spense_gemm_grouped", "spense_gemm_grouped_workspace_size", "spense_gemm_grouped_ex",
    "spense_quantize", "spense_score_glu", "spense_score_workspace_size", "spense_select_dense",
    "spense_pack_rows", "spense_plan_shapes", "spense_gemm_grouped_host",
    "spense_gemm_grouped_host_workspace_size", "spense_glu_order", "spense_noalloc_status",
)
GEMM_X_PACKED_ORDER = 1
GEMM_HOST_X = 2
GEMM_HOST_Y = 4
MAX_GROUP = 4
NOALLOC_SCRATCH_BYTES = (8 << 20) + (64 << 10)


class SpenseError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({msg})")
        self.code = code


class PackedInfo(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("Ks", ctypes.c_int64), ("Kd", ctypes.c_int64),
        ("n_tiles", ctypes.c_int64), ("sparse_blocks", ctypes.c_int64), ("dense_blocks", ctypes.c_int64),
        ("Vs_t", ctypes.c_void_p), ("E_t", ctypes.c_void_p), ("Wd_t", ctypes.c_void_p),
        ("w_scale", ctypes.c_void_p), ("Vs", ctypes.c_void_p), ("E", ctypes.c_void_p),
        ("Wd", ctypes.c_void_p), ("perm", ctypes.c_void_p), ("weight_bytes", ctypes.c_uint64),
    ]


_lib = None


PLAN_MAX_GRID = 320


class PlanInfo(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("npad", "box_rows", "m_tiles", "n_tiles", "tiles", "ctas_per_sm",
                                              "cluster", "grid", "stages", "nacc")] + \
               [(n, ctypes.c_uint32) for n in ("tmem_cols", "smem_bytes", "stage_bytes", "recv_bytes")] + \
               [("l2_prefetch", ctypes.c_int32), ("pair", ctypes.c_int32), ("y_stage_bytes", ctypes.c_uint32),
                ("total_blocks", ctypes.c_int64),
                ("workspace_bytes", ctypes.c_uint64), ("cta_start", ctypes.c_int32 * (PLAN_MAX_GRID + 1))]


def lib_path() -> str:
    """libspense.so, or its test-hook build when SPENSE_TEST_HOOKS=1 (failure tests only)."""
    return TEST_LIB_PATH if os.environ.get("SPENSE_TEST_HOOKS") == "1" else LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libspense.so (built in-tree by dense_fp8_gemm_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{os.path.basename(path)} not found at {path}; run dense_fp8_gemm_b200.build.build()")
    L = ctypes.CDLL(path)
    P, I64, SZ, U32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint32
    L.spense_pack.argtypes = [P, P, I64, I64, P, P, I64, U32, P, ctypes.POINTER(P)]
    L.spense_gemm.argtypes = [P, P, P, I64, P, P, SZ, P]
    L.spense_gemm_workspace_size.argtypes = [P, I64]
    L.spense_gemm_workspace_size.restype = SZ
    L.spense_gemm_host.argtypes = [P, P, P, I64, P, P, SZ, P]
    L.spense_gemm_host_workspace_size.argtypes = [P, I64]
    L.spense_gemm_host_workspace_size.restype = SZ
    L.spense_free.argtypes = [P]
    L.spense_get_info.argtypes = [P, ctypes.POINTER(PackedInfo)]
    L.spense_plan_shapes.argtypes = [ctypes.c_int, P, P, P, I64, ctypes.c_int, ctypes.POINTER(PlanInfo)]
    L.spense_workspace_status.argtypes = [P, P, ctypes.POINTER(U32)]
    L.spense_gemm_noalloc.argtypes = [P, P, P, I64, P, P]
    L.spense_gemm_grouped.argtypes = [ctypes.POINTER(P), ctypes.c_int, P, P, I64, ctypes.POINTER(P), P, SZ, P]
    L.spense_gemm_grouped_workspace_size.argtypes = [ctypes.POINTER(P), ctypes.c_int, I64]
    L.spense_gemm_grouped_workspace_size.restype = SZ
    L.spense_gemm_grouped_ex.argtypes = [ctypes.POINTER(P), ctypes.c_int, P, P, I64, ctypes.POINTER(P), P, P,
                                         SZ, U32, P]
    L.spense_pack_rows.argtypes = [P, P, I64, I64, P, I64, P, P, I64, U32, P, ctypes.POINTER(P)]
    L.spense_quantize.argtypes = [P, I64, I64, P, P, P, P]
    L.spense_score_glu.argtypes = [P, P, P, P, I64, I64, P, P, P, P, P, P, SZ, P]
    L.spense_score_workspace_size.argtypes = [I64, I64]
    L.spense_score_workspace_size.restype = SZ
    L.spense_select_dense.argtypes = [P, I64, I64, P, P]
    L.spense_gemm_grouped_host.argtypes = [ctypes.POINTER(P), ctypes.c_int, P, P, I64, ctypes.POINTER(P), P, SZ,
                                           U32, P]
    L.spense_gemm_grouped_host_workspace_size.argtypes = [ctypes.POINTER(P), ctypes.c_int, I64]
    L.spense_gemm_grouped_host_workspace_size.restype = SZ
    L.spense_glu_order.argtypes = [I64, P, I64, P]
    L.spense_noalloc_status.argtypes = [P, ctypes.POINTER(U32)]
    L.spense_last_error.restype = ctypes.c_char_p
    L.spense_version.restype = ctypes.c_char_p
    for name in ("spense_pack", "spense_gemm", "spense_gemm_host", "spense_free", "spense_get_info",
                 "spense_workspace_status", "spense_gemm_noalloc", "spense_gemm_grouped",
                 "spense_gemm_grouped_host", "spense_glu_order", "spense_noalloc_status"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(code: int, where: str):
    if code != SPENSE_OK:
        raise SpenseError(code, where, lib().spense_last_error().decode())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev_ptr(t: torch.Tensor | None, dtype, name: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


class _DevView:
    """Zero-copy view of library-owned device memory for torch.as_tensor (do not write through it)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"data": (ptr, False), "shape": tuple(shape), "typestr": typestr,
                                         "version": 3, "strides": None}


class PackedWeight:
    """A packed Spense weight (owns its device buffers through the C handle)."""

    def __init__(self, handle: ctypes.c_void_p):
        self._h = handle
        info = PackedInfo()
        _check(lib().spense_get_info(self._h, ctypes.byref(info)), "spense_get_info")
        self.info = info

    @property
    def handle(self):
        return self._h

    @property
    def N(self):
        return self.info.N

    @property
    def K(self):
        return self.info.K

    @property
    def Ks(self):
        return self.info.Ks

    @property
    def Kd(self):
        return self.info.Kd

    @property
    def weight_bytes(self):
        return int(self.info.weight_bytes)

    def view(self, name: str) -> torch.Tensor | None:
        """Read-only view of a packed array ('Vs_t', 'E_t', 'Wd_t', 'Vs', 'E', 'Wd', 'perm', 'w_scale')."""
        i = self.info
        nt, nsb, ndb = i.n_tiles, i.sparse_blocks, i.dense_blocks
        shapes = {
            "Vs_t": ((nt * nsb * 16384,), "|u1"), "E_t": ((nt * nsb * 4096,), "|u1"),
            "Wd_t": ((nt * ndb * 16384,), "|u1"), "Vs": ((i.N, i.Ks // 2), "|u1"),
            "E": ((i.N, i.Ks // 8), "|u1"), "Wd": ((i.N, i.Kd), "|u1"), "perm": ((i.K,), "<i4"),
            "w_scale": ((i.N,), "<f4"),
        }
        shape, ts = shapes[name]
        ptr = getattr(i, name)
        if not ptr or int(np.prod(shape)) == 0:
            return None
        return torch.as_tensor(_DevView(ptr, shape, ts), device="cuda")

    def free(self):
        if self._h is not None and self._h.value:
            _check(lib().spense_free(self._h), "spense_free")
        self._h = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def pack(W: torch.Tensor, w_scale: torch.Tensor, Kd: int | None = None, mask: torch.Tensor | None = None,
         dense_idx=None, keep_canonical: bool = False, stream=None, rows=None) -> PackedWeight:
    """spense_pack, or spense_pack_rows when `rows` (host int32 row indices) is
    given. W: uint8 [N, K] (e4m3 bytes) on the GPU; w_scale fp32 [N];
    dense_idx: host int32 index list (SpenseGPT+) or None (tail of Kd columns)."""
    N, K = W.shape
    idx = None
    if dense_idx is not None:
        idx = np.ascontiguousarray(np.asarray(dense_idx), dtype=np.int32)
        if Kd is not None and Kd != idx.shape[0]:
            raise ValueError("Kd disagrees with len(dense_idx)")
        Kd = idx.shape[0]
    if Kd is None:
        raise ValueError("Kd (or dense_idx) is required")
    out = ctypes.c_void_p()
    flags = PACK_KEEP_CANONICAL if keep_canonical else 0
    dptr = None if idx is None else idx.ctypes.data_as(ctypes.c_void_p)
    if rows is None:
        code = lib().spense_pack(
            _dev_ptr(W, torch.uint8, "W"), _dev_ptr(w_scale, torch.float32, "w_scale"), N, K,
            _dev_ptr(mask, torch.uint8, "mask"), dptr, Kd, flags, _stream(stream), ctypes.byref(out))
        _check(code, "spense_pack")
    else:
        r = np.ascontiguousarray(np.asarray(rows), dtype=np.int32)
        code = lib().spense_pack_rows(
            _dev_ptr(W, torch.uint8, "W"), _dev_ptr(w_scale, torch.float32, "w_scale"), N, K,
            r.ctypes.data_as(ctypes.c_void_p), r.shape[0], _dev_ptr(mask, torch.uint8, "mask"), dptr, Kd, flags,
            _stream(stream), ctypes.byref(out))
        _check(code, "spense_pack_rows")
    return PackedWeight(out)


def workspace_size(pw: PackedWeight, M: int) -> int:
    n = lib().spense_gemm_workspace_size(pw.handle, M)
    if n == 0:
        _check(1, "spense_gemm_workspace_size")
    return int(n)


def host_workspace_size(pw: PackedWeight, M: int) -> int:
    n = lib().spense_gemm_host_workspace_size(pw.handle, M)
    if n == 0:
        _check(1, "spense_gemm_host_workspace_size")
    return int(n)


def new_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-filled workspace (the ABI requires zeros before first use)."""
    return torch.zeros(nbytes, dtype=torch.uint8, device=device or "cuda")


def gemm(pw: PackedWeight, X: torch.Tensor, x_scale: torch.Tensor, Y: torch.Tensor | None = None,
         workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """spense_gemm: Y [M, N] bf16 = X [M, K] e4m3 x packed W^T, scaled."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty((M, pw.N), dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = new_workspace(workspace_size(pw, M), X.device)
    code = lib().spense_gemm(pw.handle, _dev_ptr(X, torch.uint8, "X"),
                             _dev_ptr(x_scale, torch.float32, "x_scale"), M,
                             _dev_ptr(Y, torch.bfloat16, "Y"), _dev_ptr(workspace, torch.uint8, "workspace"),
                             workspace.numel(), _stream(stream))
    _check(code, "spense_gemm")
    return Y


def gemm_host(pw: PackedWeight, X_host: torch.Tensor, x_scale_host: torch.Tensor, Y_host: torch.Tensor,
              workspace: torch.Tensor, stream=None) -> torch.Tensor:
    """spense_gemm_host: host (pinned) X, x_scale in; host Y out; synchronous."""
    for t, name in ((X_host, "X"), (x_scale_host, "x_scale"), (Y_host, "Y")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor")
    M = X_host.shape[0]
    code = lib().spense_gemm_host(pw.handle, ctypes.c_void_p(X_host.data_ptr()),
                                  ctypes.c_void_p(x_scale_host.data_ptr()), M,
                                  ctypes.c_void_p(Y_host.data_ptr()),
                                  _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                                  _stream(stream))
    _check(code, "spense_gemm_host")
    return Y_host


def _handles(pws):
    arr = (ctypes.c_void_p * len(pws))()
    for i, pw in enumerate(pws):
        arr[i] = pw.handle.value
    return arr


def grouped_workspace_size(pws, M: int) -> int:
    n = lib().spense_gemm_grouped_workspace_size(_handles(pws), len(pws), M)
    if n == 0:
        _check(1, "spense_gemm_grouped_workspace_size")
    return int(n)


def gemm_grouped(pws, X: torch.Tensor, x_scale: torch.Tensor, Ys=None, workspace: torch.Tensor | None = None,
                 stream=None, flags: int = 0, ldy=None):
    """spense_gemm_grouped (flags == 0, ldy None) or spense_gemm_grouped_ex:
    one launch over several packed weights sharing X (same K and column order
    of X). flags = GEMM_X_PACKED_ORDER: X is already in the packed column order
    (from quantize(..., order=pw)). ldy: per-output row strides in elements,
    with Ys given as flat device tensors (views into a wider output). Returns
    the list of outputs."""
    M = X.shape[0]
    if Ys is None:
        Ys = [torch.empty((M, pw.N), dtype=torch.bfloat16, device=X.device) for pw in pws]
    if workspace is None:
        workspace = new_workspace(grouped_workspace_size(pws, M), X.device)
    yarr = (ctypes.c_void_p * len(pws))()
    strided = any(not Y.is_contiguous() for Y in Ys)
    if strided and ldy is None:
        ldy = [Y.stride(0) for Y in Ys]  # column slices of a wider output
    for i, Y in enumerate(Ys):
        if Y.is_contiguous():
            yarr[i] = _dev_ptr(Y, torch.bfloat16, f"Y[{i}]").value
        else:
            if not Y.is_cuda or Y.dtype != torch.bfloat16 or Y.stride(1) != 1:
                raise ValueError(f"Y[{i}] must be a bfloat16 CUDA tensor with unit column stride")
            yarr[i] = Y.data_ptr()
    if flags == 0 and ldy is None:
        _check(lib().spense_gemm_grouped(_handles(pws), len(pws), _dev_ptr(X, torch.uint8, "X"),
                                         _dev_ptr(x_scale, torch.float32, "x_scale"), M, yarr,
                                         _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                                         _stream(stream)), "spense_gemm_grouped")
    else:
        larr = None if ldy is None else (ctypes.c_int64 * len(pws))(*[int(v) for v in ldy])
        _check(lib().spense_gemm_grouped_ex(_handles(pws), len(pws), _dev_ptr(X, torch.uint8, "X"),
                                            _dev_ptr(x_scale, torch.float32, "x_scale"), M, yarr, larr,
                                            _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                                            int(flags), _stream(stream)), "spense_gemm_grouped_ex")
    return Ys


class PreparedGrouped:
    """A grouped GEMM call with its arguments marshalled once (for loops that
    launch the same GEMM on the same buffers, such as a decode step): calling
    it makes one C call. The tensors must stay alive and in place."""

    def __init__(self, pws, X: torch.Tensor, x_scale: torch.Tensor, Ys, workspace: torch.Tensor, flags: int = 0):
        self._keep = (list(pws), X, x_scale, list(Ys), workspace)
        yarr = (ctypes.c_void_p * len(pws))()
        for i, Y in enumerate(Ys):
            yarr[i] = _dev_ptr(Y, torch.bfloat16, f"Y[{i}]").value
        self._fn = lib().spense_gemm_grouped_ex
        self._args = (_handles(pws), len(pws), _dev_ptr(X, torch.uint8, "X"),
                      _dev_ptr(x_scale, torch.float32, "x_scale"), X.shape[0], yarr, None,
                      _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(), int(flags))

    def __call__(self, stream=None):
        code = self._fn(*self._args, _stream(stream))
        if code != SPENSE_OK:
            _check(code, "spense_gemm_grouped_ex")


def grouped_host_workspace_size(pws, M: int) -> int:
    n = lib().spense_gemm_grouped_host_workspace_size(_handles(pws), len(pws), M)
    if n == 0:
        _check(1, "spense_gemm_grouped_host_workspace_size")
    return int(n)


def _ptr(t: torch.Tensor, dtype, name: str, host: bool):
    if host:
        if t.is_cuda or t.dtype != dtype or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {dtype} host tensor")
        return ctypes.c_void_p(t.data_ptr())
    return _dev_ptr(t, dtype, name)


class PreparedGroupedHost:
    """spense_gemm_grouped_host with its arguments marshalled once: X (and
    x_scale) in host memory when flags has GEMM_HOST_X, the outputs in host
    memory when it has GEMM_HOST_Y (the call then synchronizes the stream).
    The tensors must stay alive and in place."""

    def __init__(self, pws, X: torch.Tensor, x_scale: torch.Tensor, Ys, workspace: torch.Tensor, flags: int):
        hx, hy = bool(flags & GEMM_HOST_X), bool(flags & GEMM_HOST_Y)
        self._keep = (list(pws), X, x_scale, list(Ys), workspace)
        yarr = (ctypes.c_void_p * len(pws))()
        for i, Y in enumerate(Ys):
            yarr[i] = _ptr(Y, torch.bfloat16, f"Y[{i}]", hy).value
        self._fn = lib().spense_gemm_grouped_host
        self._args = (_handles(pws), len(pws), _ptr(X, torch.uint8, "X", hx),
                      _ptr(x_scale, torch.float32, "x_scale", hx), X.shape[0], yarr,
                      _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(), int(flags))

    def __call__(self, stream=None):
        code = self._fn(*self._args, _stream(stream))
        if code != SPENSE_OK:
            _check(code, "spense_gemm_grouped_host")


def gemm_grouped_host(pws, X: torch.Tensor, x_scale: torch.Tensor, Ys, workspace: torch.Tensor, flags: int,
                      stream=None):
    """spense_gemm_grouped_host: one grouped launch whose input (GEMM_HOST_X),
    outputs (GEMM_HOST_Y) or both live in host memory; the copies run inside
    the call. Returns Ys."""
    PreparedGroupedHost(pws, X, x_scale, Ys, workspace, flags)(stream)
    return Ys


def glu_order(I: int, dense_idx) -> np.ndarray:
    """spense_glu_order: the other intermediate indices ascending, then the
    dense set (the packed column order of a weight packed with that set)."""
    idx = np.ascontiguousarray(np.asarray(dense_idx, dtype=np.int32))
    out = np.empty((I,), dtype=np.int32)
    _check(lib().spense_glu_order(int(I), idx.ctypes.data_as(ctypes.c_void_p) if idx.size else None, idx.size,
                                  out.ctypes.data_as(ctypes.c_void_p)), "spense_glu_order")
    return out


def quantize(X: torch.Tensor, order: PackedWeight | None = None, Xq: torch.Tensor | None = None,
             x_scale: torch.Tensor | None = None, stream=None):
    """spense_quantize: per-token FP8 quantisation of bf16 activations X [M, K]
    (s = absmax / 448 in fp32, e4m3 round-to-nearest-even, saturating), with the
    columns in `order`'s packed order when a packed weight is given. Returns
    (Xq uint8 [M, K], x_scale float32 [M])."""
    M, K = X.shape
    if Xq is None:
        Xq = torch.empty((M, K), dtype=torch.uint8, device=X.device)
    if x_scale is None:
        x_scale = torch.empty((M,), dtype=torch.float32, device=X.device)
    code = lib().spense_quantize(_dev_ptr(X, torch.bfloat16, "X"), M, K, None if order is None else order.handle,
                                 _dev_ptr(Xq, torch.uint8, "Xq"), _dev_ptr(x_scale, torch.float32, "x_scale"),
                                 _stream(stream))
    _check(code, "spense_quantize")
    return Xq, x_scale


def gemm_noalloc(pw: PackedWeight, X: torch.Tensor, x_scale: torch.Tensor, Y: torch.Tensor,
                 stream=None) -> torch.Tensor:
    """spense_gemm_noalloc: the GEMM without a caller workspace, for callers that
    cannot allocate device memory when they run it. The library's built-in
    scratch array stands in for the workspace, so calls must not overlap on the
    GPU. Y must be preallocated (this call allocates nothing)."""
    code = lib().spense_gemm_noalloc(pw.handle, _dev_ptr(X, torch.uint8, "X"),
                                     _dev_ptr(x_scale, torch.float32, "x_scale"), X.shape[0],
                                     _dev_ptr(Y, torch.bfloat16, "Y"), _stream(stream))
    _check(code, "spense_gemm_noalloc")
    return Y


def noalloc_status(stream=None) -> int:
    """Reads and clears the status word of the noalloc scratch on the current
    device (0 = every noalloc GEMM since the last read completed normally)."""
    out = ctypes.c_uint32()
    _check(lib().spense_noalloc_status(_stream(stream), ctypes.byref(out)), "spense_noalloc_status")
    return int(out.value)


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Reads and clears the device status word of a workspace (0 = all good)."""
    out = ctypes.c_uint32()
    _check(lib().spense_workspace_status(_dev_ptr(workspace, torch.uint8, "workspace"), _stream(stream),
                                         ctypes.byref(out)), "spense_workspace_status")
    return int(out.value)


def plan_shapes(shapes, M: int, sms: int = 148) -> dict:
    """spense_plan_shapes: the launch plan of a grouped GEMM over weights of
    the given (N, K, Kd) shapes for M tokens on a device with `sms` SMs, from
    the shapes alone (no GPU). Returns the plan's fields; cta_start as a list
    of grid + 1 block indices."""
    n = len(shapes)
    arr = [np.ascontiguousarray([int(s[i]) for s in shapes], dtype=np.int64) for i in range(3)]
    info = PlanInfo()
    code = lib().spense_plan_shapes(n, *(a.ctypes.data_as(ctypes.c_void_p) for a in arr), int(M), int(sms),
                                    ctypes.byref(info))
    _check(code, "spense_plan_shapes")
    out = {name: getattr(info, name) for name, _ in PlanInfo._fields_ if name != "cta_start"}
    out["cta_start"] = list(info.cta_start[:info.grid + 1])
    return out


def version() -> str:
    return lib().spense_version().decode()


def score_glu(down: torch.Tensor, s_down: torch.Tensor, h_in: torch.Tensor, h_mid: torch.Tensor,
              gate: torch.Tensor | None = None, s_gate: torch.Tensor | None = None,
              up: torch.Tensor | None = None, s_up: torch.Tensor | None = None,
              score: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """spense_score_glu: SpenseGPT+ importance of every intermediate index of a
    GLU MLP. gate/up: uint8 e4m3 [I, H] (+ fp32 row scales [I]); down: uint8 e4m3
    [H, I] (+ fp32 [H]); h_in [H], h_mid [I] fp32 Hessian diagonals. Returns
    score fp32 [I]."""
    H, I = down.shape
    if score is None:
        score = torch.empty((I,), dtype=torch.float32, device=down.device)
    if workspace is None:
        workspace = new_workspace(max(256, int(lib().spense_score_workspace_size(I, H))), down.device)
    code = lib().spense_score_glu(_dev_ptr(gate, torch.uint8, "gate"), _dev_ptr(s_gate, torch.float32, "s_gate"),
                                  _dev_ptr(up, torch.uint8, "up"), _dev_ptr(s_up, torch.float32, "s_up"), I, H,
                                  _dev_ptr(down, torch.uint8, "down"), _dev_ptr(s_down, torch.float32, "s_down"),
                                  _dev_ptr(h_in, torch.float32, "h_in"), _dev_ptr(h_mid, torch.float32, "h_mid"),
                                  _dev_ptr(score, torch.float32, "score"),
                                  _dev_ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    _check(code, "spense_score_glu")
    return score


def select_dense(score: torch.Tensor, Kd: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """spense_select_dense: the Kd largest scores (ties to the lower index) as
    ascending int32 indices on the device."""
    I = score.shape[0]
    if out is None:
        out = torch.empty((Kd,), dtype=torch.int32, device=score.device)
    code = lib().spense_select_dense(_dev_ptr(score, torch.float32, "score"), I, int(Kd),
                                     _dev_ptr(out, torch.int32, "dense_idx") if Kd > 0 else None, _stream(stream))
    _check(code, "spense_select_dense")
    return out
