"""Python binding of ``libgl.so`` (see ``include/gl.h``).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of the library.  PyTorch supplies device memory and the current
stream.  The entry points keep the C names: :func:`gl_offsets`,
:func:`gl_fwd`, :func:`gl_dgrad`, :func:`gl_wgrad` and
:func:`group_quantize_mxfp8`.  There is no fallback: if the library has not
been built, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Union

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgl.so")
_lib = None

GL_OK, GL_ERR_INVALID, GL_ERR_UNSUPPORTED, GL_ERR_CUDA = 0, 1, 2, 3
GL_DEV_NEG_SPLIT, GL_DEV_SUM_MISMATCH, GL_DEV_OUT_OVERFLOW, GL_DEV_TIMEOUT = 1, 2, 4, 8
GL_STACKED, GL_PER_GROUP = 0, 1
GL_SCALES_ROWMAJOR, GL_SCALES_MMA = 0, 1

EXPORTED = ("gl_version", "gl_status_string", "gl_offsets", "gl_fwd", "gl_dgrad", "gl_wgrad",
            "gl_dbias", "group_quantize_mxfp8", "gl_mxfp8_scale_bytes", "gl_dbias_workspace_bytes",
            "group_quantize_mxfp8_dbias", "gl_fwd_mxfp8", "gl_dgrad_mxfp8", "gl_wgrad_mxfp8")


class GlGrouped(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("base", ctypes.c_void_p),
                ("ptrs", ctypes.POINTER(ctypes.c_void_p))]


GL_TILES_PAIR, GL_TILES_SINGLE = 0, 1


GL_OPT_HOLD_LOADS = 1


class GlGemmOpts(ctypes.Structure):
    _fields_ = [("tiles", ctypes.c_int), ("wait_limit_us", ctypes.c_uint32), ("flags", ctypes.c_uint32)]


class GlError(RuntimeError):
    pass


def lib_path() -> str:
    return _LIB_PATH


def load() -> ctypes.CDLL:
    """Load libgl.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise GlError(f"{_LIB_PATH} is missing: build it with `python -m grouped_gemm_splits_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    L.gl_version.restype = i32
    L.gl_status_string.restype = ctypes.c_char_p
    L.gl_status_string.argtypes = [i32]
    L.gl_offsets.restype = i32
    L.gl_offsets.argtypes = [vp, i32, i64, i64, vp, vp, vp]
    L.gl_fwd.restype = i32
    op = ctypes.POINTER(GlGemmOpts)
    L.gl_fwd.argtypes = [vp, GlGrouped, ctypes.POINTER(GlGrouped), vp, vp, i32, i64, i32, i32, vp, i64, op, vp]
    L.gl_dgrad.restype = i32
    L.gl_dgrad.argtypes = [vp, GlGrouped, vp, vp, i32, i64, i32, i32, vp, i64, op, vp]
    L.gl_wgrad.restype = i32
    L.gl_wgrad.argtypes = [vp, vp, vp, vp, i32, i64, i32, i32, GlGrouped, i32, op, vp]
    L.gl_dbias.restype = i32
    L.gl_dbias.argtypes = [vp, vp, vp, i32, i64, i32, GlGrouped, vp]
    L.group_quantize_mxfp8.restype = i32
    L.group_quantize_mxfp8.argtypes = [vp, i64, i32, vp, i32, vp, vp, vp, vp, vp, i32, vp]
    L.gl_mxfp8_scale_bytes.restype = ctypes.c_size_t
    L.gl_mxfp8_scale_bytes.argtypes = [i64, i32, i32, i32, i32]
    L.gl_dbias_workspace_bytes.restype = ctypes.c_size_t
    L.gl_dbias_workspace_bytes.argtypes = [i64, i32, i32]
    L.group_quantize_mxfp8_dbias.restype = i32
    L.group_quantize_mxfp8_dbias.argtypes = [vp, i64, i32, vp, i32, vp, vp, vp, vp, vp, i32, GlGrouped, vp,
                                             ctypes.c_size_t, vp]
    L.gl_fwd_mxfp8.restype = i32
    L.gl_fwd_mxfp8.argtypes = [vp, vp, GlGrouped, GlGrouped, ctypes.POINTER(GlGrouped), vp, vp, i32, i64, i32,
                               i32, vp, i64, op, vp]
    L.gl_dgrad_mxfp8.restype = i32
    L.gl_dgrad_mxfp8.argtypes = [vp, vp, GlGrouped, GlGrouped, vp, vp, i32, i64, i32, i32, vp, i64, op, vp]
    L.gl_wgrad_mxfp8.restype = i32
    L.gl_wgrad_mxfp8.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, GlGrouped, i32, op, vp]
    _lib = L
    return L


def _check(st: int, what: str) -> None:
    if st != GL_OK:
        raise GlError(f"{what}: {load().gl_status_string(st).decode()} ({st})")


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


TensorOrList = Union[torch.Tensor, Sequence[torch.Tensor]]


def _grouped(t: TensorOrList, G: int):
    """gl_grouped for a stacked tensor or a list of per-group tensors.

    Returns (struct, keepalive) -- keep the second value alive for the call.
    """
    if isinstance(t, torch.Tensor):
        assert t.is_contiguous() and t.shape[0] == G
        return GlGrouped(GL_STACKED, t.data_ptr(), None), None
    assert len(t) == G
    arr = (ctypes.c_void_p * G)(*[x.data_ptr() for x in t])
    return GlGrouped(GL_PER_GROUP, None, ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))), arr


def _shape_nk(w: TensorOrList):
    return tuple((w if isinstance(w, torch.Tensor) else w[0]).shape[-2:])


def _opts(pair: bool, wait_limit_us: int, flags: int = 0):
    """Per-call GEMM options (``gl_gemm_opts``); None for the defaults."""
    if pair and not wait_limit_us and not flags:
        return None
    return ctypes.pointer(GlGemmOpts(GL_TILES_PAIR if pair else GL_TILES_SINGLE, wait_limit_us, flags))


def gl_offsets(m_splits: torch.Tensor, expect_rows: int, out_rows: Optional[int] = None,
               offsets: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None):
    """Device prefix scan of ``m_splits`` (int64[G]) -> (offsets int64[G+1], status int32[1])."""
    G = m_splits.numel()
    dev = m_splits.device
    if offsets is None:
        offsets = torch.empty(G + 1, dtype=torch.int64, device=dev)
    if status is None:
        status = torch.empty(1, dtype=torch.int32, device=dev)
    out_rows = expect_rows if out_rows is None else out_rows
    _check(load().gl_offsets(m_splits.data_ptr(), G, expect_rows, out_rows, offsets.data_ptr(),
                             status.data_ptr(), _stream()), "gl_offsets")
    return offsets, status


def gl_fwd(x: torch.Tensor, w: TensorOrList, bias: Optional[TensorOrList], offsets: torch.Tensor,
           status: torch.Tensor, y: Optional[torch.Tensor] = None, pair: bool = True, wait_limit_us: int = 0, opt_flags: int = 0) -> torch.Tensor:
    """y rows of group g = x rows of group g @ W_g^T (+ b_g).  ``y`` may be a
    caller buffer with more rows than x; only the valid rows are written."""
    G = offsets.numel() - 1
    M, K = x.shape
    N, K2 = _shape_nk(w)
    assert K2 == K
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    wg, keep_w = _grouped(w, G)
    bptr = None
    keep_b = None
    if bias is not None:
        bg, keep_b = _grouped(bias, G)
        bptr = ctypes.pointer(bg)
    _check(load().gl_fwd(x.data_ptr(), wg, bptr, offsets.data_ptr(), status.data_ptr(), G, M, N, K,
                         y.data_ptr(), y.shape[0], _opts(pair, wait_limit_us, opt_flags), _stream()), "gl_fwd")
    del keep_w, keep_b
    return y


def gl_dgrad(dy: torch.Tensor, w: TensorOrList, offsets: torch.Tensor, status: torch.Tensor,
             dx: Optional[torch.Tensor] = None, pair: bool = True, wait_limit_us: int = 0, opt_flags: int = 0) -> torch.Tensor:
    """dx rows of group g = dy rows of group g @ W_g."""
    G = offsets.numel() - 1
    M, N = dy.shape
    N2, K = _shape_nk(w)
    assert N2 == N
    if dx is None:
        dx = torch.empty(M, K, dtype=torch.bfloat16, device=dy.device)
    wg, keep_w = _grouped(w, G)
    _check(load().gl_dgrad(dy.data_ptr(), wg, offsets.data_ptr(), status.data_ptr(), G, M, N, K,
                           dx.data_ptr(), dx.shape[0], _opts(pair, wait_limit_us, opt_flags), _stream()), "gl_dgrad")
    del keep_w
    return dx


def gl_wgrad(x: torch.Tensor, dy: torch.Tensor, offsets: torch.Tensor, status: torch.Tensor,
             main_grad: TensorOrList, accumulate: bool = True, pair: bool = True, wait_limit_us: int = 0, opt_flags: int = 0) -> TensorOrList:
    """main_grad[g] (+)= dy_g^T @ x_g (fp32)."""
    G = offsets.numel() - 1
    M, K = x.shape
    N = dy.shape[1]
    mg, keep = _grouped(main_grad, G)
    _check(load().gl_wgrad(x.data_ptr(), dy.data_ptr(), offsets.data_ptr(), status.data_ptr(), G,
                           M, N, K, mg, 1 if accumulate else 0, _opts(pair, wait_limit_us, opt_flags), _stream()), "gl_wgrad")
    del keep
    return main_grad


def gl_dbias(dy: torch.Tensor, offsets: torch.Tensor, status: torch.Tensor,
             dbias: Optional[TensorOrList] = None) -> TensorOrList:
    """Bias gradient: per group, the column sums of its rows of dy (bf16 out).
    ``dbias`` may be a [G, N] tensor or a list of G [N] tensors."""
    G = offsets.numel() - 1
    M, N = dy.shape
    if dbias is None:
        dbias = torch.empty(G, N, dtype=torch.bfloat16, device=dy.device)
    db, keep = _grouped(dbias, G)
    _check(load().gl_dbias(dy.data_ptr() if M > 0 else None, offsets.data_ptr(), status.data_ptr(), G, M, N, db,
                           _stream()), "gl_dbias")
    del keep
    return dbias


def mxfp8_scale_bytes(rows: int, cols: int, G: int, colwise: bool, mma: bool) -> int:
    """Bytes to allocate for a scale array (``gl_mxfp8_scale_bytes``)."""
    n = load().gl_mxfp8_scale_bytes(rows, cols, G, 1 if colwise else 0, GL_SCALES_MMA if mma else GL_SCALES_ROWMAJOR)
    if n == 0:
        raise GlError(f"gl_mxfp8_scale_bytes: invalid arguments ({rows}, {cols}, {G})")
    return n


def group_quantize_mxfp8(src: torch.Tensor, row_offsets: Optional[torch.Tensor] = None, G: int = 1,
                         rowwise: bool = True, colwise: bool = False,
                         status: Optional[torch.Tensor] = None, out: Optional[dict] = None,
                         mma_scales: bool = False) -> dict:
    """MXFP8 cast of a bf16 [rows, cols] tensor (rows in G groups).

    Returns a dict with ``codes_r``/``scales_r`` (blocks along each row) and/or
    ``codes_c``/``scales_c`` (blocks of 32 rows inside each group).  Scales are
    [rows, cols/32] and [ceil(rows/32) + G, cols] arrays, or with
    ``mma_scales`` flat byte arrays in the tcgen05 scale-factor layout that the
    MXFP8 GEMMs read (``GL_SCALES_MMA``).
    """
    src2, rows, cols, G = _cast_shape(src, row_offsets, G)
    out = _cast_outputs(src2, G, rowwise, colwise, out, mma_scales)
    _check(load().group_quantize_mxfp8(
        src2.data_ptr(), rows, cols, _ptr(row_offsets), G, _ptr(status),
        _ptr(out.get("codes_r")) if rowwise else None, _ptr(out.get("scales_r")) if rowwise else None,
        _ptr(out.get("codes_c")) if colwise else None, _ptr(out.get("scales_c")) if colwise else None,
        GL_SCALES_MMA if mma_scales else GL_SCALES_ROWMAJOR, _stream()), "group_quantize_mxfp8")
    return out


def _cast_shape(src: torch.Tensor, row_offsets: Optional[torch.Tensor], G: int):
    if src.dim() == 3:
        G = src.shape[0]
        src2 = src.reshape(-1, src.shape[-1])
    else:
        src2 = src
    if row_offsets is not None:
        G = row_offsets.numel() - 1
    rows, cols = src2.shape
    return src2, rows, cols, G


def _cast_outputs(src2: torch.Tensor, G: int, rowwise: bool, colwise: bool, out: Optional[dict],
                  mma_scales: bool) -> dict:
    rows, cols = src2.shape
    dev = src2.device
    out = {} if out is None else out

    def need(key, make):
        if key not in out:  # allocate only what the caller did not supply
            out[key] = make()

    if rowwise:
        need("codes_r", lambda: torch.empty(rows, cols, dtype=torch.uint8, device=dev))
        if mma_scales:
            need("scales_r", lambda: torch.empty(mxfp8_scale_bytes(rows, cols, G, False, True), dtype=torch.uint8,
                                                 device=dev))
        else:
            need("scales_r", lambda: torch.empty(rows, cols // 32, dtype=torch.uint8, device=dev))
    if colwise:
        need("codes_c", lambda: torch.empty(rows, cols, dtype=torch.uint8, device=dev))
        if mma_scales:
            need("scales_c", lambda: torch.empty(mxfp8_scale_bytes(rows, cols, G, True, True), dtype=torch.uint8,
                                                 device=dev))
        else:
            need("scales_c", lambda: torch.empty((rows + 31) // 32 + G, cols, dtype=torch.uint8, device=dev))
    return out


def dbias_workspace_bytes(rows: int, cols: int, G: int) -> int:
    """Workspace bytes of :func:`group_quantize_mxfp8_dbias` (``gl_dbias_workspace_bytes``)."""
    n = load().gl_dbias_workspace_bytes(rows, cols, G)
    if n == 0:
        raise GlError(f"gl_dbias_workspace_bytes: invalid arguments ({rows}, {cols}, {G})")
    return n


def group_quantize_mxfp8_dbias(dy: torch.Tensor, row_offsets: torch.Tensor, status: torch.Tensor,
                               rowwise: bool = True, colwise: bool = True, out: Optional[dict] = None,
                               mma_scales: bool = False, dbias: Optional[TensorOrList] = None,
                               workspace: Optional[torch.Tensor] = None):
    """:func:`group_quantize_mxfp8` of a ragged dy that also returns its bias
    gradient (per group, the column sums of its rows; bf16 [G, cols] or a list
    of G [cols] tensors) from the same pass.  ``workspace`` (uint8, at least
    :func:`dbias_workspace_bytes`, 256-byte aligned) is allocated when absent.
    Returns (codes/scales dict, dbias)."""
    src2, rows, cols, G = _cast_shape(dy, row_offsets, 1)
    out = _cast_outputs(src2, G, rowwise, colwise, out, mma_scales)
    if dbias is None:
        dbias = torch.empty(G, cols, dtype=torch.bfloat16, device=dy.device)
    nbytes = dbias_workspace_bytes(rows, cols, G)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dy.device)
    db, keep = _grouped(dbias, G)
    _check(load().group_quantize_mxfp8_dbias(
        src2.data_ptr(), rows, cols, row_offsets.data_ptr(), G, status.data_ptr(),
        _ptr(out.get("codes_r")) if rowwise else None, _ptr(out.get("scales_r")) if rowwise else None,
        _ptr(out.get("codes_c")) if colwise else None, _ptr(out.get("scales_c")) if colwise else None,
        GL_SCALES_MMA if mma_scales else GL_SCALES_ROWMAJOR, db, workspace.data_ptr(), workspace.numel(),
        _stream()), "group_quantize_mxfp8_dbias")
    del keep
    return out, dbias


# ---------------------------------------------------------------- MXFP8 GEMMs

def _grouped_any(t: TensorOrList, G: int):
    """gl_grouped for a stacked tensor (any leading shape) or a list of G tensors."""
    if isinstance(t, torch.Tensor):
        assert t.is_contiguous()
        return GlGrouped(GL_STACKED, t.data_ptr(), None), None
    assert len(t) == G
    arr = (ctypes.c_void_p * G)(*[x.data_ptr() for x in t])
    return GlGrouped(GL_PER_GROUP, None, ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))), arr


def gl_fwd_mxfp8(x_codes: torch.Tensor, x_scales: torch.Tensor, w_codes: TensorOrList, w_scales: TensorOrList,
                 bias: Optional[TensorOrList], offsets: torch.Tensor, status: torch.Tensor,
                 y: Optional[torch.Tensor] = None, pair: bool = True, wait_limit_us: int = 0, opt_flags: int = 0) -> torch.Tensor:
    """fprop on MXFP8 operands: x rowwise codes [M,K] + scale atoms; W rowwise
    codes [G,N,K] (or G x [N,K]) + scale atoms (all scales ``mma_scales``)."""
    G = offsets.numel() - 1
    M, K = x_codes.shape
    N = (w_codes if isinstance(w_codes, torch.Tensor) else w_codes[0]).shape[-2]
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=x_codes.device)
    wc, k1 = _grouped_any(w_codes, G)
    ws, k2 = _grouped_any(w_scales, G)
    bptr, k3 = None, None
    if bias is not None:
        bg, k3 = _grouped(bias, G)
        bptr = ctypes.pointer(bg)
    _check(load().gl_fwd_mxfp8(x_codes.data_ptr(), x_scales.data_ptr(), wc, ws, bptr, offsets.data_ptr(),
                               status.data_ptr(), G, M, N, K, y.data_ptr(), y.shape[0], _opts(pair, wait_limit_us, opt_flags), _stream()),
           "gl_fwd_mxfp8")
    del k1, k2, k3
    return y


def gl_dgrad_mxfp8(dy_codes: torch.Tensor, dy_scales: torch.Tensor, w_codes_c: TensorOrList,
                   w_scales_c: TensorOrList, offsets: torch.Tensor, status: torch.Tensor,
                   dx: Optional[torch.Tensor] = None, pair: bool = True, wait_limit_us: int = 0, opt_flags: int = 0) -> torch.Tensor:
    """dgrad on MXFP8 operands: dy rowwise codes [M,N] + scale atoms; W
    columnwise codes [G,N,K] + columnwise scale atoms."""
    G = offsets.numel() - 1
    M, N = dy_codes.shape
    K = (w_codes_c if isinstance(w_codes_c, torch.Tensor) else w_codes_c[0]).shape[-1]
    if dx is None:
        dx = torch.empty(M, K, dtype=torch.bfloat16, device=dy_codes.device)
    wc, k1 = _grouped_any(w_codes_c, G)
    ws, k2 = _grouped_any(w_scales_c, G)
    _check(load().gl_dgrad_mxfp8(dy_codes.data_ptr(), dy_scales.data_ptr(), wc, ws, offsets.data_ptr(),
                                 status.data_ptr(), G, M, N, K, dx.data_ptr(), dx.shape[0], _opts(pair, wait_limit_us, opt_flags), _stream()),
           "gl_dgrad_mxfp8")
    del k1, k2
    return dx


def gl_wgrad_mxfp8(x_codes_c: torch.Tensor, x_scales_c: torch.Tensor, dy_codes_c: torch.Tensor,
                   dy_scales_c: torch.Tensor, offsets: torch.Tensor, status: torch.Tensor,
                   main_grad: TensorOrList, accumulate: bool = True, pair: bool = True, wait_limit_us: int = 0, opt_flags: int = 0) -> TensorOrList:
    """wgrad on MXFP8 operands: x and dy columnwise codes + columnwise scale atoms."""
    G = offsets.numel() - 1
    M, K = x_codes_c.shape
    N = dy_codes_c.shape[1]
    mg, keep = _grouped(main_grad, G)
    _check(load().gl_wgrad_mxfp8(x_codes_c.data_ptr(), x_scales_c.data_ptr(), dy_codes_c.data_ptr(),
                                 dy_scales_c.data_ptr(), offsets.data_ptr(), status.data_ptr(), G, M, N, K, mg,
                                 1 if accumulate else 0, _opts(pair, wait_limit_us, opt_flags), _stream()), "gl_wgrad_mxfp8")
    del keep
    return main_grad
