"""The C-ABI library builds, loads and exports every entry point declared in
include/gl.h; host-side argument checks answer without a GPU."""
import ctypes
import os
import re

import pytest

from grouped_gemm_splits_b200 import gl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "gl.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:gl_status|int|size_t|const char\*)\s+(\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol():
    lib = gl.load()
    names = _declared()
    assert "gl_fwd" in names and "group_quantize_mxfp8" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(gl.EXPORTED) <= set(names)


def test_version_and_status_strings():
    lib = gl.load()
    assert lib.gl_version() >= 100
    assert lib.gl_status_string(gl.GL_ERR_INVALID) == b"invalid argument"


def test_host_side_validation_without_gpu():
    """Invalid arguments are rejected before any CUDA call is made."""
    lib = gl.load()
    w = gl.GlGrouped(gl.GL_STACKED, 16, None)
    # G <= 0, N/K <= 0: ValueError analogues of GroupedLinear's constructor checks
    assert lib.gl_fwd(16, w, None, 16, 16, 0, 8, 8, 8, 16, 8, None, None) == gl.GL_ERR_INVALID
    assert lib.gl_fwd(16, w, None, 16, 16, 2, 8, 0, 8, 16, 8, None, None) == gl.GL_ERR_INVALID
    # N % 8 != 0: unsupported row pitch
    assert lib.gl_fwd(16, w, None, 16, 16, 2, 8, 12, 8, 16, 8, None, None) == gl.GL_ERR_UNSUPPORTED
    # caller buffer with fewer rows than the input
    assert lib.gl_fwd(16, w, None, 16, 16, 2, 8, 8, 8, 16, 7, None, None) == gl.GL_ERR_INVALID
    # more groups than the kernels take
    assert lib.gl_fwd(16, w, None, 16, 16, 4097, 8, 8, 8, 16, 8, None, None) == gl.GL_ERR_INVALID
    assert lib.gl_offsets(16, 4097, 8, 8, 16, 16, None) == gl.GL_ERR_INVALID
    assert lib.gl_fwd_mxfp8(16, 16, w, w, None, 16, 16, 2049, 8, 128, 128, 16, 8, None, None) == gl.GL_ERR_INVALID
    # null pointers
    assert lib.gl_fwd(None, w, None, 16, 16, 2, 8, 8, 8, 16, 8, None, None) == gl.GL_ERR_INVALID
    assert lib.gl_dgrad(16, w, 16, None, 2, 8, 8, 8, 16, 8, None, None) == gl.GL_ERR_INVALID
    assert lib.gl_wgrad(16, 16, 16, 16, 2, 8, 8, 8, gl.GlGrouped(gl.GL_STACKED, None, None), 1, None, None) == gl.GL_ERR_INVALID
    assert lib.gl_offsets(None, 4, 8, 8, 16, 16, None) == gl.GL_ERR_INVALID
    assert lib.gl_offsets(16, 0, 8, 8, 16, 16, None) == gl.GL_ERR_INVALID
    # per-group mode with a null member pointer
    arr = (ctypes.c_void_p * 2)(16, None)
    pg = gl.GlGrouped(gl.GL_PER_GROUP, None, ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)))
    assert lib.gl_fwd(16, pg, None, 16, 16, 2, 8, 8, 8, 16, 8, None, None) == gl.GL_ERR_INVALID
    # quantize: cols not a multiple of 32; no output requested
    assert lib.group_quantize_mxfp8(16, 8, 48, None, 1, None, 16, 16, None, None, 0, None) == gl.GL_ERR_UNSUPPORTED
    assert lib.group_quantize_mxfp8(16, 8, 64, None, 1, None, None, None, None, None, 0, None) == gl.GL_ERR_INVALID
    assert lib.group_quantize_mxfp8(16, 9, 64, None, 2, None, 16, 16, None, None, 0, None) == gl.GL_ERR_INVALID
    # dbias: G <= 0, null status, N % 8 != 0
    st = gl.GlGrouped(gl.GL_STACKED, 16, None)
    assert lib.gl_dbias(16, 16, 16, 0, 8, 8, st, None) == gl.GL_ERR_INVALID
    assert lib.gl_dbias(16, 16, None, 2, 8, 8, st, None) == gl.GL_ERR_INVALID
    assert lib.gl_dbias(16, 16, 16, 2, 8, 12, st, None) == gl.GL_ERR_UNSUPPORTED
    # MMA-layout scales need cols % 128 == 0; unknown layout codes are rejected
    assert lib.group_quantize_mxfp8(16, 8, 96, None, 1, None, 16, 16, None, None, 1, None) == gl.GL_ERR_UNSUPPORTED
    assert lib.group_quantize_mxfp8(16, 8, 128, None, 1, None, 16, 16, None, None, 7, None) == gl.GL_ERR_INVALID


def test_gemm_options_are_checked():
    """Per-call GEMM options: tile choices and wait bounds the header does not
    define are refused before any launch; the defaults (NULL) are accepted."""
    lib = gl.load()
    w = gl.GlGrouped(gl.GL_STACKED, 16, None)
    bad_tiles = ctypes.pointer(gl.GlGemmOpts(7, 0))
    too_long = ctypes.pointer(gl.GlGemmOpts(gl.GL_TILES_PAIR, 2000001, 0))
    bad_flags = ctypes.pointer(gl.GlGemmOpts(gl.GL_TILES_PAIR, 0, 6))
    for o in (bad_tiles, too_long, bad_flags):
        assert lib.gl_fwd(16, w, None, 16, 16, 2, 8, 8, 8, 16, 8, o, None) == gl.GL_ERR_INVALID
        assert lib.gl_dgrad(16, w, 16, 16, 2, 8, 8, 8, 16, 8, o, None) == gl.GL_ERR_INVALID
        assert lib.gl_wgrad(16, 16, 16, 16, 2, 8, 8, 8, w, 1, o, None) == gl.GL_ERR_INVALID
        assert lib.gl_fwd_mxfp8(16, 16, w, w, None, 16, 16, 2, 8, 128, 128, 16, 8, o, None) == gl.GL_ERR_INVALID
        assert lib.gl_dgrad_mxfp8(16, 16, w, w, 16, 16, 2, 8, 128, 128, 16, 8, o, None) == gl.GL_ERR_INVALID
        assert lib.gl_wgrad_mxfp8(16, 16, 16, 16, 16, 16, 2, 8, 128, 128, w, 1, o, None) == gl.GL_ERR_INVALID
    # no rows: valid options (and NULL) return before any launch
    ok = ctypes.pointer(gl.GlGemmOpts(gl.GL_TILES_SINGLE, 1, gl.GL_OPT_HOLD_LOADS))
    for o in (None, ok):
        assert lib.gl_fwd(16, w, None, 16, 16, 2, 0, 8, 8, 16, 0, o, None) == gl.GL_OK
        assert lib.gl_dgrad(16, w, 16, 16, 2, 0, 8, 8, 16, 0, o, None) == gl.GL_OK


def test_fused_cast_dbias_validation_and_workspace_size():
    """group_quantize_mxfp8_dbias rejects what it cannot do before any CUDA
    call; its workspace is int64[G+1] block offsets padded to 256 bytes plus
    fp32 [ceil(rows/32) + G, cols] block partials."""
    lib = gl.load()
    assert lib.gl_dbias_workspace_bytes(100, 64, 3) == 256 + (4 + 3) * 64 * 4
    assert lib.gl_dbias_workspace_bytes(0, 64, 40) == 512 + 40 * 64 * 4
    assert lib.gl_dbias_workspace_bytes(100, 0, 3) == 0
    assert lib.gl_dbias_workspace_bytes(100, 64, 0) == 0
    db = gl.GlGrouped(gl.GL_STACKED, 16, None)
    ws = lib.gl_dbias_workspace_bytes(64, 128, 2)
    f = lib.group_quantize_mxfp8_dbias
    # row offsets, status and workspace are required
    assert f(16, 64, 128, None, 2, 16, 16, 16, None, None, 0, db, 256, ws, None) == gl.GL_ERR_INVALID
    assert f(16, 64, 128, 16, 2, None, 16, 16, None, None, 0, db, 256, ws, None) == gl.GL_ERR_INVALID
    assert f(16, 64, 128, 16, 2, 16, 16, 16, None, None, 0, db, None, ws, None) == gl.GL_ERR_INVALID
    # workspace too small / not 256-byte aligned
    assert f(16, 64, 128, 16, 2, 16, 16, 16, None, None, 0, db, 256, ws - 1, None) == gl.GL_ERR_INVALID
    assert f(16, 64, 128, 16, 2, 16, 16, 16, None, None, 0, db, 272, ws, None) == gl.GL_ERR_UNSUPPORTED
    # dbias output missing; the cast's own checks still apply
    assert f(16, 64, 128, 16, 2, 16, 16, 16, None, None, 0, gl.GlGrouped(gl.GL_STACKED, None, None), 256, ws,
             None) == gl.GL_ERR_INVALID
    assert f(16, 64, 48, 16, 2, 16, 16, 16, None, None, 0, db, 256, ws, None) == gl.GL_ERR_UNSUPPORTED


def test_scale_bytes_helper():
    """Sizes of the scale arrays (host only): row-major [rows, cols/32] and
    [ceil(rows/32) + G, cols]; MMA layout in 512-byte atoms of 128 rows x 4
    blocks, columnwise bounded by ceil(rows/128) + G k-groups."""
    lib = gl.load()
    assert lib.gl_mxfp8_scale_bytes(100, 64, 3, 0, gl.GL_SCALES_ROWMAJOR) == 100 * 2
    assert lib.gl_mxfp8_scale_bytes(100, 64, 3, 1, gl.GL_SCALES_ROWMAJOR) == (4 + 3) * 64
    assert lib.gl_mxfp8_scale_bytes(300, 256, 3, 0, gl.GL_SCALES_MMA) == 3 * 2 * 512
    assert lib.gl_mxfp8_scale_bytes(300, 256, 3, 1, gl.GL_SCALES_MMA) == (3 + 3) * 2 * 512
    assert lib.gl_mxfp8_scale_bytes(300, 96, 3, 0, gl.GL_SCALES_MMA) == 0   # cols % 128 != 0
    assert lib.gl_mxfp8_scale_bytes(300, 256, 0, 0, gl.GL_SCALES_MMA) == 0  # G <= 0
    assert lib.gl_mxfp8_scale_bytes(300, 256, 1, 0, 5) == 0                 # unknown layout
    assert lib.gl_mxfp8_scale_bytes(0, 128, 1, 1, gl.GL_SCALES_MMA) == 1 * 512


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(gl, "_lib", None)
    monkeypatch.setattr(gl, "_LIB_PATH", str(tmp_path / "libgl.so"))
    with pytest.raises(gl.GlError):
        gl.load()
