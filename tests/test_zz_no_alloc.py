"""group_quantize_mxfp8_dbias_noalloc through the C ABI.

The entry point serves callers that cannot allocate device memory where they
call it (their memory belongs to another runtime's pool and they are handed
no allocator): it runs the fused MXFP8 cast + bias gradient with the
library's own fixed 16 MiB scratch array instead of a caller workspace.  Two
calls in a row must give what group_quantize_mxfp8_dbias gives with a
workspace: the same codes and scales, and bias gradients within the tests'
bf16 bound; a call whose scratch would exceed 16 MiB is refused.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from grouped_gemm_splits_b200 import gl
from oracle import gl_oracle as orc
from tests.gpu_util import TOL_BF16, f64, offsets_on_device

pytestmark = pytest.mark.gpu

KEYS = ("codes_r", "scales_r", "codes_c", "scales_c")


def _entry():
    f = gl.load().group_quantize_mxfp8_dbias_noalloc
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    f.restype = i32
    f.argtypes = [vp, i64, i32, vp, i32, vp, vp, vp, vp, vp, i32, gl.GlGrouped, vp]
    return f


def _outputs(M, N, G, fill):
    shapes = {"codes_r": (M, N), "codes_c": (M, N), "scales_r": (gl.mxfp8_scale_bytes(M, N, G, False, True),),
              "scales_c": (gl.mxfp8_scale_bytes(M, N, G, True, True),)}
    return {k: torch.full(v, fill, dtype=torch.uint8, device="cuda") for k, v in shapes.items()}


def test_noalloc_matches_workspace_entry_two_calls():
    m = [700, 0, 2048, 33, 3000, 5]
    G, M, N = len(m), sum(m), 2048
    g = torch.Generator().manual_seed(2024)
    dy = (torch.randn(M, N, generator=g) * 2.0).to(torch.bfloat16).cuda()
    off, st = offsets_on_device(m, M)
    ref, ref_db = gl.group_quantize_mxfp8_dbias(dy, off, st, mma_scales=True, out=_outputs(M, N, G, 0x33))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    f = _entry()
    oracle_db = orc.dbias(f64(dy), m)
    for call in range(2):
        out = _outputs(M, N, G, 0x33)
        db = torch.full((G, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        grouped = gl.GlGrouped(gl.GL_STACKED, db.data_ptr(), None)
        rc = f(dy.data_ptr(), M, N, off.data_ptr(), G, st.data_ptr(), out["codes_r"].data_ptr(),
               out["scales_r"].data_ptr(), out["codes_c"].data_ptr(), out["scales_c"].data_ptr(),
               gl.GL_SCALES_MMA, grouped, torch.cuda.current_stream().cuda_stream)
        assert rc == gl.GL_OK, (call, rc)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for k in KEYS:
            assert torch.equal(out[k], ref[k]), (call, k)
        got, want = f64(db), f64(ref_db)
        for i in range(G):
            if m[i] == 0:
                assert np.all(got[i] == 0.0), (call, i)
            else:
                assert orc.rel_frobenius(got[i], want[i]) <= TOL_BF16, (call, i)
                assert orc.rel_frobenius(got[i], oracle_db[i]) <= TOL_BF16, (call, i)


def _call(f, dy, M, N, G, off, st, out, db_grouped):
    return f(dy.data_ptr(), M, N, off.data_ptr(), G, st.data_ptr(), out["codes_r"].data_ptr(),
             out["scales_r"].data_ptr(), out["codes_c"].data_ptr(), out["scales_c"].data_ptr(),
             gl.GL_SCALES_MMA, db_grouped, torch.cuda.current_stream().cuda_stream)


def test_noalloc_at_its_documented_limit():
    """9088 rows x 14336 columns in 8 groups needs 16,744,704 bytes of
    scratch, the documented limit's example: the block partials then reach
    the end of the array.  Same results as the workspace entry point (codes
    and scales bit for bit) and as the oracle's bias gradient, on two calls."""
    m = [1500, 0, 2011, 777, 3000, 33, 1767, 0]
    G, M, N = len(m), sum(m), 14336
    assert M == 9088 and gl.dbias_workspace_bytes(M, N, G) == 16744704
    g = torch.Generator().manual_seed(9088)
    dy = torch.randn(M, N, generator=g).to(torch.bfloat16).cuda()
    off, st = offsets_on_device(m, M)
    ref, ref_db = gl.group_quantize_mxfp8_dbias(dy, off, st, mma_scales=True, out=_outputs(M, N, G, 0x5A))
    torch.cuda.synchronize()
    oracle_db = orc.dbias(f64(dy), m)
    f = _entry()
    for call in range(2):
        out = _outputs(M, N, G, 0x5A)
        db = torch.full((G, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = _call(f, dy, M, N, G, off, st, out, gl.GlGrouped(gl.GL_STACKED, db.data_ptr(), None))
        assert rc == gl.GL_OK, (call, rc)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for k in KEYS:
            assert torch.equal(out[k], ref[k]), (call, k)
        got = f64(db)
        for i in range(G):
            if m[i] == 0:
                assert np.all(got[i] == 0.0), (call, i)
            else:
                assert orc.rel_frobenius(got[i], f64(ref_db)[i]) <= TOL_BF16, (call, i)
                assert orc.rel_frobenius(got[i], oracle_db[i]) <= TOL_BF16, (call, i)


def test_noalloc_per_group_bias_gradient():
    """dbias given as G separate [N] tensors (GL_PER_GROUP)."""
    m = [64, 0, 300, 17]
    G, M, N = len(m), sum(m), 512
    g = torch.Generator().manual_seed(512)
    dy = torch.randn(M, N, generator=g).to(torch.bfloat16).cuda()
    off, st = offsets_on_device(m, M)
    ref, _ = gl.group_quantize_mxfp8_dbias(dy, off, st, mma_scales=True, out=_outputs(M, N, G, 0))
    dbs = [torch.full((N,), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    arr = (ctypes.c_void_p * G)(*[t.data_ptr() for t in dbs])
    grouped = gl.GlGrouped(gl.GL_PER_GROUP, None, ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)))
    out = _outputs(M, N, G, 0)
    assert _call(_entry(), dy, M, N, G, off, st, out, grouped) == gl.GL_OK
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for k in KEYS:
        assert torch.equal(out[k], ref[k]), k
    oracle_db = orc.dbias(f64(dy), m)
    for i in range(G):
        got = f64(dbs[i])
        if m[i] == 0:
            assert np.all(got == 0.0), i
        else:
            assert orc.rel_frobenius(got, oracle_db[i]) <= TOL_BF16, i


def test_noalloc_refuses_more_than_its_scratch():
    """rows x cols whose workspace exceeds 16 MiB: refused before any work;
    with an invalid argument as well, the argument error is reported first."""
    f = _entry()
    M, N, G = 9120, 14336, 8  # needs 16.8 MB of scratch
    assert gl.dbias_workspace_bytes(M, N, G) > 16 << 20
    db = gl.GlGrouped(gl.GL_STACKED, 16, None)
    rc = f(16, M, N, 16, G, 16, 16, 16, 16, 16, gl.GL_SCALES_MMA, db, None)
    assert rc == gl.GL_ERR_UNSUPPORTED
    rc = f(16, M, N, None, G, 16, 16, 16, 16, 16, gl.GL_SCALES_MMA, db, None)  # no row offsets
    assert rc == gl.GL_ERR_INVALID
    rc = f(16, M, N, 16, G, None, 16, 16, 16, 16, gl.GL_SCALES_MMA, db, None)  # no status word
    assert rc == gl.GL_ERR_INVALID
