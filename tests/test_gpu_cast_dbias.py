"""group_quantize_mxfp8_dbias on the GPU (through the C ABI): the MXFP8 cast
of dy and its bias gradient in one pass.

``grouped_linear.py`` (ops/basic, fuser_backward) quantizes grad_output per
split and, with a bias, sums each split over its rows.  The fused call must
give exactly the codes and scales of group_quantize_mxfp8, and a bias
gradient within the gl_dbias bound of the fp64 oracle (relative Frobenius
error <= 5e-3 per group; bit-exact in the integer mode, where every partial
sum is exact); empty groups give zeros, a non-zero status word blocks every
write, and two calls give bit-identical results (fixed summation order).
"""
import numpy as np
import pytest
import torch

from grouped_gemm_splits_b200 import gl, synth
from oracle import gl_oracle as orc
from tests.gpu_util import TOL_BF16, f64, offsets_on_device

pytestmark = pytest.mark.gpu

KEYS = ("codes_r", "scales_r", "codes_c", "scales_c")


def _prefilled(M, N, G, mma, fill=0x5A):
    """Output buffers holding the same bytes everywhere, so that the bytes a
    cast leaves unwritten (scale rows of blocks that do not exist) compare
    equal too."""
    def scales(colwise):
        if mma:
            return (gl.mxfp8_scale_bytes(M, N, G, colwise, True),)
        return ((M + 31) // 32 + G, N) if colwise else (M, N // 32)
    shapes = {"codes_r": (M, N), "codes_c": (M, N), "scales_r": scales(False), "scales_c": scales(True)}
    return {k: torch.full(v, fill, dtype=torch.uint8, device="cuda") for k, v in shapes.items()}


def _check_against_cast(dy, off, st, out, mma):
    M, N = dy.shape
    ref = gl.group_quantize_mxfp8(dy, off, rowwise=True, colwise=True, status=st, mma_scales=mma,
                                  out=_prefilled(M, N, off.numel() - 1, mma))
    torch.cuda.synchronize()
    for k in KEYS:
        assert torch.equal(out[k], ref[k]), k


@pytest.mark.parametrize("N,m", [
    (256, [0, 96, 160, 256]),
    (1408, [5, 0, 33, 1000, 1]),
    (128, [300]),
    (512, [0, 0, 7, 0]),
    (384, [31, 32, 33, 64, 65]),
])
@pytest.mark.parametrize("mma", [False, True])
def test_cast_dbias_small(N, m, mma):
    G, M = len(m), int(sum(m))
    g = torch.Generator().manual_seed(N + M + 7)
    dy = (torch.randn(M, N, generator=g) * 3.0).to(torch.bfloat16).cuda()
    off, st = offsets_on_device(m, M)
    out, db = gl.group_quantize_mxfp8_dbias(dy, off, st, mma_scales=mma, out=_prefilled(M, N, G, mma))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _check_against_cast(dy, off, st, out, mma)
    got = f64(db)
    ref = orc.dbias(f64(dy), m)
    for i in range(G):
        if m[i] == 0:
            assert np.all(got[i] == 0.0)
        else:
            assert orc.rel_frobenius(got[i], ref[i]) <= TOL_BF16, i


def test_cast_dbias_rowwise_only_and_per_group_outputs():
    m = [40, 0, 200, 17]
    G, M, N = len(m), sum(m), 256
    g = torch.Generator().manual_seed(11)
    dy = torch.randn(M, N, generator=g).to(torch.bfloat16).cuda()
    off, st = offsets_on_device(m, M)
    outs = [torch.full((N,), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    out, _ = gl.group_quantize_mxfp8_dbias(dy, off, st, rowwise=True, colwise=False, dbias=outs)
    ref_cast = gl.group_quantize_mxfp8(dy, off, rowwise=True, colwise=False, status=st)  # rowwise: all written
    torch.cuda.synchronize()
    assert torch.equal(out["codes_r"], ref_cast["codes_r"]) and torch.equal(out["scales_r"], ref_cast["scales_r"])
    ref = orc.dbias(f64(dy), m)
    for i in range(G):
        got = f64(outs[i])
        if m[i] == 0:
            assert np.all(got == 0.0)
        else:
            assert orc.rel_frobenius(got, ref[i]) <= TOL_BF16, i


def test_cast_dbias_integer_mode_bit_exact():
    m = [0, 100, 156, 300]
    G, M, N = len(m), sum(m), 256
    d = synth.integer_operands(G, M, N, 128, seed=5)
    dy = d["dy"].cuda()
    off, st = offsets_on_device(m, M)
    _, db = gl.group_quantize_mxfp8_dbias(dy, off, st)
    torch.cuda.synchronize()
    assert np.array_equal(synth.bf16_bits(db), orc.f64_to_bf16_rne(orc.dbias(f64(dy), m)))


def test_cast_dbias_bad_splits_write_nothing():
    M, N = 64, 128
    dy = torch.ones(M, N, dtype=torch.bfloat16, device="cuda")
    off, st = offsets_on_device([40, 40], M)  # sums to 80 != 64
    out = {k: torch.full((M, N) if k.startswith("codes") else (gl.mxfp8_scale_bytes(M, N, 2, k == "scales_c", True),),
                         7, dtype=torch.uint8, device="cuda") for k in KEYS}
    db = torch.full((2, N), 7.0, dtype=torch.bfloat16, device="cuda")
    gl.group_quantize_mxfp8_dbias(dy, off, st, out=out, mma_scales=True, dbias=db)
    torch.cuda.synchronize()
    assert int(st.item()) != 0
    assert bool((db == 7.0).all().item())
    for k in KEYS:
        assert bool((out[k] == 7).all().item()), k


def test_cast_dbias_full_size_bf16_g8_repeatable():
    """The bf16_g8 dy (16384 x 14336, G=8): codes and scales equal the plain
    cast's, every group's bias gradient within the bound, and a second call
    on a dirty workspace gives the same bits."""
    wl = synth.WORKLOADS["bf16_g8"]
    m = synth.m_splits_for("bf16_g8")
    d = synth.operands(wl.G, wl.rows, wl.N, wl.K, wl.seed, device="cuda", bias=False)
    dy = d["dy"]
    off, st = offsets_on_device(m, wl.rows)
    ws = torch.full((gl.dbias_workspace_bytes(wl.rows, wl.N, wl.G),), 0xFF, dtype=torch.uint8, device="cuda")
    out, db = gl.group_quantize_mxfp8_dbias(dy, off, st, mma_scales=True, workspace=ws,
                                            out=_prefilled(wl.rows, wl.N, wl.G, True))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _check_against_cast(dy, off, st, out, True)
    got = f64(db)
    ref = orc.dbias(f64(dy), m)
    for i in range(wl.G):
        assert orc.rel_frobenius(got[i], ref[i]) <= TOL_BF16, i
    _, db2 = gl.group_quantize_mxfp8_dbias(dy, off, st, mma_scales=True, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(db, db2)


def test_many_groups_per_group_outputs():
    """130 groups with per-group bias-gradient pointers: the reduction runs in
    launches of 64 groups; the fused call and gl_dbias both match the oracle,
    including the empty groups."""
    rng = np.random.default_rng(130)
    m = rng.integers(0, 40, size=130)
    m[[3, 64, 65, 129]] = 0
    G, M, N = len(m), int(m.sum()), 256
    g = torch.Generator().manual_seed(130)
    dy = torch.randn(M, N, generator=g).to(torch.bfloat16).cuda()
    off, st = offsets_on_device(m, M)
    fused = [torch.full((N,), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    alone = [torch.full((N,), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    gl.group_quantize_mxfp8_dbias(dy, off, st, mma_scales=True, dbias=fused)
    gl.gl_dbias(dy, off, st, alone)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = orc.dbias(f64(dy), m)
    for i in range(G):
        for t in (fused[i], alone[i]):
            got = f64(t)
            if m[i] == 0:
                assert np.all(got == 0.0), i
            else:
                assert orc.rel_frobenius(got, ref[i]) <= TOL_BF16, i
