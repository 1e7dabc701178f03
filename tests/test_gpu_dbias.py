"""gl_dbias on the GPU (through the C ABI) against the fp64 oracle.

The bias gradient of ``grouped_linear.py`` (ops/basic, fuser_backward): the
column sums of each split of grad_output.  fp32 accumulation and one bf16
rounding per output: relative Frobenius error <= 5e-3 per group; bit-exact in
the integer mode (sums of values in {-1, 0, 1} are exact); empty groups give
zeros; a non-zero status word blocks every write.
"""
import numpy as np
import pytest
import torch

from grouped_gemm_splits_b200 import gl, synth
from oracle import gl_oracle as orc
from tests.gpu_util import TOL_BF16, f64, offsets_on_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,m", [
    (256, [0, 96, 160, 256]),
    (1408, [5, 0, 33, 1000, 1]),
    (136, [300]),
    (512, [0, 0, 7, 0]),
])
@pytest.mark.parametrize("per_group", [False, True])
def test_dbias_small(N, m, per_group):
    G, M = len(m), int(sum(m))
    g = torch.Generator().manual_seed(N + M)
    dy = torch.randn(M, N, generator=g).to(torch.bfloat16).cuda()
    off, st = offsets_on_device(m, M)
    if per_group:
        out = [torch.full((N,), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
        gl.gl_dbias(dy, off, st, out)
        got = np.stack([f64(t) for t in out])
    else:
        got = f64(gl.gl_dbias(dy, off, st))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = orc.dbias(f64(dy), m)
    for i in range(G):
        if m[i] == 0:
            assert np.all(got[i] == 0.0)
        else:
            assert orc.rel_frobenius(got[i], ref[i]) <= TOL_BF16, i


def test_dbias_integer_mode_bit_exact():
    m = [0, 100, 156, 300]
    G, M, N = len(m), sum(m), 264
    d = synth.integer_operands(G, M, N, 128, seed=5)
    dy = d["dy"].cuda()
    off, st = offsets_on_device(m, M)
    got = gl.gl_dbias(dy, off, st)
    torch.cuda.synchronize()
    assert np.array_equal(synth.bf16_bits(got), orc.f64_to_bf16_rne(orc.dbias(f64(dy), m)))


def test_dbias_bad_splits_write_nothing():
    M, N = 64, 128
    dy = torch.ones(M, N, dtype=torch.bfloat16, device="cuda")
    off, st = offsets_on_device([40, 40], M)  # sums to 80 != 64
    out = torch.full((2, N), 7.0, dtype=torch.bfloat16, device="cuda")
    gl.gl_dbias(dy, off, st, out)
    torch.cuda.synchronize()
    assert int(st.item()) != 0
    assert bool((out == 7.0).all().item())


def test_dbias_full_size_bf16_g8():
    """The bf16_g8 shapes (16384 x 14336, G=8), every group against the oracle."""
    wl = synth.WORKLOADS["bf16_g8"]
    m = synth.m_splits_for("bf16_g8")
    d = synth.operands(wl.G, wl.rows, wl.N, wl.K, wl.seed, device="cuda", bias=False)
    off, st = offsets_on_device(m, wl.rows)
    got = f64(gl.gl_dbias(d["dy"], off, st))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = orc.dbias(f64(d["dy"]), m)
    for i in range(wl.G):
        assert orc.rel_frobenius(got[i], ref[i]) <= TOL_BF16, i
