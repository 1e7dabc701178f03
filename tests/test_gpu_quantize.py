"""group_quantize_mxfp8 on the GPU against the oracle: codes and scales
bit-exact, rowwise and columnwise, ragged groups (each split quantized as its
own tensor) and equal groups (a stacked weight)."""
import numpy as np
import pytest
import torch

from grouped_gemm_splits_b200 import gl, synth
from oracle import gl_oracle as orc
from tests.gpu_util import f64

pytestmark = pytest.mark.gpu


def _check(src_bf16, m, got, rowwise=True, colwise=True):
    src = f64(src_bf16)
    if rowwise:
        c, s = orc.quantize_rowwise(src)
        assert np.array_equal(got["codes_r"].cpu().numpy(), c)
        assert np.array_equal(got["scales_r"].cpu().numpy(), s)
    if colwise:
        c, s = orc.quantize_colwise(src, m)
        assert np.array_equal(got["codes_c"].cpu().numpy(), c)
        assert np.array_equal(got["scales_c"][: s.shape[0]].cpu().numpy(), s)


@pytest.mark.parametrize("m,cols", [
    ([0, 96, 160, 256], 128),
    ([5, 40, 0, 33, 300, 1], 288),
    ([1000], 64),
    ([31, 32, 33, 0, 64, 65], 544),
])
def test_ragged_groups_bit_exact(m, cols):
    rows = sum(m)
    g = torch.Generator().manual_seed(rows + cols)
    scale = torch.exp(torch.empty(rows, 1).uniform_(-8, 8, generator=g))
    src = (torch.randn(rows, cols, generator=g) * scale).to(torch.bfloat16).cuda()
    off, st = gl.gl_offsets(torch.tensor(m, dtype=torch.int64, device="cuda"), rows)
    got = gl.group_quantize_mxfp8(src, off, rowwise=True, colwise=True, status=st)
    torch.cuda.synchronize()
    _check(src, m, got)


@pytest.mark.parametrize("m,cols", [([0, 96, 160, 256], 128), ([5, 123, 0, 2], 384), ([130, 1, 257], 256)])
def test_mma_layout_scales(m, cols):
    """Scales in the tcgen05 scale-factor layout: every byte the oracle places
    (its own offset functions) equals the oracle's scale; codes unchanged."""
    rows = sum(m)
    g = torch.Generator().manual_seed(cols + rows)
    scale = torch.exp(torch.empty(rows, 1).uniform_(-6, 6, generator=g))
    src = (torch.randn(rows, cols, generator=g) * scale).to(torch.bfloat16).cuda()
    off, st = gl.gl_offsets(torch.tensor(m, dtype=torch.int64, device="cuda"), rows)
    got = gl.group_quantize_mxfp8(src, off, rowwise=True, colwise=True, status=st, mma_scales=True)
    torch.cuda.synchronize()
    assert got["scales_r"].numel() == ((rows + 127) // 128) * (cols // 128) * 512
    assert got["scales_c"].numel() == ((rows + 127) // 128 + len(m)) * (cols // 128) * 512
    c, s = orc.quantize_rowwise(f64(src))
    assert np.array_equal(got["codes_r"].cpu().numpy(), c)
    assert np.array_equal(got["scales_r"].cpu().numpy()[orc.mma_offsets_rowwise(rows, cols)], s)
    cc, sc = orc.quantize_colwise(f64(src), m)
    assert np.array_equal(got["codes_c"].cpu().numpy(), cc)
    assert np.array_equal(got["scales_c"].cpu().numpy()[orc.mma_offsets_colwise(m, cols)], sc)


def test_mma_layout_equal_groups():
    """A stacked weight (equal groups, no offsets array) in the MMA layout:
    member i owns k-groups i * ceil(rows_i / 128) onwards."""
    G, R, C = 3, 256, 256
    w = torch.randn(G, R, C, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).cuda()
    got = gl.group_quantize_mxfp8(w, rowwise=True, colwise=True, mma_scales=True)
    torch.cuda.synchronize()
    src = f64(w.reshape(G * R, C))
    _, s = orc.quantize_rowwise(src)
    assert np.array_equal(got["scales_r"].cpu().numpy()[orc.mma_offsets_rowwise(G * R, C)], s)
    _, sc = orc.quantize_colwise(src, [R] * G)
    assert np.array_equal(got["scales_c"].cpu().numpy()[orc.mma_offsets_colwise([R] * G, C)], sc)


def test_every_bf16_value_bit_exact():
    """All 65536 bf16 patterns (finite ones), each alone in a 32-element block."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = orc.bf16_to_f64(bits)
    bits = bits[np.isfinite(vals)]
    n = len(bits)
    src = np.zeros((n, 32), dtype=np.uint16)
    src[:, 7] = bits
    t = torch.from_numpy(src.view(np.int16)).view(torch.bfloat16).cuda()
    got = gl.group_quantize_mxfp8(t, rowwise=True, colwise=False)
    torch.cuda.synchronize()
    _check(t, [n], got, colwise=False)


def test_equal_groups_stacked_weight():
    """Rows split into G equal members without an offsets array: member i's
    columnwise blocks start at its first row and its scale rows at
    i * ceil(rows_i / 32)."""
    G, R, C = 6, 100, 96
    w = torch.randn(G, R, C, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).cuda()
    got = gl.group_quantize_mxfp8(w, rowwise=True, colwise=True)
    torch.cuda.synchronize()
    _check(w.reshape(G * R, C), [R] * G, got)


def test_status_blocks_writes():
    src = torch.randn(64, 64).to(torch.bfloat16).cuda()
    off, st = gl.gl_offsets(torch.tensor([32, 33], dtype=torch.int64, device="cuda"), 64)
    out = {"codes_r": torch.full((64, 64), 7, dtype=torch.uint8, device="cuda"),
           "scales_r": torch.full((64, 2), 7, dtype=torch.uint8, device="cuda")}
    gl.group_quantize_mxfp8(src, off, rowwise=True, colwise=False, status=st, out=out)
    torch.cuda.synchronize()
    assert int(st.item()) != 0
    assert bool((out["codes_r"] == 7).all()) and bool((out["scales_r"] == 7).all())


@pytest.mark.parametrize("which", ["x", "dy", "w"])
def test_full_size_sampled_blocks(which):
    """The MXFP8 workload's operands (G=8, K=4096, N=14336, 16384 rows) at full
    size; every 32-row block of a random sample is checked bit for bit."""
    wl = synth.WORKLOADS["mxfp8_g8"]
    m = synth.m_splits_for("mxfp8_g8")
    gen = torch.Generator(device="cuda").manual_seed(wl.seed)
    if which == "x":
        src = torch.randn(wl.rows, wl.K, generator=gen, device="cuda").to(torch.bfloat16)
        groups = m
    elif which == "dy":
        src = torch.randn(wl.rows, wl.N, generator=gen, device="cuda").to(torch.bfloat16)
        groups = m
    else:
        src = (torch.rand(wl.G * wl.N, wl.K, generator=gen, device="cuda") - 0.5).to(torch.bfloat16) / 32
        groups = [wl.N] * wl.G
    rows, cols = src.shape
    if which == "w":
        got = gl.group_quantize_mxfp8(src.view(wl.G, wl.N, wl.K), rowwise=True, colwise=True)
    else:
        off, st = gl.gl_offsets(torch.tensor(groups, dtype=torch.int64, device="cuda"), rows)
        got = gl.group_quantize_mxfp8(src, off, rowwise=True, colwise=True, status=st)
    torch.cuda.synchronize()
    o = orc.offsets(groups)
    base = orc.colwise_scale_rows(groups)
    rng = np.random.default_rng(0)
    for _ in range(24):
        g = int(rng.integers(len(groups)))
        if groups[g] == 0:
            continue
        j = int(rng.integers((groups[g] + 31) // 32))
        r0 = int(o[g]) + 32 * j
        r1 = min(r0 + 32, int(o[g + 1]))
        c0 = int(rng.integers(0, cols // 256)) * 256
        blk = f64(src[r0:r1, c0:c0 + 256])
        c, s = orc.quantize_rowwise(blk)
        assert np.array_equal(got["codes_r"][r0:r1, c0:c0 + 256].cpu().numpy(), c)
        assert np.array_equal(got["scales_r"][r0:r1, c0 // 32:c0 // 32 + 8].cpu().numpy(), s)
        cc, cs = orc.quantize_colwise(blk, [r1 - r0])
        assert np.array_equal(got["codes_c"][r0:r1, c0:c0 + 256].cpu().numpy(), cc)
        assert np.array_equal(got["scales_c"][int(base[g]) + j, c0:c0 + 256].cpu().numpy(), cs[0])
