"""Seeded random configurations of the whole path on the GPU against the oracle.

Each case draws the group count, the layer sizes (bf16: multiples of 8;
MXFP8: multiples of 128), split sizes with empty and very short groups,
stacked or per-group weights, bias or none, CTA pairs or single CTAs, and
accumulate or overwrite; every output is checked per group: bf16 products
and wgrad within 5e-3, MXFP8 products within 1e-2 (relative Frobenius, the
fp64 oracle of ``grouped_linear.py``'s split -> per-split linear -> concat),
and the MXFP8 codes and scales of x (rowwise) and dy (columnwise) bit for
bit.
"""
import numpy as np
import pytest
import torch

from grouped_gemm_splits_b200 import gl, synth
from oracle import gl_oracle as orc
from tests.gpu_util import TOL_BF16, assert_groups_close, f64, offsets_on_device, sentinel_like, untouched

pytestmark = pytest.mark.gpu

TOL_MX = 1e-2
CASES = 10


def _splits(rng, G, cap):
    """Split sizes: about a fifth empty, some of 1..40 rows, the rest up to cap."""
    m = []
    for _ in range(G):
        u = rng.random()
        m.append(0 if u < 0.2 else int(rng.integers(1, 41)) if u < 0.45 else int(rng.integers(1, cap + 1)))
    return m


def _draw(seed, mx):
    rng = np.random.default_rng((2000 if mx else 1000) + seed)
    G = int(rng.integers(1, 10))
    unit = 128 if mx else 8
    N = unit * int(rng.integers(1, (640 if mx else 520) // unit + 1))
    K = unit * int(rng.integers(1, (640 if mx else 520) // unit + 1))
    m = _splits(rng, G, 400)
    if sum(m) == 0:
        m[0] = 1
    return rng, G, N, K, m


@pytest.mark.parametrize("seed", range(CASES))
def test_bf16_random_configurations(seed):
    rng, G, N, K, m = _draw(seed, mx=False)
    M = sum(m)
    pair = bool(rng.integers(0, 2))
    per_group = bool(rng.integers(0, 2))
    use_bias = bool(rng.integers(0, 2))
    accumulate = bool(rng.integers(0, 2))
    d = {k: v.cuda() for k, v in synth.operands(G, M, N, K, seed=seed, bias=True).items()}
    off, st = offsets_on_device(m, M, M + 8)
    w = [d["w"][g].clone() for g in range(G)] if per_group else d["w"]
    b = None
    if use_bias:
        b = [d["bias"][g].clone() for g in range(G)] if per_group else d["bias"]
    y = sentinel_like(M + 8, N)
    gl.gl_fwd(d["x"], w, b, off, st, y, pair=pair)
    dx = sentinel_like(M + 8, K)
    gl.gl_dgrad(d["dy"], w, off, st, dx, pair=pair)
    mg = d["main_grad"].clone() if accumulate else torch.full_like(d["main_grad"], float("nan"))
    mg_arg = [mg[g] for g in range(G)] if per_group else mg
    gl.gl_wgrad(d["x"], d["dy"], off, st, mg_arg, accumulate=accumulate, pair=pair)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, (G, N, K, m)

    x64, w64, dy64 = f64(d["x"]), f64(d["w"]), f64(d["dy"])
    b64 = f64(d["bias"]) if use_bias else None
    assert_groups_close(f64(y[:M]), orc.fwd(x64, w64, b64, m), m, what=("fwd", G, N, K, m))
    assert_groups_close(f64(dx[:M]), orc.dgrad(dy64, w64, m), m, what=("dgrad", G, N, K, m))
    assert untouched(y[M:]) and untouched(dx[M:])
    mg0 = f64(d["main_grad"])
    ref = orc.wgrad(x64, dy64, m, mg0 if accumulate else None, accumulate)
    got = f64(mg)
    for g in range(G):
        if m[g] == 0:
            if accumulate:
                assert np.array_equal(got[g], mg0[g])
            else:
                assert np.all(got[g] == 0.0)
        elif accumulate:
            assert orc.rel_frobenius(got[g] - mg0[g], ref[g] - mg0[g]) <= TOL_BF16, ("wgrad", g, G, N, K, m)
        else:
            assert orc.rel_frobenius(got[g], ref[g]) <= TOL_BF16, ("wgrad", g, G, N, K, m)


@pytest.mark.parametrize("seed", range(CASES))
def test_mxfp8_random_configurations(seed):
    rng, G, N, K, m = _draw(seed, mx=True)
    M = sum(m)
    pair = bool(rng.integers(0, 2))
    use_bias = bool(rng.integers(0, 2))
    accumulate = bool(rng.integers(0, 2))
    d = {k: v.cuda() for k, v in synth.operands(G, M, N, K, seed=100 + seed, bias=True).items()}
    off, st = offsets_on_device(m, M, M + 8)
    qx = gl.group_quantize_mxfp8(d["x"], off, rowwise=True, colwise=True, status=st, mma_scales=True)
    qdy = gl.group_quantize_mxfp8(d["dy"], off, rowwise=True, colwise=True, status=st, mma_scales=True)
    qw = gl.group_quantize_mxfp8(d["w"], rowwise=True, colwise=True, mma_scales=True)
    y = sentinel_like(M + 8, N)
    gl.gl_fwd_mxfp8(qx["codes_r"], qx["scales_r"], qw["codes_r"].view(G, N, K), qw["scales_r"],
                    d["bias"] if use_bias else None, off, st, y, pair=pair)
    dx = sentinel_like(M + 8, K)
    gl.gl_dgrad_mxfp8(qdy["codes_r"], qdy["scales_r"], qw["codes_c"].view(G, N, K), qw["scales_c"], off, st, dx,
                      pair=pair)
    mg = d["main_grad"].clone() if accumulate else torch.full_like(d["main_grad"], float("nan"))
    gl.gl_wgrad_mxfp8(qx["codes_c"], qx["scales_c"], qdy["codes_c"], qdy["scales_c"], off, st, mg,
                      accumulate=accumulate, pair=pair)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, (G, N, K, m)

    x, w, dy = f64(d["x"]), f64(d["w"]), f64(d["dy"])
    xq, xs = orc.quantize_rowwise(x)
    xcq, xcs = orc.quantize_colwise(x, m)
    dyq, dys = orc.quantize_rowwise(dy)
    dycq, dycs = orc.quantize_colwise(dy, m)
    wq, ws = orc.quantize_rowwise(w.reshape(G * N, K))
    wcq, wcs = orc.quantize_colwise(w.reshape(G * N, K), [N] * G)
    # the GPU's codes and scales bit for bit against the oracle's: x rowwise
    # (scales in the MMA layout), dy columnwise
    assert np.array_equal(qx["codes_r"].cpu().numpy().reshape(M, K), xq)
    assert np.array_equal(qx["scales_r"].cpu().numpy()[orc.mma_offsets_rowwise(M, K)], xs)
    assert np.array_equal(qdy["codes_c"].cpu().numpy().reshape(M, N), dycq)
    assert np.array_equal(qdy["scales_c"].cpu().numpy()[orc.mma_offsets_colwise(m, N)], dycs)
    ref_y = orc.fwd_mxfp8(xq, xs, wq.reshape(G, N, K), ws.reshape(G, N, K // 32),
                          f64(d["bias"]) if use_bias else None, m)
    ref_dx = orc.dgrad_mxfp8(dyq, dys, wcq.reshape(G, N, K), wcs, m)
    ref_w = orc.wgrad_mxfp8(xcq, xcs, dycq, dycs, m, None, False)
    o = orc.offsets(m)
    got_y, got_dx, got_w = f64(y), f64(dx), f64(mg)
    mg0 = f64(d["main_grad"])
    for g in range(G):
        a, b = int(o[g]), int(o[g + 1])
        if a == b:
            if accumulate:
                assert np.array_equal(got_w[g], mg0[g])
            else:
                assert np.all(got_w[g] == 0.0)
            continue
        assert orc.rel_frobenius(got_y[a:b], ref_y[a:b]) <= TOL_MX, ("fwd", g, G, N, K, m)
        assert orc.rel_frobenius(got_dx[a:b], ref_dx[a:b]) <= TOL_MX, ("dgrad", g, G, N, K, m)
        got_g = got_w[g] - mg0[g] if accumulate else got_w[g]
        assert orc.rel_frobenius(got_g, ref_w[g]) <= TOL_MX, ("wgrad", g, G, N, K, m)
    assert untouched(y[M:]) and untouched(dx[M:])
