"""MXFP8 grouped GEMMs on the GPU (through the C ABI) against the fp64 oracle.

Both sides quantize the same bf16 inputs: the GPU with group_quantize_mxfp8
(checked bit-exact against the oracle quantizer in test_gpu_quantize.py), the
oracle with its own quantizer; the oracle then multiplies the dequantized
operands in fp64.  Bar: relative Frobenius error <= 1e-2 per group; bit-exact
in an integer-valued mode; caller-buffer tails untouched; accumulate and
overwrite of main_grad as for bf16 (``grouped_linear.py`` fuser_forward /
fuser_backward with MXFP8 quantizers).
"""
import numpy as np
import pytest
import torch

from grouped_gemm_splits_b200 import gl, synth
from oracle import gl_oracle as orc
from tests.gpu_util import f64, offsets_on_device, sample_rows, sentinel_like, untouched

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[True, False], ids=["pair", "single"])
def pair(request):
    """256-row tiles on CTA pairs, or 128-row tiles on single CTAs (a per-call
    option of every GEMM)."""
    return request.param

TOL_MX = 1e-2


def _quantize_all(d, m, G, N, K, off, st):
    """GPU MXFP8 copies of x, W and dy in the forms the GEMMs read."""
    q = {}
    q["x"] = gl.group_quantize_mxfp8(d["x"], off, rowwise=True, colwise=True, status=st, mma_scales=True)
    q["dy"] = gl.group_quantize_mxfp8(d["dy"], off, rowwise=True, colwise=True, status=st, mma_scales=True)
    q["w"] = gl.group_quantize_mxfp8(d["w"], rowwise=True, colwise=True, mma_scales=True)  # G equal groups
    return q


def _oracle_all(d, m, G, N, K):
    x, w, dy = f64(d["x"]), f64(d["w"]), f64(d["dy"])
    xq, xs = orc.quantize_rowwise(x)
    xcq, xcs = orc.quantize_colwise(x, m)
    dyq, dys = orc.quantize_rowwise(dy)
    dycq, dycs = orc.quantize_colwise(dy, m)
    wq, ws = orc.quantize_rowwise(w.reshape(G * N, K))
    wcq, wcs = orc.quantize_colwise(w.reshape(G * N, K), [N] * G)
    return {
        "fwd": orc.fwd_mxfp8(xq, xs, wq.reshape(G, N, K), ws.reshape(G, N, K // 32),
                             f64(d["bias"]) if "bias" in d else None, m),
        "dgrad": orc.dgrad_mxfp8(dyq, dys, wcq.reshape(G, N, K), wcs, m),
        "wgrad_over": orc.wgrad_mxfp8(xcq, xcs, dycq, dycs, m, None, False),
    }


SMALL = [
    (4, 256, 128, [0, 96, 160, 256]),
    (5, 384, 512, [130, 0, 301, 7, 262]),
    (1, 256, 256, [300]),
    (8, 128, 256, [1, 15, 17, 63, 64, 65, 0, 130]),
    (3, 512, 384, [257, 0, 511]),
    (2, 896, 128, [200, 70]),  # five B tiles, starting 0 or 64 rows into a scale atom
]


@pytest.mark.parametrize("G,N,K,m", SMALL)
@pytest.mark.parametrize("per_group", [False, True])
def test_mxfp8_small(G, N, K, m, per_group, pair):
    M = int(sum(m))
    d = {k: v.cuda() for k, v in synth.operands(G, M, N, K, seed=G + N + K, bias=True).items()}
    off, st = offsets_on_device(m, M, M + 32)
    q = _quantize_all(d, m, G, N, K, off, st)
    if per_group:
        # each weight quantized as its own [N, K] tensor: separate buffers per group
        qg = [gl.group_quantize_mxfp8(d["w"][g].contiguous(), rowwise=True, colwise=True, mma_scales=True)
              for g in range(G)]
        wc = [t["codes_r"] for t in qg]
        ws = [t["scales_r"] for t in qg]
        wcc = [t["codes_c"] for t in qg]
        wcs = [t["scales_c"] for t in qg]
        bias = [d["bias"][g].clone() for g in range(G)]
    else:
        wc = q["w"]["codes_r"].view(G, N, K)
        ws = q["w"]["scales_r"]
        wcc = q["w"]["codes_c"].view(G, N, K)
        wcs = q["w"]["scales_c"]
        bias = d["bias"]
    y = sentinel_like(M + 32, N)
    gl.gl_fwd_mxfp8(q["x"]["codes_r"], q["x"]["scales_r"], wc, ws, bias, off, st, y, pair=pair)
    dx = sentinel_like(M + 32, K)
    gl.gl_dgrad_mxfp8(q["dy"]["codes_r"], q["dy"]["scales_r"], wcc, wcs, off, st, dx, pair=pair)
    mg = torch.full((G, N, K), float("nan"), device="cuda")
    mg_arg = [mg[g] for g in range(G)] if per_group else mg
    gl.gl_wgrad_mxfp8(q["x"]["codes_c"], q["x"]["scales_c"], q["dy"]["codes_c"], q["dy"]["scales_c"], off, st,
                      mg_arg, accumulate=False, pair=pair)
    mga = d["main_grad"].clone()
    gl.gl_wgrad_mxfp8(q["x"]["codes_c"], q["x"]["scales_c"], q["dy"]["codes_c"], q["dy"]["scales_c"], off, st,
                      mga, accumulate=True, pair=pair)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = _oracle_all(d, m, G, N, K)
    o = orc.offsets(m)
    got_y, got_dx, got_w, got_a = f64(y), f64(dx), f64(mg), f64(mga)
    mg0 = f64(d["main_grad"])
    for g in range(G):
        a, b = int(o[g]), int(o[g + 1])
        if a == b:
            assert np.all(got_w[g] == 0.0)
            assert np.array_equal(got_a[g], mg0[g])
            continue
        assert orc.rel_frobenius(got_y[a:b], ref["fwd"][a:b]) <= TOL_MX, ("fwd", g)
        assert orc.rel_frobenius(got_dx[a:b], ref["dgrad"][a:b]) <= TOL_MX, ("dgrad", g)
        assert orc.rel_frobenius(got_w[g], ref["wgrad_over"][g]) <= TOL_MX, ("wgrad", g)
        assert orc.rel_frobenius(got_a[g] - mg0[g], ref["wgrad_over"][g]) <= TOL_MX, ("wgrad acc", g)
    assert untouched(y[M:]) and untouched(dx[M:])


def test_mxfp8_many_groups_per_group(pair):
    """70 groups with per-group weights and main_grad: the launches cover 64
    groups each, so the second one starts at a group whose scale k-groups
    follow those of all earlier groups."""
    G, N, K = 70, 128, 128
    rng = np.random.default_rng(70)
    m = [int(v) for v in rng.integers(0, 90, size=G)]
    m[3] = m[64] = 0
    M = sum(m)
    d = {k: v.cuda() for k, v in synth.operands(G, M, N, K, seed=70, bias=True).items()}
    off, st = offsets_on_device(m, M)
    q = _quantize_all(d, m, G, N, K, off, st)
    qg = [gl.group_quantize_mxfp8(d["w"][g].contiguous(), rowwise=True, colwise=True, mma_scales=True)
          for g in range(G)]
    y = gl.gl_fwd_mxfp8(q["x"]["codes_r"], q["x"]["scales_r"], [t["codes_r"] for t in qg],
                        [t["scales_r"] for t in qg], [d["bias"][g].clone() for g in range(G)], off, st, pair=pair)
    dx = gl.gl_dgrad_mxfp8(q["dy"]["codes_r"], q["dy"]["scales_r"], [t["codes_c"] for t in qg],
                           [t["scales_c"] for t in qg], off, st, pair=pair)
    mg = torch.full((G, N, K), float("nan"), device="cuda")
    gl.gl_wgrad_mxfp8(q["x"]["codes_c"], q["x"]["scales_c"], q["dy"]["codes_c"], q["dy"]["scales_c"], off, st,
                      [mg[g] for g in range(G)], accumulate=False, pair=pair)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = _oracle_all(d, m, G, N, K)
    o = orc.offsets(m)
    got_y, got_dx, got_w = f64(y), f64(dx), f64(mg)
    for g in range(G):
        a, b = int(o[g]), int(o[g + 1])
        if a == b:
            assert np.all(got_w[g] == 0.0)
            continue
        assert orc.rel_frobenius(got_y[a:b], ref["fwd"][a:b]) <= TOL_MX, ("fwd", g)
        assert orc.rel_frobenius(got_dx[a:b], ref["dgrad"][a:b]) <= TOL_MX, ("dgrad", g)
        assert orc.rel_frobenius(got_w[g], ref["wgrad_over"][g]) <= TOL_MX, ("wgrad", g)


def test_mxfp8_integer_mode_bit_exact(pair):
    """Values in {-1,0,1}: every block scales by 2^-8 (or is all zero), the
    codes are exact, and every product sum is an exact small integer."""
    G, N, K, m = 3, 256, 128, [0, 100, 156]
    M = sum(m)
    d = {k: v.cuda() for k, v in synth.integer_operands(G, M, N, K, seed=3).items()}
    off, st = offsets_on_device(m, M)
    q = _quantize_all(d, m, G, N, K, off, st)
    y = gl.gl_fwd_mxfp8(q["x"]["codes_r"], q["x"]["scales_r"], q["w"]["codes_r"].view(G, N, K),
                        q["w"]["scales_r"], d["bias"], off, st, pair=pair)
    dx = gl.gl_dgrad_mxfp8(q["dy"]["codes_r"], q["dy"]["scales_r"], q["w"]["codes_c"].view(G, N, K),
                           q["w"]["scales_c"], off, st, pair=pair)
    mg = d["main_grad"].clone()
    gl.gl_wgrad_mxfp8(q["x"]["codes_c"], q["x"]["scales_c"], q["dy"]["codes_c"], q["dy"]["scales_c"], off, st,
                      mg, accumulate=True, pair=pair)
    torch.cuda.synchronize()
    x64, w64, dy64 = f64(d["x"]), f64(d["w"]), f64(d["dy"])
    assert np.array_equal(synth.bf16_bits(y), orc.f64_to_bf16_rne(orc.fwd(x64, w64, f64(d["bias"]), m)))
    assert np.array_equal(f64(dx), orc.dgrad(dy64, w64, m))
    assert np.array_equal(f64(mg), orc.wgrad(x64, dy64, m, f64(d["main_grad"]), True))


@pytest.mark.parametrize("pair_", [False, True], ids=["single", "pair"])
def test_mxfp8_wait_timeout_sets_status_and_recovers(pair_):
    """GL_OPT_HOLD_LOADS with 2 ms pipeline waits on the MXFP8 GEMMs: the
    status word gets GL_DEV_TIMEOUT and nothing is written; the same calls
    with the default options then match the oracle."""
    G, N, K, m = 3, 256, 512, [300, 0, 212]
    M = sum(m)
    d = {k: v.cuda() for k, v in synth.operands(G, M, N, K, seed=43, bias=True).items()}
    off, st = offsets_on_device(m, M)
    q = _quantize_all(d, m, G, N, K, off, st)
    torch.cuda.synchronize()
    args_f = (q["x"]["codes_r"], q["x"]["scales_r"], q["w"]["codes_r"].view(G, N, K), q["w"]["scales_r"],
              d["bias"], off, st)
    args_w = (q["x"]["codes_c"], q["x"]["scales_c"], q["dy"]["codes_c"], q["dy"]["scales_c"], off, st)
    y = sentinel_like(M, N)
    mg = d["main_grad"].clone()
    hold = dict(pair=pair_, wait_limit_us=2000, opt_flags=gl.GL_OPT_HOLD_LOADS)
    gl.gl_fwd_mxfp8(*args_f, y, **hold)
    gl.gl_wgrad_mxfp8(*args_w, mg, accumulate=True, **hold)
    torch.cuda.synchronize()
    assert int(st.item()) == gl.GL_DEV_TIMEOUT
    assert untouched(y)
    assert torch.equal(mg, d["main_grad"])
    st.zero_()
    gl.gl_fwd_mxfp8(*args_f, y, pair=pair_)
    gl.gl_wgrad_mxfp8(*args_w, mg, accumulate=True, pair=pair_)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = _oracle_all(d, m, G, N, K)
    o = orc.offsets(m)
    got_y, got_w, mg0 = f64(y), f64(mg), f64(d["main_grad"])
    for g in range(G):
        a, b = int(o[g]), int(o[g + 1])
        if a == b:
            continue
        assert orc.rel_frobenius(got_y[a:b], ref["fwd"][a:b]) <= TOL_MX, ("fwd", g)
        assert orc.rel_frobenius(got_w[g] - mg0[g], ref["wgrad_over"][g]) <= TOL_MX, ("wgrad", g)


def test_mxfp8_max_groups_stacked(pair):
    """GL_MAX_GROUPS_MXFP8 (2048) groups in one stacked call, most of them
    empty or short: the scale k-groups of the columnwise operands restart at
    every group; each non-empty group checked on its own."""
    rng = np.random.default_rng(2048)
    G, N, K = 2048, 128, 128
    m = [int(v) for v in synth.random_splits(rng, G, 12000, p_empty=0.5)]
    M = sum(m)
    d = {k: v.cuda() for k, v in synth.operands(G, M, N, K, seed=2048, bias=True).items()}
    off, st = offsets_on_device(m, M)
    q = _quantize_all(d, m, G, N, K, off, st)
    y = gl.gl_fwd_mxfp8(q["x"]["codes_r"], q["x"]["scales_r"], q["w"]["codes_r"].view(G, N, K), q["w"]["scales_r"],
                        d["bias"], off, st, pair=pair)
    dx = gl.gl_dgrad_mxfp8(q["dy"]["codes_r"], q["dy"]["scales_r"], q["w"]["codes_c"].view(G, N, K),
                           q["w"]["scales_c"], off, st, pair=pair)
    mg = torch.full((G, N, K), float("nan"), device="cuda")
    gl.gl_wgrad_mxfp8(q["x"]["codes_c"], q["x"]["scales_c"], q["dy"]["codes_c"], q["dy"]["scales_c"], off, st, mg,
                      accumulate=False, pair=pair)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = _oracle_all(d, m, G, N, K)
    o = orc.offsets(m)
    got_y, got_dx, got_w = f64(y), f64(dx), f64(mg)
    for g in range(G):
        a, b = int(o[g]), int(o[g + 1])
        if a == b:
            assert np.all(got_w[g] == 0.0), g
            continue
        assert orc.rel_frobenius(got_y[a:b], ref["fwd"][a:b]) <= TOL_MX, ("fwd", g)
        assert orc.rel_frobenius(got_dx[a:b], ref["dgrad"][a:b]) <= TOL_MX, ("dgrad", g)
        assert orc.rel_frobenius(got_w[g], ref["wgrad_over"][g]) <= TOL_MX, ("wgrad", g)


FULL_MX = ["mxfp8_g8", "stacked_g128_uniform", "stacked_g128_ragged"]
ROWS_PER_GROUP = 8   # random rows per group, besides the group's first and last row
COLS = 64            # output columns sampled per group
WG = 8               # wgrad: WG x WG sampled (n, k) entries per group


def _idx(v):
    return torch.as_tensor(np.asarray(v, dtype=np.int64), device="cuda")


@pytest.mark.parametrize("name", FULL_MX)
def test_mxfp8_full_size_sampled(name, pair):
    """A full-size workload through the MXFP8 path: the GPU casts x, W and dy,
    the three block-scaled GEMMs run, and every non-empty group is checked on
    its own against the oracle, which quantizes exactly the rows / columns each
    sampled entry needs with its own quantizer: its first, last and
    ROWS_PER_GROUP random rows x COLS columns of y and dx, and WG x WG entries
    of main_grad, each within 1e-2 relative Frobenius error.  The ragged
    stacked workload keeps its unaligned split sizes, so columnwise blocks
    restart inside 32-row blocks and groups end in partial blocks."""
    wl = synth.WORKLOADS[name]
    m = synth.m_splits_for(name)
    G, N, K, M = wl.G, wl.N, wl.K, wl.rows
    d = synth.operands(G, M, N, K, wl.seed, device="cuda", bias=False)
    off, st = offsets_on_device(m, M)
    q = _quantize_all(d, m, G, N, K, off, st)
    y = gl.gl_fwd_mxfp8(q["x"]["codes_r"], q["x"]["scales_r"], q["w"]["codes_r"].view(G, N, K),
                        q["w"]["scales_r"], None, off, st, pair=pair)
    dx = gl.gl_dgrad_mxfp8(q["dy"]["codes_r"], q["dy"]["scales_r"], q["w"]["codes_c"].view(G, N, K),
                           q["w"]["scales_c"], off, st, pair=pair)
    mg = d["main_grad"].clone()
    gl.gl_wgrad_mxfp8(q["x"]["codes_c"], q["x"]["scales_c"], q["dy"]["codes_c"], q["dy"]["scales_c"], off, st,
                      mg, accumulate=True, pair=pair)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    del q
    rng = np.random.default_rng(wl.seed + 7)
    o = orc.offsets(m)
    deq_r = lambda a: orc.dequant_rowwise(*orc.quantize_rowwise(a))
    checked = 0
    for g in range(G):
        a, b = int(o[g]), int(o[g + 1])
        if a == b:
            assert torch.equal(mg[g], d["main_grad"][g]), ("accumulate touched an empty group", g)
            continue
        rows = np.unique(np.concatenate([[a, b - 1], rng.integers(a, b, size=ROWS_PER_GROUP)]))
        ns = rng.choice(N, size=COLS, replace=False)
        ks = rng.choice(K, size=COLS, replace=False)
        xr = deq_r(f64(d["x"][_idx(rows)]))           # x rows, blocks along K
        dyr = deq_r(f64(d["dy"][_idx(rows)]))         # dy rows, blocks along N
        wr = deq_r(f64(d["w"][g][_idx(ns)]))          # W_g rows n, blocks along K
        wcol = f64(d["w"][g][:, _idx(ks)])            # W_g columns k, blocks of 32 along N
        wc = orc.dequant_colwise(*orc.quantize_colwise(wcol, [N]), [N]).T
        ref_f = np.array([[orc.fwd_entry(xr[i], wr[j], None) for j in range(COLS)] for i in range(len(rows))])
        got_f = f64(y[_idx(rows)][:, _idx(ns)])
        assert orc.rel_frobenius(got_f, ref_f) <= TOL_MX, ("fwd", g)
        ref_d = np.array([[orc.dgrad_entry(dyr[i], wc[j]) for j in range(COLS)] for i in range(len(rows))])
        got_d = f64(dx[_idx(rows)][:, _idx(ks)])
        assert orc.rel_frobenius(got_d, ref_d) <= TOL_MX, ("dgrad", g)
        nw = rng.choice(N, size=WG, replace=False)
        kw = rng.choice(K, size=WG, replace=False)
        mg_g = [b - a]
        dyc = orc.dequant_colwise(*orc.quantize_colwise(f64(d["dy"][a:b][:, _idx(nw)]), mg_g), mg_g)
        xc = orc.dequant_colwise(*orc.quantize_colwise(f64(d["x"][a:b][:, _idx(kw)]), mg_g), mg_g)
        old = f64(d["main_grad"][g][_idx(nw)][:, _idx(kw)])
        new = f64(mg[g][_idx(nw)][:, _idx(kw)])
        ref_w = np.array([[orc.wgrad_entry(dyc[:, i], xc[:, j], old[i, j], True) for j in range(WG)]
                          for i in range(WG)])
        assert orc.rel_frobenius(new - old, ref_w - old) <= TOL_MX, ("wgrad", g)
        checked += 1
    assert checked == int((m > 0).sum())
    torch.cuda.empty_cache()
