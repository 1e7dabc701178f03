"""bf16 grouped GEMMs on the GPU (through the C ABI) against the fp64 oracle.

Bar: relative Frobenius error <= 5e-3 per group for fwd / dgrad / wgrad;
bit-exact results in the integer-valued mode; rows outside the groups and the
padded tail of a caller buffer untouched ("Add optional caller-provided
output/grad-input buffers", TransformerEngine PR #3161); accumulate vs
overwrite of main_grad and empty groups as in ``grouped_linear.py``
fuser_backward.
"""
import numpy as np
import pytest
import torch

from grouped_gemm_splits_b200 import gl, synth
from oracle import gl_oracle as orc
from tests.gpu_util import (TOL_BF16, assert_groups_close, f64, offsets_on_device, sample_rows,
                            sentinel_like, untouched)

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[True, False], ids=["pair", "single"])
def pair(request):
    """256x256 tiles on CTA pairs, or 128x256 tiles on single CTAs (a per-call
    option of every GEMM)."""
    return request.param

# (G, N, K, m_splits): several tiles, ragged tails in every dimension,
# empty groups, groups shorter than one MMA step.
SMALL = [
    (4, 256, 128, [0, 96, 160, 256]),                        # the tiny workload
    (5, 392, 320, [130, 0, 301, 7, 262]),                    # N, K not multiples of the tile
    (1, 512, 512, [300]),                                    # G = 1: a plain linear layer
    (8, 136, 200, [1, 15, 17, 63, 64, 65, 0, 130]),          # tiny groups, ragged wgrad tails
    (3, 264, 1032, [257, 0, 511]),                           # longer contraction, K tail of 8
]


def _inputs(G, N, K, m, seed, bias=True, device="cuda"):
    M = int(sum(m))
    d = synth.operands(G, M, N, K, seed, device="cpu", bias=bias)
    return {k: v.to(device) for k, v in d.items()}


@pytest.mark.parametrize("G,N,K,m", SMALL)
@pytest.mark.parametrize("per_group", [False, True])
def test_fwd_dgrad_wgrad_small(G, N, K, m, per_group, pair):
    M = int(sum(m))
    d = _inputs(G, N, K, m, seed=G * 7 + N)
    off, st = offsets_on_device(m, M, M + 64)
    w = [d["w"][i].clone() for i in range(G)] if per_group else d["w"]
    b = [d["bias"][i].clone() for i in range(G)] if per_group else d["bias"]
    x64, w64, b64, dy64 = f64(d["x"]), f64(d["w"]), f64(d["bias"]), f64(d["dy"])

    y = sentinel_like(M + 64, N)
    gl.gl_fwd(d["x"], w, b, off, st, y, pair=pair)
    dx = sentinel_like(M + 64, K)
    gl.gl_dgrad(d["dy"], w, off, st, dx, pair=pair)
    mg_acc = d["main_grad"].clone()
    mg_acc_arg = [mg_acc[i] for i in range(G)] if per_group else mg_acc
    gl.gl_wgrad(d["x"], d["dy"], off, st, mg_acc_arg, accumulate=True, pair=pair)
    mg_over = torch.full_like(d["main_grad"], float("nan"))
    gl.gl_wgrad(d["x"], d["dy"], off, st, mg_over, accumulate=False, pair=pair)
    torch.cuda.synchronize()
    assert int(st.item()) == 0

    assert_groups_close(f64(y[:M]), orc.fwd(x64, w64, b64, m), m, what="fwd")
    assert untouched(y[M:]), "padded tail of the output buffer was written"
    assert_groups_close(f64(dx[:M]), orc.dgrad(dy64, w64, m), m, what="dgrad")
    assert untouched(dx[M:])
    mg0 = f64(d["main_grad"])
    ref_acc = orc.wgrad(x64, dy64, m, mg0, True)
    ref_over = orc.wgrad(x64, dy64, m, None, False)
    got_acc, got_over = f64(mg_acc), f64(mg_over)
    for g in range(G):
        if m[g] == 0:
            assert np.array_equal(got_acc[g], mg0[g]), "accumulate must leave an empty group alone"
            assert np.all(got_over[g] == 0.0), "overwrite of an empty group must give zeros"
        else:
            assert orc.rel_frobenius(got_acc[g] - mg0[g], ref_acc[g] - mg0[g]) <= TOL_BF16, g
            assert orc.rel_frobenius(got_over[g], ref_over[g]) <= TOL_BF16, g


def test_integer_mode_bit_exact(pair):
    """{-1,0,1} operands and integer biases: every sum is exact, so the GPU
    must reproduce the oracle bit for bit (tiny workload shapes)."""
    G, N, K, m = 4, 256, 128, [0, 96, 160, 256]
    M = sum(m)
    d = {k: v.cuda() for k, v in synth.integer_operands(G, M, N, K, seed=11).items()}
    off, st = offsets_on_device(m, M)
    y = gl.gl_fwd(d["x"], d["w"], d["bias"], off, st, pair=pair)
    dx = gl.gl_dgrad(d["dy"], d["w"], off, st, pair=pair)
    mg = d["main_grad"].clone()
    gl.gl_wgrad(d["x"], d["dy"], off, st, mg, accumulate=True, pair=pair)
    torch.cuda.synchronize()
    x64, w64, b64, dy64 = f64(d["x"]), f64(d["w"]), f64(d["bias"]), f64(d["dy"])
    ref_y = orc.fwd(x64, w64, b64, m)
    assert np.array_equal(synth.bf16_bits(y), orc.f64_to_bf16_rne(ref_y))
    assert np.array_equal(f64(dx), orc.dgrad(dy64, w64, m))
    assert np.array_equal(f64(mg), orc.wgrad(x64, dy64, m, f64(d["main_grad"]), True))


def test_stacked_and_per_group_weights_identical():
    G, N, K, m = 5, 392, 320, [130, 0, 301, 7, 262]
    M = sum(m)
    d = _inputs(G, N, K, m, seed=3)
    off, st = offsets_on_device(m, M)
    ys = gl.gl_fwd(d["x"], d["w"], d["bias"], off, st)
    yp = gl.gl_fwd(d["x"], [d["w"][i].clone() for i in range(G)], [d["bias"][i].clone() for i in range(G)], off, st)
    dxs = gl.gl_dgrad(d["dy"], d["w"], off, st)
    dxp = gl.gl_dgrad(d["dy"], [d["w"][i].clone() for i in range(G)], off, st)
    torch.cuda.synchronize()
    assert torch.equal(ys.view(torch.int16), yp.view(torch.int16))
    assert torch.equal(dxs.view(torch.int16), dxp.view(torch.int16))


def test_caller_buffer_matches_internal_allocation():
    G, N, K, m = 4, 256, 128, [0, 96, 160, 256]
    M = sum(m)
    d = _inputs(G, N, K, m, seed=5)
    off, st = offsets_on_device(m, M, M + 1024)
    y_int = gl.gl_fwd(d["x"], d["w"], d["bias"], off, st)
    y_buf = sentinel_like(M + 1024, N)
    gl.gl_fwd(d["x"], d["w"], d["bias"], off, st, y_buf)
    torch.cuda.synchronize()
    assert torch.equal(y_buf[:M].view(torch.int16), y_int.view(torch.int16))
    assert untouched(y_buf[M:])


def test_many_groups_per_group_chunking(pair):
    """More groups than one launch carries in per-group mode (64)."""
    rng = np.random.default_rng(9)
    G, N, K = 150, 136, 64
    m = synth.random_splits(rng, G, 3000)
    M = int(m.sum())
    d = _inputs(G, N, K, m, seed=9)
    off, st = offsets_on_device(m, M)
    wl = [d["w"][i].clone() for i in range(G)]
    y = gl.gl_fwd(d["x"], wl, [d["bias"][i] for i in range(G)], off, st, pair=pair)
    mg = [d["main_grad"][i].clone() for i in range(G)]
    gl.gl_wgrad(d["x"], d["dy"], off, st, mg, accumulate=True, pair=pair)
    torch.cuda.synchronize()
    x64, w64, dy64 = f64(d["x"]), f64(d["w"]), f64(d["dy"])
    assert_groups_close(f64(y), orc.fwd(x64, w64, f64(d["bias"]), m), m)
    ref = orc.wgrad(x64, dy64, m, f64(d["main_grad"]), True)
    got = np.stack([f64(t) for t in mg])
    mg0 = f64(d["main_grad"])
    for g in range(G):
        if m[g]:
            assert orc.rel_frobenius(got[g] - mg0[g], ref[g] - mg0[g]) <= TOL_BF16


def test_all_groups_empty(pair):
    G, N, K, m = 3, 256, 128, [0, 0, 0]
    d = synth.operands(G, 8, N, K, 1)
    x = d["x"].cuda()[:0]      # zero rows, but a valid base pointer
    dy = d["dy"].cuda()[:0]
    off, st = offsets_on_device(m, 0, 16)
    y = sentinel_like(16, N)
    gl.gl_fwd(x, d["w"].cuda(), None, off, st, y, pair=pair)
    mg = d["main_grad"].cuda()
    mg0 = mg.clone()
    gl.gl_wgrad(x, dy, off, st, mg, accumulate=True, pair=pair)
    mgo = torch.full_like(mg, 3.0)
    gl.gl_wgrad(x, dy, off, st, mgo, accumulate=False, pair=pair)
    torch.cuda.synchronize()
    assert untouched(y)
    assert torch.equal(mg, mg0)
    assert bool((mgo == 0).all())


def test_bad_splits_write_nothing():
    """A split sum that does not match the input, or a negative split, is
    reported in the status word and every later kernel writes nothing."""
    G, N, K = 3, 256, 128
    d = _inputs(G, N, K, [10, 20, 30], seed=2)
    for m in ([10, 20, 31], [10, -5, 55]):
        off, st = offsets_on_device(m, 60, 60)
        y = sentinel_like(60, N)
        gl.gl_fwd(d["x"], d["w"], d["bias"], off, st, y)
        mg = d["main_grad"].clone()
        gl.gl_wgrad(d["x"], d["dy"], off, st, mg, accumulate=False)
        torch.cuda.synchronize()
        assert int(st.item()) == orc.split_status(m, 60, 60) != 0
        assert untouched(y)
        assert torch.equal(mg, d["main_grad"])


def test_max_groups_stacked(pair):
    """GL_MAX_GROUPS (4096) groups in one stacked call, most of them empty or
    a few rows long: every tile prefix, empty-group skip and ragged tail at
    once; each non-empty group checked on its own."""
    rng = np.random.default_rng(4096)
    G, N, K = 4096, 128, 64
    m = synth.random_splits(rng, G, 12000, p_empty=0.5)
    M = int(m.sum())
    d = _inputs(G, N, K, m, seed=4096)
    off, st = offsets_on_device(m, M)
    y = gl.gl_fwd(d["x"], d["w"], d["bias"], off, st, pair=pair)
    dx = gl.gl_dgrad(d["dy"], d["w"], off, st, pair=pair)
    mg = d["main_grad"].clone()
    gl.gl_wgrad(d["x"], d["dy"], off, st, mg, accumulate=True, pair=pair)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    x64, w64, b64, dy64 = f64(d["x"]), f64(d["w"]), f64(d["bias"]), f64(d["dy"])
    assert_groups_close(f64(y), orc.fwd(x64, w64, b64, m), m, what="fwd")
    assert_groups_close(f64(dx), orc.dgrad(dy64, w64, m), m, what="dgrad")
    mg0 = f64(d["main_grad"])
    ref = orc.wgrad(x64, dy64, m, mg0, True)
    got = f64(mg)
    for g in range(G):
        if m[g] == 0:
            assert np.array_equal(got[g], mg0[g]), g
        else:
            assert orc.rel_frobenius(got[g] - mg0[g], ref[g] - mg0[g]) <= TOL_BF16, g


# ----------------------------------------------------------------------------
# Full-size workloads, checked group by group on sampled outputs
# ----------------------------------------------------------------------------

FULL = ["bf16_g8", "fine_g64", "stacked_g128_uniform", "stacked_g128_ragged"]
ROWS_PER_GROUP = 8   # random rows per group, besides the group's first and last row
COLS = 64            # output columns sampled per group (fwd: of N, dgrad: of K)
WG = 8               # wgrad: WG x WG sampled (n, k) entries per group


def _idx(v):
    return torch.as_tensor(np.asarray(v, dtype=np.int64), device="cuda")


def _sampled_parity(name, pair):
    """Run fwd, dgrad and wgrad (accumulate) at full size, then check every
    non-empty group on its own against the oracle's single-entry products:
    its first, last and ROWS_PER_GROUP random rows x COLS random columns of y
    and dx, and WG x WG entries of main_grad, each within 5e-3 relative
    Frobenius error; empty groups keep main_grad bit-identical."""
    wl = synth.WORKLOADS[name]
    m = synth.m_splits_for(name)
    G, N, K, M = wl.G, wl.N, wl.K, wl.rows
    d = synth.operands(G, M, N, K, wl.seed, device="cuda", bias=wl.bias)
    off, st = offsets_on_device(m, M, wl.out_rows)
    y = sentinel_like(wl.out_rows, N)
    gl.gl_fwd(d["x"], d["w"], d.get("bias"), off, st, y, pair=pair)
    dx = sentinel_like(wl.out_rows, K)
    gl.gl_dgrad(d["dy"], d["w"], off, st, dx, pair=pair)
    mg = d["main_grad"].clone()
    gl.gl_wgrad(d["x"], d["dy"], off, st, mg, accumulate=True, pair=pair)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert untouched(y[M:]) and untouched(dx[M:])

    rng = np.random.default_rng(wl.seed)
    o = orc.offsets(m)
    checked = 0
    for g in range(G):
        a, b = int(o[g]), int(o[g + 1])
        if a == b:
            assert torch.equal(mg[g], d["main_grad"][g]), ("accumulate touched an empty group", g)
            continue
        rows = np.unique(np.concatenate([[a, b - 1], rng.integers(a, b, size=ROWS_PER_GROUP)]))
        ns = rng.choice(N, size=min(COLS, N), replace=False)
        ks = rng.choice(K, size=min(COLS, K), replace=False)
        xr, dyr = f64(d["x"][_idx(rows)]), f64(d["dy"][_idx(rows)])
        wr = f64(d["w"][g][_idx(ns)])            # [COLS, K]: rows n of W_g
        wc = f64(d["w"][g][:, _idx(ks)]).T       # [COLS, N]: columns k of W_g
        bias = f64(d["bias"][g]) if wl.bias else None
        ref_f = np.array([[orc.fwd_entry(xr[i], wr[j], None if bias is None else bias[n])
                           for j, n in enumerate(ns)] for i in range(len(rows))])
        got_f = f64(y[_idx(rows)][:, _idx(ns)])
        assert orc.rel_frobenius(got_f, ref_f) <= TOL_BF16, ("fwd", g)
        ref_d = np.array([[orc.dgrad_entry(dyr[i], wc[j]) for j in range(len(ks))] for i in range(len(rows))])
        got_d = f64(dx[_idx(rows)][:, _idx(ks)])
        assert orc.rel_frobenius(got_d, ref_d) <= TOL_BF16, ("dgrad", g)
        nw = rng.choice(N, size=WG, replace=False)
        kw = rng.choice(K, size=WG, replace=False)
        dyc = f64(d["dy"][a:b][:, _idx(nw)])
        xc = f64(d["x"][a:b][:, _idx(kw)])
        old = f64(d["main_grad"][g][_idx(nw)][:, _idx(kw)])
        new = f64(mg[g][_idx(nw)][:, _idx(kw)])
        ref_w = np.array([[orc.wgrad_entry(dyc[:, i], xc[:, j], old[i, j], True) for j in range(WG)]
                          for i in range(WG)])
        # the group's gradient (new - old) against the oracle's; old is ~1e-3
        assert orc.rel_frobenius(new - old, ref_w - old) <= TOL_BF16, ("wgrad", g)
        checked += 1
    assert checked == int((m > 0).sum())


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(name, pair):
    _sampled_parity(name, pair)
    torch.cuda.empty_cache()


# ----------------------------------------------------------------------------
# Bounded waits: a pipeline wait that runs out is reported, and the context
# stays usable
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("pair_", [False, True], ids=["single", "pair"])
def test_pipeline_wait_timeout_sets_status_and_recovers(pair_):
    """A call whose load warp is held (GL_OPT_HOLD_LOADS: no stage ever
    lands) with its pipeline waits bounded at 2 ms: every wait runs out,
    GL_DEV_TIMEOUT is ORed into the status word, the kernel returns, and it
    writes nothing (the output buffer keeps its sentinel, main_grad its
    bytes).  The same calls with the default options then match the oracle:
    the context is still usable."""
    G, N, K, m = 3, 512, 1024, [300, 0, 212]
    M = sum(m)
    d = _inputs(G, N, K, m, seed=41)
    off, st = offsets_on_device(m, M)
    y = sentinel_like(M, N)
    mg = d["main_grad"].clone()
    hold = dict(pair=pair_, wait_limit_us=2000, opt_flags=gl.GL_OPT_HOLD_LOADS)
    gl.gl_fwd(d["x"], d["w"], d["bias"], off, st, y, **hold)
    gl.gl_wgrad(d["x"], d["dy"], off, st, mg, accumulate=True, **hold)
    torch.cuda.synchronize()
    assert int(st.item()) == gl.GL_DEV_TIMEOUT
    assert untouched(y)
    assert torch.equal(mg, d["main_grad"])
    st.zero_()
    gl.gl_fwd(d["x"], d["w"], d["bias"], off, st, y, pair=pair_)
    gl.gl_wgrad(d["x"], d["dy"], off, st, mg, accumulate=True, pair=pair_)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    x64, w64, dy64 = f64(d["x"]), f64(d["w"]), f64(d["dy"])
    assert_groups_close(f64(y), orc.fwd(x64, w64, f64(d["bias"]), m), m, what="fwd after a timeout")
    mg0 = f64(d["main_grad"])
    ref = orc.wgrad(x64, dy64, m, mg0, True)
    got = f64(mg)
    for g in range(G):
        if m[g]:
            assert orc.rel_frobenius(got[g] - mg0[g], ref[g] - mg0[g]) <= TOL_BF16, g
