"""Pins for the oracle's grouped products (CPU only).

The grouped linear is defined in ``grouped_linear.py`` (TransformerEngine
ops/basic), ``GroupedLinear`` docstring: split the input along dim 0, apply an
independent linear layer to every split, concatenate.  The checks below pin the
oracle against that definition as computed by torch (fp64 CPU, autograd for the
gradients), against brute-force loops, and against invariants the pages fix:
empty groups, the stacked weight equal to per-group weights, and
accumulate-vs-overwrite of main_grad (``fuser_backward``).
"""
import itertools

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import gl_oracle as orc


def _rand(seed, G, N, K, m):
    rng = np.random.default_rng(seed)
    M = int(sum(m))
    x = rng.standard_normal((M, K))
    w = rng.uniform(-1, 1, (G, N, K)) / np.sqrt(K)
    b = 0.02 * rng.standard_normal((G, N))
    dy = rng.standard_normal((M, N))
    mg = 1e-3 * rng.standard_normal((G, N, K))
    return x, w, b, dy, mg


def _torch_reference(x, w, b, dy, m):
    """split -> one F.linear per split -> cat, and autograd for the grads."""
    xt = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    ws = [torch.tensor(w[i], dtype=torch.float64, requires_grad=True) for i in range(len(m))]
    bs = [torch.tensor(b[i], dtype=torch.float64, requires_grad=True) for i in range(len(m))]
    parts = torch.split(xt, [int(v) for v in m])
    y = torch.cat([F.linear(p, ws[i], bs[i]) for i, p in enumerate(parts)], dim=0)
    y.backward(torch.tensor(dy, dtype=torch.float64))
    dW = np.stack([wi.grad.numpy() if wi.grad is not None else np.zeros_like(w[0]) for wi in ws])
    db = np.stack([bi.grad.numpy() if bi.grad is not None else np.zeros_like(b[0]) for bi in bs])
    return y.detach().numpy(), xt.grad.numpy(), dW, db


CASES = [
    (1, 16, 24, [37]),              # G=1: a plain linear layer
    (4, 32, 16, [0, 5, 11, 16]),    # leading empty group
    (5, 8, 40, [3, 0, 0, 9, 1]),    # empty groups in the middle
    (3, 64, 32, [17, 33, 0]),       # trailing empty group
]


@pytest.mark.parametrize("G,N,K,m", CASES)
def test_matches_split_linear_cat(G, N, K, m):
    x, w, b, dy, mg = _rand(G + N, G, N, K, m)
    y_ref, dx_ref, dW_ref, db_ref = _torch_reference(x, w, b, dy, m)
    np.testing.assert_allclose(orc.fwd(x, w, b, m), y_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(orc.dgrad(dy, w, m), dx_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(orc.wgrad(x, dy, m, None, False), dW_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(orc.dbias(dy, m), db_ref, rtol=1e-12, atol=1e-12)


def test_brute_force_tiny():
    G, N, K, m = 3, 3, 4, [2, 0, 3]
    x, w, b, dy, mg = _rand(7, G, N, K, m)
    o = [0, 2, 2, 5]
    y = orc.fwd(x, w, b, m)
    dx = orc.dgrad(dy, w, m)
    dW = orc.wgrad(x, dy, m, mg, True)
    for g in range(G):
        for r in range(o[g], o[g + 1]):
            for n in range(N):
                s = b[g, n]
                for k in range(K):
                    s += x[r, k] * w[g, n, k]
                assert abs(y[r, n] - s) < 1e-12
            for k in range(K):
                s = 0.0
                for n in range(N):
                    s += dy[r, n] * w[g, n, k]
                assert abs(dx[r, k] - s) < 1e-12
        for n, k in itertools.product(range(N), range(K)):
            s = mg[g, n, k]
            for r in range(o[g], o[g + 1]):
                s += dy[r, n] * x[r, k]
            assert abs(dW[g, n, k] - s) < 1e-12


def test_stacked_equals_per_group_lists():
    G, N, K, m = 4, 16, 32, [5, 0, 9, 2]
    x, w, b, dy, mg = _rand(3, G, N, K, m)
    wl = [w[i].copy() for i in range(G)]
    bl = [b[i].copy() for i in range(G)]
    assert np.array_equal(orc.fwd(x, w, b, m), orc.fwd(x, wl, bl, m))
    assert np.array_equal(orc.dgrad(dy, w, m), orc.dgrad(dy, wl, m))


def test_accumulate_is_overwrite_plus_old_and_empty_groups():
    G, N, K, m = 4, 8, 16, [0, 7, 0, 5]
    x, w, b, dy, mg = _rand(11, G, N, K, m)
    over = orc.wgrad(x, dy, m, mg, False)
    acc = orc.wgrad(x, dy, m, mg, True)
    np.testing.assert_allclose(acc, over + mg, rtol=0, atol=1e-15)
    # empty groups: overwrite gives exact zeros, accumulate leaves main_grad as is
    for g in (0, 2):
        assert np.all(over[g] == 0.0)
        assert np.array_equal(acc[g], mg[g])
    # fwd/dgrad have no rows for an empty group: total rows is sum(m)
    assert orc.fwd(x, w, b, m).shape == (12, N)


def test_no_bias_and_all_rows_in_one_group():
    G, N, K, m = 3, 8, 8, [0, 10, 0]
    x, w, b, dy, mg = _rand(5, G, N, K, m)
    np.testing.assert_allclose(orc.fwd(x, w, None, m), x @ w[1].T, rtol=1e-13)
    np.testing.assert_allclose(orc.dgrad(dy, w, m), dy @ w[1], rtol=1e-13)


def test_all_groups_empty():
    G, N, K, m = 3, 8, 8, [0, 0, 0]
    x, w, b, dy, mg = _rand(5, G, N, K, m)
    assert orc.fwd(x, w, b, m).shape == (0, N)
    assert np.all(orc.wgrad(x, dy, m, mg, False) == 0)
    assert np.array_equal(orc.wgrad(x, dy, m, mg, True), mg)


def test_integer_mode_is_exact():
    # {-1,0,1} operands: every partial sum is an exact small integer
    rng = np.random.default_rng(0)
    G, N, K, m = 4, 32, 64, [0, 20, 30, 14]
    M = sum(m)
    x = rng.integers(-1, 2, (M, K)).astype(np.float64)
    w = rng.integers(-1, 2, (G, N, K)).astype(np.float64)
    b = rng.integers(-8, 9, (G, N)).astype(np.float64)
    y = orc.fwd(x, w, b, m)
    assert np.all(y == np.rint(y)) and np.abs(y).max() <= K + 8
    xi, wi = x.astype(np.int64), w.astype(np.int64)
    o = orc.offsets(m)
    for g in range(G):
        a, c = int(o[g]), int(o[g + 1])
        assert np.array_equal(y[a:c].astype(np.int64), xi[a:c] @ wi[g].T + b[g].astype(np.int64))


def test_fwd_rows_sample_matches_full():
    G, N, K, m = 4, 16, 8, [3, 0, 6, 4]
    x, w, b, dy, mg = _rand(9, G, N, K, m)
    full = orc.fwd(x, w, b, m)
    rows = np.array([0, 2, 3, 8, 9, 12])
    np.testing.assert_allclose(orc.fwd_rows(x[rows], rows, w, b, m), full[rows], rtol=1e-14)


def test_bf16_round_trip_and_rounding():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    v = orc.bf16_to_f64(bits)
    fin = np.isfinite(v)
    # every finite bf16 value rounds to itself
    assert np.array_equal(orc.f64_to_bf16_rne(v[fin]) & 0x7FFF, bits[fin] & 0x7FFF)
    # midpoint between 1 and 1+2^-7 rounds to even (1.0); just above rounds up
    assert orc.f64_to_bf16_rne(np.array([1 + 2.0**-8]))[0] == 0x3F80
    assert orc.f64_to_bf16_rne(np.array([1 + 3 * 2.0**-8]))[0] == 0x3F82
    assert orc.f64_to_bf16_rne(np.array([1 + 2.0**-8 + 2.0**-30]))[0] == 0x3F81


def test_planted_mistakes_are_caught():
    """A transposed weight or a dropped bias in the oracle fails the pins."""
    G, N, K, m = 2, 8, 8, [3, 4]
    x, w, b, dy, mg = _rand(1, G, N, K, m)
    y_ref, dx_ref, _, _ = _torch_reference(x, w, b, dy, m)
    wt = np.transpose(w, (0, 2, 1)).copy()
    assert not np.allclose(orc.fwd(x, wt, b, m), y_ref)
    assert not np.allclose(orc.fwd(x, w, None, m), y_ref)
    assert not np.allclose(orc.dgrad(dy, wt, m), dx_ref)
