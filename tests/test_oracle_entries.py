"""Pins for the oracle's single-entry helpers and its acceptance metric (CPU).

The full-size GPU parity tests cannot run the whole fp64 products, so they
compare sampled outputs against ``fwd_entry`` / ``dgrad_entry`` /
``wgrad_entry`` and check every group with ``rel_frobenius``.  These helpers
are pinned here against things other than themselves:

* each entry helper against torch fp64 ``split`` -> ``F.linear`` -> ``cat``
  with autograd (``grouped_linear.py``, ``GroupedLinear`` docstring: one linear
  layer per split; ``fuser_backward``: dgrad "NN", wgrad "NT" accumulated into
  or overwriting main_grad), element by element on random ragged shapes;
* ``rel_frobenius`` against hand-worked values of ||got - ref|| / ||ref||;
* planted mistakes (a dropped ``old`` under accumulation, a doubled bias, a
  transposed weight, normalising by ||got||) that each check must reject.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import gl_oracle as orc

CASES = [
    (3, 12, 20, [5, 0, 9]),
    (4, 8, 33, [1, 7, 0, 12]),
    (1, 16, 24, [11]),
]


def _data(seed, G, N, K, m):
    rng = np.random.default_rng(seed)
    M = int(sum(m))
    return (rng.standard_normal((M, K)), rng.uniform(-1, 1, (G, N, K)) / math.sqrt(K),
            0.02 * rng.standard_normal((G, N)), rng.standard_normal((M, N)),
            1e-1 * rng.standard_normal((G, N, K)))


def _torch_products(x, w, b, dy, m):
    """split -> F.linear per split -> cat; autograd gives dgrad and wgrad."""
    xt = torch.tensor(x, requires_grad=True)
    ws = [torch.tensor(w[i], requires_grad=True) for i in range(len(m))]
    parts = torch.split(xt, [int(v) for v in m])
    y = torch.cat([F.linear(p, ws[i], torch.tensor(b[i])) for i, p in enumerate(parts)], dim=0)
    y.backward(torch.tensor(dy))
    dW = np.stack([wi.grad.numpy() if wi.grad is not None else np.zeros_like(w[0]) for wi in ws])
    return y.detach().numpy(), xt.grad.numpy(), dW


def _group_of(m):
    o = np.concatenate([[0], np.cumsum(m)])
    return o, np.repeat(np.arange(len(m)), m)


# -- checks, written once so that the planted mistakes run through the same code


def _check_fwd_entry(fn, case, bias=True):
    G, N, K, m = case
    x, w, b, dy, _ = _data(7 + G, G, N, K, m)
    if not bias:
        b = np.zeros_like(b)
    y, _, _ = _torch_products(x, w, b, dy, m)
    _, grp = _group_of(m)
    for r in range(x.shape[0]):
        g = grp[r]
        for n in range(N):
            v = fn(x[r], w[g, n], b[g, n] if bias else None)
            if not math.isclose(v, y[r, n], rel_tol=1e-12, abs_tol=1e-12):
                return False
    return True


def _check_dgrad_entry(fn, case):
    G, N, K, m = case
    x, w, b, dy, _ = _data(11 + G, G, N, K, m)
    _, dx, _ = _torch_products(x, w, b, dy, m)
    _, grp = _group_of(m)
    for r in range(x.shape[0]):
        g = grp[r]
        for k in range(K):
            if not math.isclose(fn(dy[r], w[g][:, k]), dx[r, k], rel_tol=1e-12, abs_tol=1e-12):
                return False
    return True


def _check_wgrad_entry(fn, case):
    G, N, K, m = case
    x, w, b, dy, old = _data(13 + G, G, N, K, m)
    _, _, dW = _torch_products(x, w, b, dy, m)
    o, _ = _group_of(m)
    for g in range(G):
        a, e = int(o[g]), int(o[g + 1])
        for n in range(N):
            for k in range(K):
                acc = fn(dy[a:e, n], x[a:e, k], old[g, n, k], True)
                over = fn(dy[a:e, n], x[a:e, k], old[g, n, k], False)
                if not math.isclose(acc, old[g, n, k] + dW[g, n, k], rel_tol=1e-12, abs_tol=1e-12):
                    return False
                if not math.isclose(over, dW[g, n, k], rel_tol=1e-12, abs_tol=1e-12):
                    return False
    return True


# (got, ref, ||got - ref|| / ||ref||) worked by hand
FROB_CASES = [
    ([1.0, 1.0], [1.0, 0.0], 1.0),
    ([2.0, 0.0], [1.0, 0.0], 1.0),                 # ||got|| = 2 would give 0.5
    ([0.0, 0.0], [3.0, 4.0], 1.0),                 # ||got|| = 0 would give inf
    ([3.0, 4.0], [3.0, 4.0], 0.0),
    ([1.0, 2.0], [1.0, 0.0], 2.0),
    ([[1.0, 2.0], [3.0, 4.0]], [[1.0, 2.0], [3.0, 5.0]], 1.0 / math.sqrt(39.0)),
    ([6.0, 8.0, 0.0], [3.0, 4.0, 0.0], 1.0),       # ||got|| = 10 would give 0.5
    ([0.0, 0.0], [0.0, 0.0], 0.0),                 # both zero: 0 by definition
    ([3.0, 4.0], [0.0, 0.0], math.inf),            # zero reference, non-zero result
]


def _check_frobenius(fn):
    for got, ref, want in FROB_CASES:
        v = fn(np.array(got), np.array(ref))
        if math.isinf(want):
            if not math.isinf(v):
                return False
        elif not math.isclose(v, want, rel_tol=1e-14, abs_tol=1e-15):
            return False
    return True


# -- the oracle's helpers pass


@pytest.mark.parametrize("case", CASES)
def test_fwd_entry_matches_split_linear_cat(case):
    assert _check_fwd_entry(orc.fwd_entry, case, bias=True)
    assert _check_fwd_entry(orc.fwd_entry, case, bias=False)


@pytest.mark.parametrize("case", CASES)
def test_dgrad_entry_matches_autograd(case):
    assert _check_dgrad_entry(orc.dgrad_entry, case)


@pytest.mark.parametrize("case", CASES)
def test_wgrad_entry_matches_autograd_accumulate_and_overwrite(case):
    assert _check_wgrad_entry(orc.wgrad_entry, case)


def test_rel_frobenius_hand_worked():
    assert _check_frobenius(orc.rel_frobenius)


def test_entries_agree_with_full_products():
    """The entry helpers and the full products give the same numbers."""
    G, N, K, m = 3, 10, 14, [4, 0, 6]
    x, w, b, dy, old = _data(3, G, N, K, m)
    y = orc.fwd(x, w, b, m)
    dx = orc.dgrad(dy, w, m)
    mg = orc.wgrad(x, dy, m, old, True)
    o, grp = _group_of(m)
    for r in range(x.shape[0]):
        g = grp[r]
        for n in range(N):
            assert math.isclose(orc.fwd_entry(x[r], w[g, n], b[g, n]), y[r, n], rel_tol=1e-12, abs_tol=1e-12)
        for k in range(K):
            assert math.isclose(orc.dgrad_entry(dy[r], w[g][:, k]), dx[r, k], rel_tol=1e-12, abs_tol=1e-12)
    for g in range(G):
        a, e = int(o[g]), int(o[g + 1])
        for n in range(N):
            for k in range(K):
                assert math.isclose(orc.wgrad_entry(dy[a:e, n], x[a:e, k], old[g, n, k], True), mg[g, n, k],
                                    rel_tol=1e-12, abs_tol=1e-12)


# -- planted mistakes are caught by the same checks


def test_planted_fwd_entry_mistakes_fail():
    doubled_bias = lambda xr, wr, b: orc.fwd_entry(xr, wr, b) + (0.0 if b is None else float(b))
    dropped_bias = lambda xr, wr, b: orc.fwd_entry(xr, wr, None)
    reversed_row = lambda xr, wr, b: orc.fwd_entry(xr, wr[::-1], b)
    for bad in (doubled_bias, dropped_bias, reversed_row):
        assert not _check_fwd_entry(bad, CASES[0], bias=True)


def test_planted_dgrad_entry_mistake_fails():
    wrong_sign = lambda dyr, wc: -orc.dgrad_entry(dyr, wc)
    shifted = lambda dyr, wc: orc.dgrad_entry(dyr, np.roll(wc, 1))
    for bad in (wrong_sign, shifted):
        assert not _check_dgrad_entry(bad, CASES[0])


def test_planted_wgrad_entry_mistakes_fail():
    drops_old = lambda dyc, xc, old, acc: float(np.dot(dyc, xc))
    keeps_old_always = lambda dyc, xc, old, acc: float(old) + float(np.dot(dyc, xc))
    one_row_short = lambda dyc, xc, old, acc: orc.wgrad_entry(dyc[:-1], xc[:-1], old, acc)
    for bad in (drops_old, keeps_old_always, one_row_short):
        assert not _check_wgrad_entry(bad, CASES[0])


def test_planted_frobenius_mistakes_fail():
    by_got = lambda got, ref: float(np.linalg.norm(got - ref) / np.linalg.norm(got)) if np.linalg.norm(got) else 0.0
    squared = lambda got, ref: orc.rel_frobenius(got, ref) ** 2
    max_norm = lambda got, ref: (float(np.max(np.abs(got - ref)) / np.max(np.abs(ref)))
                                 if np.max(np.abs(ref)) else orc.rel_frobenius(got, ref))
    for bad in (by_got, squared, max_norm):
        assert not _check_frobenius(bad)
