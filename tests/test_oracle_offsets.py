"""Pins for the oracle's offset scan and split-size status flags (CPU only).

Offsets: "Single parameter for GroupedLinear module" (TransformerEngine PR
#2727) describes nvte_cumsum as a prefix sum with a leading zero over int64
split sizes, tested on known values, sizes 1, 2, 17, 256, 257, 513, 1024 and
negative entries.
"""
import json
import os

import numpy as np
import pytest

from oracle import gl_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_known_values():
    with open(os.path.join(GOLDEN, "offsets_known.json")) as f:
        data = json.load(f)
    for case in data["cases"]:
        got = orc.offsets(case["m"])
        assert got.dtype == np.int64
        assert got.tolist() == case["offsets"], case


@pytest.mark.parametrize("n", [1, 2, 17, 256, 257, 513, 1024])
def test_sizes_with_negatives_match_closed_form(n):
    rng = np.random.default_rng(n)
    m = rng.integers(-1000, 5000, size=n)
    got = orc.offsets(m)
    assert got.shape == (n + 1,)
    assert got[0] == 0
    # closed form o[i] = sum_{j<i} m_j, each entry summed independently
    for i in range(0, n + 1, max(1, n // 37)):
        assert got[i] == int(sum(int(v) for v in m[:i]))
    # the scan's differences give back the sizes
    assert np.array_equal(np.diff(got), m)


def test_int64_no_overflow():
    m = [2**40, 2**40, -(2**39)]
    assert orc.offsets(m).tolist() == [0, 2**40, 2**41, 2**41 - 2**39]


def test_status_flags():
    assert orc.split_status([1, 2, 3], 6, 6) == 0
    assert orc.split_status([1, -2, 7], 6, 6) == orc.DEV_NEG_SPLIT
    assert orc.split_status([1, 2, 3], 7, 10) == orc.DEV_SUM_MISMATCH
    assert orc.split_status([4, 4], 8, 6) == orc.DEV_OUT_OVERFLOW
    assert orc.split_status([4, 5], 8, 6) == orc.DEV_SUM_MISMATCH | orc.DEV_OUT_OVERFLOW
    assert orc.split_status([0, 0], 0, 0) == 0
