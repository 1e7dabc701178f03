"""gl_offsets on the GPU against the oracle: bit-exact offsets and status flags.

Sizes follow the nvte_cumsum test described in "Single parameter for
GroupedLinear module" (TransformerEngine PR #2727): 1, 2, 17, 256, 257, 513,
1024 entries with negative values, plus chunk boundaries of the scan.
"""
import numpy as np
import pytest
import torch

from grouped_gemm_splits_b200 import gl
from oracle import gl_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n", [1, 2, 17, 256, 257, 513, 1024, 1025, 2048, 4096])
def test_offsets_bit_exact(n):
    rng = np.random.default_rng(n)
    m = rng.integers(-500, 5000, size=n).astype(np.int64)
    m_t = torch.tensor(m, device="cuda")
    total = int(m.sum())
    off, st = gl.gl_offsets(m_t, total, total + 10)
    assert np.array_equal(off.cpu().numpy(), orc.offsets(m))
    assert int(st.item()) == orc.split_status(m, total, total + 10)


def test_offsets_large_values_int64():
    m = np.array([2**40, 2**40, 3], dtype=np.int64)
    off, st = gl.gl_offsets(torch.tensor(m, device="cuda"), int(m.sum()), int(m.sum()))
    assert off.cpu().tolist() == orc.offsets(m).tolist()
    assert int(st.item()) == 0


@pytest.mark.parametrize("m,expect,out_rows", [
    ([1, 2, 3], 6, 6), ([1, -2, 7], 6, 6), ([1, 2, 3], 7, 10), ([4, 4], 8, 6), ([4, 5], 8, 6), ([0, 0], 0, 0),
])
def test_status_flags(m, expect, out_rows):
    off, st = gl.gl_offsets(torch.tensor(m, dtype=torch.int64, device="cuda"), expect, out_rows)
    assert int(st.item()) == orc.split_status(m, expect, out_rows)
    assert off.cpu().tolist() == orc.offsets(m).tolist()
