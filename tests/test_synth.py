"""The seeded input recipes hold what the workload table states.

Split sizes sum to the workload's rows and have its structure (Dirichlet
splits, Zipf(1.2) with four empty groups, multiples of 128 for the MXFP8
workload, 512 rows per group for the uniform stacked one); they are
reproducible from the seed; the operand draws have the stated distributions
(x, dy ~ N(0,1), W ~ U(+-1/sqrt(K)), bias ~ N(0, 0.02), main_grad ~ 1e-3 N(0,1))
and the integer mode stays in {-1, 0, 1}.  CPU only.
"""
import numpy as np
import pytest
import torch

from grouped_gemm_splits_b200 import synth


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
def test_splits_sum_and_shape(name):
    w = synth.WORKLOADS[name]
    m = synth.m_splits_for(name)
    assert m.dtype == np.int64 and m.shape == (w.G,)
    assert int(m.sum()) == w.rows and (m >= 0).all()
    assert w.out_rows >= w.rows
    assert np.array_equal(m, synth.m_splits_for(name))  # seeded: reproducible


def test_split_structures():
    assert synth.m_splits_for("tiny").tolist() == [0, 96, 160, 256]
    fine = synth.m_splits_for("fine_g64")
    assert int((fine == 0).sum()) == 4
    # Zipf(1.2) over 64 groups: the largest group holds a large share
    assert fine.max() > 0.15 * fine.sum()
    mx = synth.m_splits_for("mxfp8_g8")
    assert (mx % 128 == 0).all()
    uni = synth.m_splits_for("stacked_g128_uniform")
    assert (uni == 512).all()
    rag = synth.m_splits_for("stacked_g128_ragged")
    # Dirichlet(0.3) over 128 groups is far from uniform
    assert rag.max() > 4 * 512 and rag.min() < 512 // 4
    # a different seed gives different Dirichlet splits
    assert not np.array_equal(synth.m_splits_for("bf16_g8"), synth.m_splits_for("bf16_g8", seed=7))


def test_random_splits_helper():
    rng = np.random.default_rng(0)
    for align in (1, 32, 128):
        m = synth.random_splits(rng, 17, 128 * 40, align=align)
        assert int(m.sum()) == 128 * 40 and (m % align == 0).all() and (m >= 0).all()


def test_operand_distributions():
    G, M, N, K = 3, 4096, 256, 1024
    d = synth.operands(G, M, N, K, seed=5, bias=True)
    assert d["x"].dtype == torch.bfloat16 and d["w"].dtype == torch.bfloat16
    assert d["main_grad"].dtype == torch.float32
    assert d["w"].shape == (G, N, K) and d["bias"].shape == (G, N)
    x = d["x"].double()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1.0) < 0.01
    dy = d["dy"].double()
    assert abs(dy.mean().item()) < 0.01 and abs(dy.std().item() - 1.0) < 0.01
    w = d["w"].double()
    bound = 1.0 / np.sqrt(K)
    assert w.abs().max().item() <= bound * (1 + 2 ** -8)  # bf16 rounding of the bound
    assert abs(w.std().item() - bound / np.sqrt(3.0)) < 0.02 * bound  # uniform: bound / sqrt(3)
    b = d["bias"].double()
    assert abs(b.std().item() - 0.02) < 0.003
    mg = d["main_grad"].double()
    assert abs(mg.std().item() - 1e-3) < 2e-5
    e = synth.operands(G, M, N, K, seed=5, bias=True)
    assert torch.equal(d["x"], e["x"]) and torch.equal(d["w"], e["w"])  # seeded


def test_integer_operands_range():
    d = synth.integer_operands(2, 300, 64, 32, seed=1)
    for k in ("x", "w", "dy"):
        assert set(torch.unique(d[k].float()).tolist()) <= {-1.0, 0.0, 1.0}, k
    assert d["bias"].abs().max().item() <= 8
    assert d["main_grad"].abs().max().item() <= 64
