"""Seeded synthetic inputs for the grouped-linear workloads.

This module only draws random numbers: group split sizes and operand tensors
with the value distributions of the workloads below.  It holds none of the
grouped-linear arithmetic, so both the CPU oracle checks and the CUDA path can
take their inputs from here without sharing any computation.

Workloads (sizes are the ones the grouped expert linear is exercised at):

* ``tiny``          G=4,   K=128,  N=256,   rows 512, splits [0,96,160,256]
* ``bf16_g8``       G=8,   K=4096, N=14336, rows 16384, Multinomial(Dirichlet(1))
* ``fine_g64``      G=64,  K=2048, N=1408,  rows 32768, Zipf(1.2) with 4 empty
                    groups, output buffer of 33792 rows (1024-row padded tail)
* ``mxfp8_g8``      bf16_g8 shapes, splits 128 * Multinomial(128, Dirichlet(1))
* ``stacked_g128_uniform``  G=128, K=7168, N=2048, rows 65536, 512 per group
* ``stacked_g128_ragged``   same shapes, Multinomial(Dirichlet(0.3))

Distributions: x, dy ~ N(0,1); W ~ U(-1/sqrt(K), 1/sqrt(K)) (the
kaiming-uniform(a=sqrt(5)) init of a linear layer); bias ~ N(0, 0.02);
initial fp32 main_grad ~ 1e-3 * N(0,1).  Seed = 1234 + workload index.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    G: int
    K: int
    N: int
    rows: int
    bias: bool
    out_rows: int  # rows of the caller output buffer (>= rows)

    @property
    def seed(self) -> int:
        return 1234 + self.index


WORKLOADS = {
    w.name: w
    for w in (
        Workload("tiny", 1, 4, 128, 256, 512, True, 512),
        Workload("bf16_g8", 2, 8, 4096, 14336, 16384, False, 16384),
        Workload("fine_g64", 3, 64, 2048, 1408, 32768, True, 33792),
        Workload("mxfp8_g8", 4, 8, 4096, 14336, 16384, False, 16384),
        Workload("stacked_g128_uniform", 5, 128, 7168, 2048, 65536, False, 65536),
        Workload("stacked_g128_ragged", 6, 128, 7168, 2048, 65536, False, 65536),
    )
}


def m_splits_for(name: str, seed: Optional[int] = None) -> np.ndarray:
    """Group row counts (int64[G]) for a named workload."""
    w = WORKLOADS[name]
    rng = np.random.default_rng(w.seed if seed is None else seed)
    if name == "tiny":
        return np.array([0, 96, 160, 256], dtype=np.int64)
    if name == "bf16_g8":
        p = rng.dirichlet(np.ones(w.G))
        return rng.multinomial(w.rows, p).astype(np.int64)
    if name == "fine_g64":
        ranks = rng.permutation(w.G) + 1
        p = ranks.astype(np.float64) ** -1.2
        zero = rng.choice(w.G, size=4, replace=False)
        p[zero] = 0.0
        p /= p.sum()
        return rng.multinomial(w.rows, p).astype(np.int64)
    if name == "mxfp8_g8":
        p = rng.dirichlet(np.ones(w.G))
        return (128 * rng.multinomial(w.rows // 128, p)).astype(np.int64)
    if name == "stacked_g128_uniform":
        return np.full(w.G, w.rows // w.G, dtype=np.int64)
    if name == "stacked_g128_ragged":
        p = rng.dirichlet(np.full(w.G, 0.3))
        return rng.multinomial(w.rows, p).astype(np.int64)
    raise KeyError(name)


def random_splits(rng: np.random.Generator, G: int, rows: int, p_empty: float = 0.2,
                  align: int = 1) -> np.ndarray:
    """Ragged split sizes summing to ``rows`` with some empty groups (for tests)."""
    assert rows % align == 0
    w = rng.dirichlet(np.full(G, 0.5))
    w[rng.random(G) < p_empty] = 0.0
    if w.sum() == 0:
        w[rng.integers(G)] = 1.0
    w /= w.sum()
    return (align * rng.multinomial(rows // align, w)).astype(np.int64)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def operands(G: int, rows: int, N: int, K: int, seed: int, device="cpu",
             bias: bool = False, dy: bool = True, main_grad: bool = True,
             out_rows: Optional[int] = None) -> dict:
    """Draw x, W (stacked [G,N,K]), bias, dy and an initial fp32 main_grad.

    All floating tensors except main_grad are bf16.  Draws happen on ``device``
    (a CUDA generator for large workloads, the CPU one for small ones).
    """
    g = _gen(device, seed)
    out = {}
    out["x"] = torch.randn(rows, K, generator=g, device=device).to(torch.bfloat16)
    bound = 1.0 / float(np.sqrt(K))
    w = torch.empty(G, N, K, device=device, dtype=torch.float32)
    w.uniform_(-bound, bound, generator=g)
    out["w"] = w.to(torch.bfloat16)
    del w
    if bias:
        out["bias"] = (0.02 * torch.randn(G, N, generator=g, device=device)).to(torch.bfloat16)
    if dy:
        out["dy"] = torch.randn(rows, N, generator=g, device=device).to(torch.bfloat16)
    if main_grad:
        out["main_grad"] = 1e-3 * torch.randn(G, N, K, generator=g, device=device)
    return out


def integer_operands(G: int, rows: int, N: int, K: int, seed: int, device="cpu") -> dict:
    """Operands with values in {-1,0,1} and small integer biases.

    Every partial sum of the three products is then a small integer, exact in
    fp32 and (for |value| <= 256) in bf16, whatever the summation order.
    """
    g = _gen(device, seed)
    out = {}
    out["x"] = torch.randint(-1, 2, (rows, K), generator=g, device=device).to(torch.bfloat16)
    out["w"] = torch.randint(-1, 2, (G, N, K), generator=g, device=device).to(torch.bfloat16)
    out["bias"] = torch.randint(-8, 9, (G, N), generator=g, device=device).to(torch.bfloat16)
    out["dy"] = torch.randint(-1, 2, (rows, N), generator=g, device=device).to(torch.bfloat16)
    out["main_grad"] = torch.randint(-64, 65, (G, N, K), generator=g, device=device).to(torch.float32)
    return out


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a bf16 tensor (moved to host)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
