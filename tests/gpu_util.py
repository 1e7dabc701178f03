"""Helpers shared by the GPU parity tests (host-side comparisons only)."""
from __future__ import annotations

import numpy as np
import torch

from grouped_gemm_splits_b200 import gl, synth
from oracle import gl_oracle as orc

# Acceptance bound for bf16 outputs and fp32 wgrad: relative Frobenius error
# per group against the fp64 oracle.
TOL_BF16 = 5e-3

SENTINEL_BF16 = -1  # 0xFFFF as int16: a NaN pattern no kernel result can equal


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bf16 / fp32 tensor."""
    if t.dtype == torch.bfloat16:
        return orc.bf16_to_f64(synth.bf16_bits(t))
    return t.detach().cpu().double().numpy()


def offsets_on_device(m, M, out_rows=None, device="cuda"):
    m_t = torch.tensor(np.asarray(m, dtype=np.int64), device=device)
    return gl.gl_offsets(m_t, int(M), out_rows)


def per_group_errors(got: np.ndarray, ref: np.ndarray, m) -> list:
    o = orc.offsets(m)
    errs = []
    for g in range(len(m)):
        a, b = int(o[g]), int(o[g + 1])
        if a == b:
            continue
        errs.append(orc.rel_frobenius(got[a:b], ref[a:b]))
    return errs


def assert_groups_close(got, ref, m, tol=TOL_BF16, what=""):
    errs = per_group_errors(got, ref, m)
    assert max(errs, default=0.0) <= tol, (what, errs)


def sentinel_like(rows: int, cols: int, device="cuda") -> torch.Tensor:
    return torch.full((rows, cols), SENTINEL_BF16, dtype=torch.int16, device=device).view(torch.bfloat16)


def untouched(t: torch.Tensor) -> bool:
    return bool((t.view(torch.int16) == SENTINEL_BF16).all().item())


def sample_rows(m, per_group: int, rng) -> np.ndarray:
    """First, last and random rows of every non-empty group."""
    o = orc.offsets(m)
    rows = []
    for g in range(len(m)):
        a, b = int(o[g]), int(o[g + 1])
        if a == b:
            continue
        rows += [a, b - 1]
        rows += list(rng.integers(a, b, size=per_group))
    return np.unique(np.array(rows, dtype=np.int64))
