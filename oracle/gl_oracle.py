"""Plain CPU oracle for the grouped linear layer (fp64, numpy).

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
baseline leg of the benchmark may import this module.  The library itself never
calls it and shares no code with it: there is no common kernel, helper, table or
constant generator between this file and the CUDA sources.

What is computed, and where it is defined:

* ``offsets``      -- exclusive prefix sum of the split sizes with a leading
  zero, int64.  "Single parameter for GroupedLinear module" (TransformerEngine
  PR #2727), description of ``nvte_cumsum`` / ``build_grouped_tensor_offsets``.
* ``fwd``          -- y_i = x_i W_i^T + b_i on the rows of group i.
  ``grouped_linear.py`` (TransformerEngine ops/basic), ``GroupedLinear`` class
  docstring (split along dim 0, one linear per split, concatenate) and
  ``fuser_forward`` (grouped GEMM with per-group bias).
* ``dgrad``        -- dx_i = dy_i W_i.  ``grouped_linear.py``,
  ``fuser_backward``, "Perform dgrad GEMMs" (layout "NN").
* ``wgrad``        -- dW_i = dy_i^T x_i, added into main_grad or overwriting
  it.  ``grouped_linear.py``, ``fuser_backward``, "Initialize grad weight
  buffers" and "Perform wgrad GEMMs" (layout "NT", ``accumulate``).
* ``dbias``        -- column sums of dy_i.  ``grouped_linear.py``,
  ``fuser_backward``, ``grad_biases``.
* MXFP8 quantizer  -- E4M3 codes with one E8M0 power-of-two scale per block
  of 32 consecutive elements along the contraction dimension.
  ``grouped_linear.py``, ``_quantize_weights_mxfp8`` (E4M3 data, rowwise and
  columnwise scale shapes) and ``fuser_forward``/``fuser_backward``
  (``split_quantize``: each split quantized as its own tensor).  The scale
  rule (smallest power of two 2^e with amax <= 448 * 2^e) and the other points
  the pages leave open are listed in the design notes.
* MXFP8 GEMMs      -- the same three products on the dequantized operands
  q * 2^(s - 127).

Numerics: every product and sum is taken in float64.  bf16 inputs are exact in
float64; the fp64 result is what the GPU's fp32-accumulated result is compared
against (relative Frobenius error per group).
"""
from __future__ import annotations

from typing import Optional, Sequence, Union

import numpy as np

# ---------------------------------------------------------------------------
# bf16 <-> float64 (bit-level; numpy has no bf16 type)
# ---------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (uint16) as float64."""
    bits = np.asarray(bits, dtype=np.uint16)
    with np.errstate(invalid="ignore"):
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f64_to_bf16_rne(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even); return bits.

    Finite inputs of magnitude below the bf16 overflow threshold only.  Works
    on the value directly (one rounding), never through float32.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, e = np.frexp(a)                       # a = m * 2^e, m in [0.5, 1)
    # bf16 keeps 8 significant bits: quantum 2^(e-8); subnormal quantum 2^-133
    q = np.maximum(e - 8, -133)
    r = np.ldexp(np.rint(np.ldexp(a, -q)), q)  # rint: round half to even
    r = np.copysign(r, v)
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# Offsets (PR #2727, nvte_cumsum: prefix sum with leading zero)
# ---------------------------------------------------------------------------

DEV_NEG_SPLIT = 1      # some m_i < 0
DEV_SUM_MISMATCH = 2   # sum(m) != expected rows
DEV_OUT_OVERFLOW = 4   # sum(m) > rows of the output buffer


def offsets(m_splits: Sequence[int]) -> np.ndarray:
    """o[0] = 0, o[i+1] = o[i] + m_i, in int64 (G+1 entries)."""
    m = [int(v) for v in m_splits]
    o = [0]
    for v in m:
        o.append(o[-1] + v)
    return np.array(o, dtype=np.int64)


def split_status(m_splits: Sequence[int], expect_rows: int, out_rows: int) -> int:
    """Data errors the offset scan reports instead of a host-side check.

    The reference raises when the number of splits or their sizes do not
    match the input (``fuser_forward``: "Expected ... splits"; torch.split
    raises on a size mismatch; PR #3161 raises when the caller buffer is too
    small).  The scan reports those conditions as bit flags.
    """
    o = offsets(m_splits)
    flags = 0
    if any(int(v) < 0 for v in m_splits):
        flags |= DEV_NEG_SPLIT
    if int(o[-1]) != int(expect_rows):
        flags |= DEV_SUM_MISMATCH
    if int(o[-1]) > int(out_rows):
        flags |= DEV_OUT_OVERFLOW
    return flags


# ---------------------------------------------------------------------------
# Grouped products (grouped_linear.py, fuser_forward / fuser_backward)
# ---------------------------------------------------------------------------

Weights = Union[np.ndarray, Sequence[np.ndarray]]


def _w(w: Weights, i: int) -> np.ndarray:
    return np.asarray(w[i], dtype=np.float64)


def fwd(x: np.ndarray, w: Weights, bias: Optional[Weights], m_splits) -> np.ndarray:
    """y rows of group i = x_i @ W_i^T (+ b_i); returns float64 [sum(m), N].

    ``w`` is a stacked [G,N,K] array or a list of G [N,K] arrays; ``bias`` is
    [G,N], a list of [N] arrays, or None.
    """
    x = np.asarray(x, dtype=np.float64)
    o = offsets(m_splits)
    N = _w(w, 0).shape[0]
    y = np.zeros((int(o[-1]), N), dtype=np.float64)
    for i in range(len(m_splits)):
        a, b = int(o[i]), int(o[i + 1])
        if a == b:
            continue
        y[a:b] = x[a:b] @ _w(w, i).T
        if bias is not None:
            y[a:b] += np.asarray(bias[i], dtype=np.float64)[None, :]
    return y


def dgrad(dy: np.ndarray, w: Weights, m_splits) -> np.ndarray:
    """dx rows of group i = dy_i @ W_i; returns float64 [sum(m), K]."""
    dy = np.asarray(dy, dtype=np.float64)
    o = offsets(m_splits)
    K = _w(w, 0).shape[1]
    dx = np.zeros((int(o[-1]), K), dtype=np.float64)
    for i in range(len(m_splits)):
        a, b = int(o[i]), int(o[i + 1])
        if a == b:
            continue
        dx[a:b] = dy[a:b] @ _w(w, i)
    return dx


def wgrad(x: np.ndarray, dy: np.ndarray, m_splits, main_grad: Optional[np.ndarray],
          accumulate: bool) -> np.ndarray:
    """main_grad[i] (+)= dy_i^T @ x_i; returns float64 [G,N,K].

    With ``accumulate`` the old main_grad is added (Megatron-style wgrad
    fusion); without it the result overwrites main_grad, so an empty group
    yields zeros (the empty sum).
    """
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    o = offsets(m_splits)
    G = len(m_splits)
    N, K = dy.shape[1], x.shape[1]
    out = np.zeros((G, N, K), dtype=np.float64)
    for i in range(G):
        a, b = int(o[i]), int(o[i + 1])
        if accumulate:
            out[i] = np.asarray(main_grad[i], dtype=np.float64)
        if a != b:
            out[i] += dy[a:b].T @ x[a:b]
    return out


def dbias(dy: np.ndarray, m_splits) -> np.ndarray:
    """Column sums of dy over each group's rows; float64 [G,N]."""
    dy = np.asarray(dy, dtype=np.float64)
    o = offsets(m_splits)
    out = np.zeros((len(m_splits), dy.shape[1]), dtype=np.float64)
    for i in range(len(m_splits)):
        out[i] = dy[int(o[i]):int(o[i + 1])].sum(axis=0)
    return out


def fwd_rows(x_rows: np.ndarray, rows: np.ndarray, w: Weights, bias: Optional[Weights],
             m_splits) -> np.ndarray:
    """fwd for a sample of output rows only (global row indices ``rows``).

    ``x_rows[j]`` is input row ``rows[j]``.  Used to check full-size runs one
    row at a time.
    """
    o = offsets(m_splits)
    grp = np.searchsorted(o, rows, side="right") - 1
    out = []
    for j, r in enumerate(rows):
        g = int(grp[j])
        v = _w(w, g) @ np.asarray(x_rows[j], dtype=np.float64)
        if bias is not None:
            v = v + np.asarray(bias[g], dtype=np.float64)
        out.append(v)
    return np.array(out)


# ---------------------------------------------------------------------------
# MXFP8: E4M3 codes, E8M0 block scales (32 elements per block)
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0
MX_BLOCK = 32


def e4m3_value(code: int) -> float:
    """Value of an E4M3 code (OCP MX v1.0: bias 7, 3 mantissa bits, no inf).

    S.1111.111 is NaN; exponent field 0 holds subnormals m * 2^-9.
    """
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_table() -> np.ndarray:
    return np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def e8m0_exponent(amax: np.ndarray) -> np.ndarray:
    """Smallest integer e with amax <= 448 * 2^e, clamped to [-127, 127].

    Exact: with amax = f * 2^E (f in [0.5, 1)) and 448 = 0.875 * 2^9 the
    answer is E - 9 when f <= 0.875, else E - 8.  amax == 0 gives e = 0.
    """
    amax = np.asarray(amax, dtype=np.float64)
    f, E = np.frexp(amax)
    e = np.where(f <= 0.875, E - 9, E - 8)
    e = np.where(amax == 0.0, 0, e)
    return np.clip(e, -127, 127).astype(np.int64)


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Round to the nearest E4M3 value, ties to even, saturating at +-448."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, E = np.frexp(a)                      # a = f * 2^E, floor(log2 a) = E - 1
    q = np.where(a >= 2.0 ** -6, E - 1 - 3, -9)  # 3 fraction bits; subnormal step 2^-9
    r = np.ldexp(np.rint(np.ldexp(a, -q)), q)
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, v)


def e4m3_encode(r: np.ndarray) -> np.ndarray:
    """Bit pattern of values that are exactly representable in E4M3."""
    r = np.asarray(r, dtype=np.float64)
    a = np.abs(r)
    sign = np.signbit(r).astype(np.uint8) << np.uint8(7)
    _, E = np.frexp(a)
    normal = a >= 2.0 ** -6
    e_unb = E - 1
    exp_field = np.where(normal, e_unb + 7, 0)
    mant = np.where(normal, np.ldexp(a, -e_unb) * 8.0 - 8.0, np.ldexp(a, 9))
    mant = np.rint(mant).astype(np.int64)
    code = (exp_field.astype(np.int64) << 3) | mant
    return (code.astype(np.uint8) | sign).astype(np.uint8)


def quantize_block(vals: np.ndarray):
    """One MX block (<= 32 values, float64 exact bf16 values).

    Returns (codes uint8[len], scale byte).  The block's scale is 2^e with e
    from ``e8m0_exponent(amax)``; each code is E4M3(v * 2^-e).
    """
    vals = np.asarray(vals, dtype=np.float64)
    amax = np.max(np.abs(vals)) if vals.size else 0.0
    e = int(e8m0_exponent(amax))
    codes = e4m3_encode(e4m3_round(np.ldexp(vals, -e)))
    return codes, np.uint8(e + 127)


def quantize_rowwise(src: np.ndarray):
    """Blocks of 32 along the last dimension of a [rows, cols] array.

    Returns codes uint8[rows, cols] and scales uint8[rows, cols/32].
    """
    src = np.asarray(src, dtype=np.float64)
    rows, cols = src.shape
    assert cols % MX_BLOCK == 0
    blk = src.reshape(rows, cols // MX_BLOCK, MX_BLOCK)
    amax = np.max(np.abs(blk), axis=2)
    e = e8m0_exponent(amax)
    codes = e4m3_encode(e4m3_round(np.ldexp(blk, -e[:, :, None])))
    return codes.reshape(rows, cols), (e + 127).astype(np.uint8)


MMA_ATOM_BYTES = 512  # 128 operand rows x 4 blocks of 32 contraction elements


def mma_atom_byte(i: int, j: int) -> int:
    """Byte of operand row i (0..127) and block j (0..3) inside one 512-byte
    scale atom of the tcgen05 block-scaled MMA: 32 lines of 16 bytes; line
    i % 32 holds rows i, i+32, i+64, i+96 (4 bytes each, one per block)."""
    return (i % 32) * 16 + (i // 32) * 4 + j


def mma_offsets_rowwise(rows: int, cols: int) -> np.ndarray:
    """Byte offset of every rowwise scale [rows, cols/32] in the MMA layout.

    Atom (q, b) -- k-blocks 4q..4q+3 of rows 128b..128b+127 -- starts at
    byte (q * R + b) * 512, R = ceil(rows / 128) (k-group-major, so one
    k-group of consecutive row blocks is contiguous)."""
    assert cols % 128 == 0
    R = (rows + 127) // 128
    off = np.empty((rows, cols // MX_BLOCK), dtype=np.int64)
    for r in range(rows):
        for k in range(cols // MX_BLOCK):
            atom = (k // 4) * R + r // 128
            off[r, k] = atom * MMA_ATOM_BYTES + mma_atom_byte(r % 128, k % 4)
    return off


def mma_offsets_colwise(m_splits, cols: int) -> np.ndarray:
    """Byte offset of every columnwise scale [S, cols] (S = colwise_scale_rows
    total; row base_i + j = block j of group i) in the MMA layout.

    Group i owns k-groups T_i .. T_i + ceil(m_i/128) - 1 with
    T_i = sum_{l<i} ceil(m_l / 128); k-group T_i + t holds the group's blocks
    4t..4t+3; atom (T_i + t, c) -- columns 128c..128c+127 -- starts at byte
    ((T_i + t) * cols/128 + c) * 512."""
    assert cols % 128 == 0
    C = cols // 128
    base = colwise_scale_rows(m_splits)
    off = np.empty((int(base[-1]), cols), dtype=np.int64)
    T = 0
    for i, m in enumerate(m_splits):
        nblk = int(base[i + 1] - base[i])
        for j in range(nblk):
            kq = T + j // 4
            for n in range(cols):
                off[base[i] + j, n] = (kq * C + n // 128) * MMA_ATOM_BYTES + mma_atom_byte(n % 128, j % 4)
        T += (int(m) + 127) // 128
    return off


def colwise_scale_rows(m_splits) -> np.ndarray:
    """First scale row of each group in the columnwise scale array.

    Each group is quantized as its own tensor, so its blocks of 32 rows start
    at the group's first row and its last block may be partial; the groups'
    scale rows are packed: base_i = sum_{j<i} ceil(m_j / 32).  Returns G+1
    entries (the last is the total number of scale rows).
    """
    base = [0]
    for m in m_splits:
        base.append(base[-1] + (int(m) + MX_BLOCK - 1) // MX_BLOCK)
    return np.array(base, dtype=np.int64)


def quantize_colwise(src: np.ndarray, m_splits):
    """Blocks of 32 rows along dim 0, restarting at every group start.

    Returns codes uint8[rows, cols] (same positions as ``src``) and scales
    uint8[total_scale_rows, cols]; group i's block j is scale row
    ``colwise_scale_rows(m)[i] + j``.  A trailing partial block takes its
    amax over the rows it has.
    """
    src = np.asarray(src, dtype=np.float64)
    rows, cols = src.shape
    o = offsets(m_splits)
    base = colwise_scale_rows(m_splits)
    codes = np.zeros((rows, cols), dtype=np.uint8)
    scales = np.zeros((int(base[-1]), cols), dtype=np.uint8)
    for i in range(len(m_splits)):
        a, b = int(o[i]), int(o[i + 1])
        for j, r0 in enumerate(range(a, b, MX_BLOCK)):
            r1 = min(r0 + MX_BLOCK, b)
            blk = src[r0:r1]
            e = e8m0_exponent(np.max(np.abs(blk), axis=0))
            codes[r0:r1] = e4m3_encode(e4m3_round(np.ldexp(blk, -e[None, :])))
            scales[int(base[i]) + j] = (e + 127).astype(np.uint8)
    return codes, scales


_E4M3 = None


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    global _E4M3
    if _E4M3 is None:
        _E4M3 = e4m3_table()
    return _E4M3[np.asarray(codes, dtype=np.uint8)]


def dequant_rowwise(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """q * 2^(s-127) with the scale of each 32-block along the last dim."""
    rows, cols = codes.shape
    v = e4m3_decode(codes).reshape(rows, cols // MX_BLOCK, MX_BLOCK)
    e = scales.astype(np.int64) - 127
    return np.ldexp(v, e[:, :, None]).reshape(rows, cols)


def dequant_colwise(codes: np.ndarray, scales: np.ndarray, m_splits) -> np.ndarray:
    """Inverse of ``quantize_colwise``'s block assignment."""
    rows, cols = codes.shape
    v = e4m3_decode(codes)
    o = offsets(m_splits)
    base = colwise_scale_rows(m_splits)
    out = np.zeros((rows, cols), dtype=np.float64)
    for i in range(len(m_splits)):
        a, b = int(o[i]), int(o[i + 1])
        for j, r0 in enumerate(range(a, b, MX_BLOCK)):
            r1 = min(r0 + MX_BLOCK, b)
            e = scales[int(base[i]) + j].astype(np.int64) - 127
            out[r0:r1] = np.ldexp(v[r0:r1], e[None, :])
    return out


def fwd_mxfp8(xq, xs, wq, ws, bias, m_splits) -> np.ndarray:
    """fwd on dequantized operands: x rowwise [M,K], W rowwise [G,N,K]."""
    x = dequant_rowwise(xq, xs)
    G, N, K = wq.shape
    w = dequant_rowwise(wq.reshape(G * N, K), ws.reshape(G * N, K // MX_BLOCK)).reshape(G, N, K)
    return fwd(x, w, bias, m_splits)


def dgrad_mxfp8(dyq, dys, wq_c, ws_c, m_splits) -> np.ndarray:
    """dgrad on dequantized operands: dy rowwise [M,N] (blocks along N) and
    W columnwise (blocks of 32 along N inside every group's [N,K])."""
    dy = dequant_rowwise(dyq, dys)
    G, N, K = wq_c.shape
    w = dequant_colwise(wq_c.reshape(G * N, K), ws_c, [N] * G).reshape(G, N, K)
    return dgrad(dy, w, m_splits)


def wgrad_mxfp8(xq_c, xs_c, dyq_c, dys_c, m_splits, main_grad, accumulate) -> np.ndarray:
    """wgrad on dequantized columnwise operands (blocks along the rows of
    every group, the contraction dimension of dy_i^T x_i)."""
    x = dequant_colwise(xq_c, xs_c, m_splits)
    dy = dequant_colwise(dyq_c, dys_c, m_splits)
    return wgrad(x, dy, m_splits, main_grad, accumulate)


# ---------------------------------------------------------------------------
# Acceptance metric
# ---------------------------------------------------------------------------


def rel_frobenius(got: np.ndarray, ref: np.ndarray) -> float:
    """||got - ref||_F / ||ref||_F (0 when both are zero)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)


# ---------------------------------------------------------------------------
# Single output entries (for checking full-size runs on a sample)
# ---------------------------------------------------------------------------


def fwd_entry(x_row: np.ndarray, w_row: np.ndarray, b: Optional[float]) -> float:
    """y[r, n] = sum_k x[r, k] W_g[n, k] (+ b_g[n]) for one (r, n)."""
    v = float(np.dot(np.asarray(x_row, np.float64), np.asarray(w_row, np.float64)))
    return v + (0.0 if b is None else float(b))


def dgrad_entry(dy_row: np.ndarray, w_col: np.ndarray) -> float:
    """dx[r, k] = sum_n dy[r, n] W_g[n, k] for one (r, k)."""
    return float(np.dot(np.asarray(dy_row, np.float64), np.asarray(w_col, np.float64)))


def wgrad_entry(dy_col: np.ndarray, x_col: np.ndarray, old: float, accumulate: bool) -> float:
    """main_grad_g[n, k] (+)= sum_{r in g} dy[r, n] x[r, k] for one (g, n, k);
    ``dy_col`` / ``x_col`` hold the group's rows only."""
    v = float(np.dot(np.asarray(dy_col, np.float64), np.asarray(x_col, np.float64)))
    return (float(old) if accumulate else 0.0) + v
