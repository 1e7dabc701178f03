"""Pins for the oracle's MXFP8 quantizer and MXFP8 products (CPU only).

MXFP8 as used by the grouped linear (``grouped_linear.py``, TransformerEngine
ops/basic, ``_quantize_weights_mxfp8``): E4M3 data, one E8M0 power-of-two
scale per 32 elements along the contraction dimension, rowwise and columnwise
copies, every split quantized as its own tensor (``split_quantize``).  The
E4M3 and E8M0 encodings are the OCP Microscaling v1.0 ones.

Pins: hand-worked blocks (golden file), an exhaustive sweep over all finite bf16
values checked against a brute-force nearest-value search in an independently
built code table and an exact rational scale search, invariants, and the
columnwise quantizer reducing to the rowwise one on transposed data.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import gl_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _pad(vals):
    v = np.zeros(32)
    v[: len(vals)] = vals
    return v


def test_hand_worked_blocks():
    with open(os.path.join(GOLDEN, "mxfp8_blocks.json")) as f:
        data = json.load(f)
    for case in data["cases"]:
        codes, scale = orc.quantize_block(_pad(case["block"]))
        assert int(scale) == case["scale"], case
        n = len(case["codes"])
        assert codes[:n].tolist() == case["codes"], case
        assert np.all(codes[n:] == 0)


def _table_from_definition():
    """E4M3 values built from the format's field layout, written independently
    of the oracle: 1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent 0 is
    subnormal; S.1111.111 is NaN."""
    vals = {}
    for code in range(0x7F):          # positive finite codes 0x00..0x7E
        e, mnt = code >> 3, code & 7
        if e == 0:
            vals[code] = Fraction(mnt, 8) * Fraction(1, 2**6)
        else:
            vals[code] = (1 + Fraction(mnt, 8)) * (Fraction(2) ** (e - 7))
    return vals


def _scale_exponent_exact(amax: float) -> int:
    """Smallest integer e with amax <= 448 * 2^e, by exact rational search."""
    if amax == 0:
        return 0
    a = Fraction(amax)
    e = -200
    while a > 448 * Fraction(2) ** e:
        e += 1
    return max(-127, min(127, e))


def _nearest_code(v: Fraction, table):
    """Brute-force nearest E4M3 code to |v| (ties to the even code)."""
    best = None
    for code, t in table.items():
        d = abs(v - t)
        key = (d, code & 1)
        if best is None or key < best[0]:
            best = (key, code)
    return best[1]


def test_code_table_matches_definition():
    table = _table_from_definition()
    dec = orc.e4m3_table()
    for code, t in table.items():
        assert dec[code] == float(t)
        assert dec[code | 0x80] == -float(t)
    assert np.isnan(dec[0x7F]) and np.isnan(dec[0xFF])
    assert dec[0x7E] == 448.0


def test_exhaustive_bf16_single_element_blocks():
    """Every finite bf16 value, alone in a block: scale and code are exact."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = orc.bf16_to_f64(bits)
    vals = vals[np.isfinite(vals)]
    # scale exponents, vectorised oracle vs exact rational search on a sample
    e = orc.e8m0_exponent(np.abs(vals))
    rng = np.random.default_rng(0)
    for i in rng.choice(len(vals), 3000, replace=False):
        assert e[i] == _scale_exponent_exact(abs(float(vals[i]))), vals[i]
    # codes: the scaled element is checked against brute-force nearest search
    codes = orc.e4m3_encode(orc.e4m3_round(np.ldexp(vals, -e)))
    table = _table_from_definition()
    tv = np.array([float(table[c]) for c in range(0x7F)])
    scaled = np.abs(np.ldexp(vals, -e))
    # vectorised nearest with tie -> even code, then exact spot checks
    d = np.abs(scaled[:, None] - tv[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = (d == dmin)
    odd = (np.arange(0x7F) & 1).astype(bool)
    pick_even = cand & ~odd[None, :]
    choose = np.where(pick_even.any(axis=1), np.argmax(pick_even, axis=1), np.argmax(cand, axis=1))
    expect = choose.astype(np.uint8) | (np.signbit(vals).astype(np.uint8) << 7)
    assert np.array_equal(codes, expect)
    for i in rng.choice(len(vals), 300, replace=False):
        c = _nearest_code(Fraction(float(scaled[i])), table)
        assert (int(codes[i]) & 0x7F) == c


def test_invariants_random_blocks():
    rng = np.random.default_rng(1)
    src = rng.standard_normal((64, 256)) * np.exp(rng.uniform(-20, 20, (64, 1)))
    src = orc.bf16_to_f64(orc.f64_to_bf16_rne(src))
    codes, scales = orc.quantize_rowwise(src)
    deq = orc.dequant_rowwise(codes, scales)
    q = orc.e4m3_decode(codes)
    assert np.all(np.abs(q) <= 448.0)
    blk = np.abs(q).reshape(64, 8, 32).max(axis=2)
    # the scaled amax lies in (224, 448]; rounding can take it down to 224
    assert np.all((blk >= 224.0) & (blk <= 448.0))
    amax = np.abs(src).reshape(64, 8, 32).max(axis=2)
    scaled = np.ldexp(amax, 127 - scales.astype(np.int64))
    assert np.all((scaled > 224.0) & (scaled <= 448.0))
    # relative error of every element is within half an E4M3 ulp of its block
    err = np.abs(deq - src)
    step = np.ldexp(1.0, scales.astype(np.int64) - 127 - 9)  # subnormal step of the block
    rel_bound = np.maximum(np.abs(src) * 2.0**-4, np.repeat(step, 32, axis=1))
    assert np.all(err <= rel_bound)
    # quantizing the dequantized data again reproduces the same values (the
    # bytes can differ: an amax rounded down to 224 * 2^e re-scales by 2^(e-1))
    codes2, scales2 = orc.quantize_rowwise(deq)
    assert np.array_equal(orc.dequant_rowwise(codes2, scales2), deq)


def test_colwise_equals_rowwise_of_transpose_when_aligned():
    rng = np.random.default_rng(2)
    m = [64, 0, 32, 96]
    src = orc.bf16_to_f64(orc.f64_to_bf16_rne(rng.standard_normal((sum(m), 64))))
    cc, cs = orc.quantize_colwise(src, m)
    o = orc.offsets(m)
    base = orc.colwise_scale_rows(m)
    for g in range(len(m)):
        a, b = int(o[g]), int(o[g + 1])
        if a == b:
            continue
        rc, rs = orc.quantize_rowwise(src[a:b].T)
        assert np.array_equal(cc[a:b], rc.T)
        assert np.array_equal(cs[int(base[g]):int(base[g + 1])], rs.T)


def test_colwise_partial_block_and_scale_base():
    rng = np.random.default_rng(3)
    m = [5, 40, 0, 33]
    src = orc.bf16_to_f64(orc.f64_to_bf16_rne(rng.standard_normal((sum(m), 32))))
    base = orc.colwise_scale_rows(m)
    assert base.tolist() == [0, 1, 3, 3, 5]
    cc, cs = orc.quantize_colwise(src, m)
    # group 0 (5 rows) is a single partial block: amax over its 5 rows only
    c0, s0 = orc.quantize_block(src[0:5, 7])
    assert int(cs[0, 7]) == int(s0) and np.array_equal(cc[0:5, 7], c0)
    # group 3's second block holds exactly its last row
    r = 45 + 32
    c1, s1 = orc.quantize_block(src[r:r + 1, 3])
    assert int(cs[4, 3]) == int(s1) and cc[r, 3] == c1[0]
    # half an E4M3 step: 2^-4 relative, or the block's subnormal half-step
    # (block amax < 8 here, so scale <= 2^-5 and that half-step <= 2^-15)
    assert np.all(np.abs(orc.dequant_colwise(cc, cs, m) - src) <= np.abs(src) * 2.0**-4 + 2.0**-15)


def test_uniform_members_scale_base():
    """G equal members: member i's scale rows start at i * ceil(rows_i/32)
    (the scale-base fix described in TransformerEngine PR #3224)."""
    for rows_i in (32, 64, 100, 128):
        m = [rows_i] * 5
        base = orc.colwise_scale_rows(m)
        assert base.tolist() == [i * ((rows_i + 31) // 32) for i in range(6)]


def test_mxfp8_products_on_integer_codes():
    """With scale byte 127 and small-integer codes the dequantized products are
    exact integer matrix products."""
    rng = np.random.default_rng(4)
    G, N, K, m = 2, 32, 64, [32, 64]
    M = sum(m)
    ints = np.array([0, 1, 2, 3, -1, -2, -3])
    def enc(a):
        return orc.e4m3_encode(a.astype(np.float64))
    xi = rng.choice(ints, (M, K)); wi = rng.choice(ints, (G, N, K)); dyi = rng.choice(ints, (M, N))
    ones_r = lambda r, c: np.full((r, c // 32), 127, np.uint8)
    y = orc.fwd_mxfp8(enc(xi), ones_r(M, K), enc(wi), ones_r(G * N, K).reshape(G, N, K // 32), None, m)
    o = orc.offsets(m)
    for g in range(G):
        a, b = int(o[g]), int(o[g + 1])
        assert np.array_equal(y[a:b], (xi[a:b] @ wi[g].T).astype(np.float64))
    # dgrad: W columnwise, blocks along N inside every group -> scale rows G*N/32
    wcs = np.full((G * N // 32, K), 127, np.uint8)
    dx = orc.dgrad_mxfp8(enc(dyi), ones_r(M, N), enc(wi), wcs, m)
    for g in range(G):
        a, b = int(o[g]), int(o[g + 1])
        assert np.array_equal(dx[a:b], (dyi[a:b] @ wi[g]).astype(np.float64))
    # wgrad: x and dy columnwise (blocks along each group's rows)
    ncs = int(orc.colwise_scale_rows(m)[-1])
    dw = orc.wgrad_mxfp8(enc(xi), np.full((ncs, K), 127, np.uint8), enc(dyi),
                         np.full((ncs, N), 127, np.uint8), m, None, False)
    for g in range(G):
        a, b = int(o[g]), int(o[g + 1])
        assert np.array_equal(dw[g], (dyi[a:b].T @ xi[a:b]).astype(np.float64))


def test_planted_scale_mistake_is_caught():
    """Using floor(log2 amax) - 8 (the other common scale rule) instead of the
    chosen one changes the hand-worked blocks."""
    with open(os.path.join(GOLDEN, "mxfp8_blocks.json")) as f:
        data = json.load(f)
    diffs = 0
    for case in data["cases"]:
        a = max(abs(v) for v in case["block"])
        if a == 0:
            continue
        e_other = int(np.floor(np.log2(a))) - 8
        diffs += e_other + 127 != case["scale"]
    assert diffs > 0


def test_mma_rowwise_offsets_hand_worked():
    """Positions worked by hand from the tcgen05 scale-factor layout (rows i,
    i+32, i+64, i+96 of an atom share a 16-byte line, one byte per block;
    atoms k-group-major): rows=300 (R = 3 row atoms), cols=256 (2 k-groups)."""
    off = orc.mma_offsets_rowwise(300, 256)
    assert off.shape == (300, 8)
    assert off[0, 0] == 0
    assert off[1, 0] == 16
    assert off[32, 0] == 4
    assert off[33, 2] == 16 + 4 + 2
    assert off[127, 3] == 31 * 16 + 3 * 4 + 3
    assert off[128, 0] == 512            # second row atom of k-group 0
    assert off[0, 4] == 3 * 512          # k-group 1 starts after R = 3 atoms
    assert off[299, 7] == 5 * 512 + 11 * 16 + 1 * 4 + 3   # row 299 = atom 2, i = 43


def test_mma_colwise_offsets_hand_worked():
    """Groups [100, 0, 300] x 128 columns: k-group bases T = [0, 1, 1]."""
    off = orc.mma_offsets_colwise([100, 0, 300], 128)
    base = orc.colwise_scale_rows([100, 0, 300])
    assert off.shape == (int(base[-1]), 128)
    assert off[base[0] + 3, 5] == 5 * 16 + 0 * 4 + 3          # group 0, block 3 (rows 96..99)
    assert off[base[2] + 0, 0] == 512                          # group 2 starts k-group 1
    assert off[base[2] + 9, 127] == 3 * 512 + 31 * 16 + 3 * 4 + 1  # block 9 -> k-group 1 + 2, j = 1
    assert off[base[2] + 4, 64] == 2 * 512 + 0 * 16 + 2 * 4 + 0


@pytest.mark.parametrize("rows,cols", [(1, 128), (130, 256), (300, 384)])
def test_mma_rowwise_offsets_injective_in_bounds(rows, cols):
    off = orc.mma_offsets_rowwise(rows, cols)
    bound = ((rows + 127) // 128) * (cols // 128) * 512
    assert len(np.unique(off)) == off.size
    assert off.min() >= 0 and off.max() < bound


@pytest.mark.parametrize("m", [[1], [100, 0, 300], [128, 129, 127, 33], [0, 0, 5]])
def test_mma_colwise_offsets_injective_in_bounds(m):
    cols = 256
    off = orc.mma_offsets_colwise(m, cols)
    rows, G = sum(m), len(m)
    bound = ((rows + 127) // 128 + G) * (cols // 128) * 512
    assert len(np.unique(off)) == off.size
    assert off.min() >= 0 and off.max() < bound
    # one group alone lands in the rowwise layout of its transpose
    if len(m) == 1:
        t = orc.mma_offsets_rowwise(cols, ((m[0] + 127) // 128) * 128)
        nblk = (m[0] + 31) // 32
        assert np.array_equal(off, t[:, :nblk].T)
