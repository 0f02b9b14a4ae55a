"""Pins for the CPU oracle: checks against values and properties that the pages
and the mathematics fix, none of which re-types the oracle's own formulas.

  * hand-worked examples with dyadic values (tests/golden/*.txt)
  * the page's 8-bit scale example ("大模型量化实战" section 2.2)
  * invariants: code range, |x - dequant| <= s/2, group ends within s/2
  * constant groups, one-signed groups, the all-zero group
  * optimality brute force: each code is a nearest grid point, ties to even
  * exact rational arithmetic for the fp32 steps (independent rounding code)
  * packing: hand-derived positions, bijection, canonical word examples
  * element decoding against numpy / torch conversions
  * the linear layer against a closed form and an exactly-rounded sum
  * its input gradient against a closed form, the adjoint identity with the
    forward product, and one-hot rows of the dequantized matrix
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def read_golden(name):
    d = {}
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            d[key] = vals
    return d


# --------------------------------------------------------------------------
# independent exact arithmetic (Fractions) for IEEE binary32 round-to-nearest
# --------------------------------------------------------------------------

def rne_int(q: Fraction) -> int:
    n = math.floor(q)
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n


def rne_f32(q: Fraction) -> Fraction:
    """Round a rational to the nearest binary32 value (ties to even), exactly."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    qe = max(e - 23, -149)
    n = rne_int(a / Fraction(2) ** qe)
    return sign * Fraction(n) * Fraction(2) ** qe


def exact_group(x32: np.ndarray, bits: int):
    """The quantizer's steps (reading R1-R3) in exact rational arithmetic."""
    qmax = (1 << bits) - 1
    xs = [Fraction(float(v)) for v in x32]
    lo = min(min(xs), Fraction(0))
    hi = max(max(xs), Fraction(0))
    s = rne_f32(rne_f32(hi - lo) / qmax)
    if s == 0:
        return 0.0, 0, [0] * len(xs)
    z = rne_int(rne_f32(-lo / s))
    q = [min(max(rne_int(rne_f32(v / s)) + z, 0), qmax) for v in xs]
    return float(s), z, q


# --------------------------------------------------------------------------
# worked examples
# --------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["int4_g8_worked.txt", "int2_g8_worked.txt", "int4_clamp_worked.txt",
                                  "int4_zero_tie_worked.txt"])
def test_worked_examples(name):
    g = read_golden(name)
    bits = int(g["bits"][0])
    x = np.array([float(v) for v in g["x"]], dtype=np.float32)
    s, z, q = O.quantize_group(x, bits)
    assert s == float(g["s"][0])
    assert z == int(g["z"][0])
    assert q.tolist() == [int(v) for v in g["q"]]
    deq = (q.astype(np.float64) - z) * s
    assert deq.tolist() == [float(v) for v in g["dequant"]]
    # the oracle's own dequantization functions reproduce the hand-worked values
    c1, s1, z1 = q.reshape(1, -1).astype(np.uint8), np.array([[s]], np.float32), np.array([[z]], np.uint8)
    assert O.dequant_f32(c1, s1, z1, x.size)[0].tolist() == [float(v) for v in g["dequant"]]
    assert O.dequant_f64(c1, s1, z1, x.size)[0].tolist() == [float(v) for v in g["dequant"]]
    for key in ("canonical_word32", "canonical_word16"):
        if key in g:
            packed = O.pack(q.reshape(1, -1), bits, "canonical")
            assert int.from_bytes(packed.tobytes(), "little") == int(g[key][0], 16)


def _f16_bits(vals) -> np.ndarray:
    return np.array(vals, dtype=np.float16).view(np.uint16)


def test_dequant_two_rows_two_groups():
    """Hand-worked matrix with a different scale per (row, group): the
    oracle's quantizer gives the hand-worked codes, scales and zeros, and both
    dequantization functions return (q - z) * s of the right row and group."""
    g = read_golden("int4_2x2_groups_worked.txt")
    bits, group = int(g["bits"][0]), int(g["group"][0])
    x = np.stack([np.array([float(v) for v in g[f"x{r}"]]) for r in (0, 1)])
    codes, scales, zeros = O.quantize(_f16_bits(x), "f16", bits, group)
    assert codes.tolist() == [[int(v) for v in g[f"q{r}"]] for r in (0, 1)]
    assert scales.reshape(-1).tolist() == [float(v) for v in g["scales"]]
    assert zeros.reshape(-1).tolist() == [int(v) for v in g["zeros"]]
    want = [[float(v) for v in g[f"dequant{r}"]] for r in (0, 1)]
    assert O.dequant_f32(codes, scales, zeros, group).tolist() == want
    assert O.dequant_f64(codes, scales, zeros, group).tolist() == want


def test_mixed_dequant_and_linear_tiled():
    """Mixed widths through the oracle's block-by-block path: a 4-bit block
    (group 128) whose rows repeat the 8-element 4-bit worked example and a
    2-bit block (group 64) whose rows repeat the 2-bit one.  Repeating a
    group's vector keeps its min and max, so every group has the worked
    example's scale, zero point and codes; the dequantized matrix is the
    worked dequantization repeated, and a one-hot x selects its columns."""
    g4, g2 = read_golden("int4_g8_worked.txt"), read_golden("int2_g8_worked.txt")
    K = 128
    rows4 = np.tile(np.array([float(v) for v in g4["x"]]), K // 8)
    rows2 = np.tile(np.array([float(v) for v in g2["x"]]), K // 8)
    W = np.concatenate([np.tile(rows4, (128, 1)), np.tile(rows2, (128, 1))])
    bit_map = [4, 2]
    _, _, _, blocks = O.quantize_mixed(_f16_bits(W), "f16", bit_map, "interleaved")
    want = np.concatenate([np.tile(np.array([float(v) for v in g4["dequant"]]), (128, K // 8)),
                           np.tile(np.array([float(v) for v in g2["dequant"]]), (128, K // 8))])
    got = np.concatenate([O.dequant_f32(c, s, z, O.GROUP_OF_BITS[b]) for (c, s, z), b in zip(blocks, bit_map)])
    assert (got == want).all()
    for (c, s, z), b in zip(blocks, bit_map):
        assert (s == float((g4 if b == 4 else g2)["s"][0])).all()
        assert (z == int((g4 if b == 4 else g2)["z"][0])).all()
    for k in (0, 5, 7, 64, 127):
        x = np.zeros((1, K))
        x[0, k] = 1.0
        y = O.linear_mixed_f64(x, blocks, bit_map)
        assert (y[0] == want[:, k]).all()


def test_page_scale_example():
    g = read_golden("page_scale_example.txt")
    x = np.array([float(v) for v in g["x"]], dtype=np.float32)
    s, z, q = O.quantize_group(x, int(g["bits"][0]))
    assert abs(s - float(g["s_approx"][0])) < float(g["s_abs_tol"][0])
    assert z == int(g["z"][0])
    assert q.tolist() == [int(v) for v in g["q"]]


# --------------------------------------------------------------------------
# invariants and special groups
# --------------------------------------------------------------------------

def _random_groups(rng, count, g):
    kinds = []
    for i in range(count):
        k = i % 7
        if k == 0:
            v = rng.normal(0, 0.02, g)
        elif k == 1:
            v = rng.standard_t(4, g) * 0.01
        elif k == 2:
            v = np.abs(rng.normal(0, 1, g)) + 0.1          # one-signed positive
        elif k == 3:
            v = -np.abs(rng.normal(0, 1, g)) - 0.1         # one-signed negative
        elif k == 4:
            v = rng.integers(-8, 9, g) * 0.125             # dyadic grid: many ties
        elif k == 5:
            v = rng.normal(0, 1, g)
            v[rng.integers(0, g)] *= 50.0                  # one outlier
        else:
            v = rng.uniform(-3, 7, g)
        kinds.append(v.astype(np.float16).astype(np.float32))
    return kinds


@pytest.mark.parametrize("bits,g", [(4, 128), (2, 64), (4, 32), (2, 8)])
def test_invariants(bits, g):
    rng = np.random.default_rng(1000 + bits * 7 + g)
    qmax = (1 << bits) - 1
    for x in _random_groups(rng, 300, g):
        s, z, q = O.quantize_group(x, bits)
        assert 0 <= z <= qmax
        assert q.min() >= 0 and q.max() <= qmax
        deq = (q.astype(np.float64) - z) * s
        err = np.abs(deq - x.astype(np.float64))
        bound = s / 2 + s * 2.0 ** -18
        assert err.max() <= bound, (err.max(), s)
        # the two ends of the (zero-widened) range reconstruct within s/2
        i_lo, i_hi = int(np.argmin(x)), int(np.argmax(x))
        assert err[i_lo] <= bound and err[i_hi] <= bound


def test_constant_groups():
    # all zero: the guarded case, s = 0
    s, z, q = O.quantize_group(np.zeros(64, np.float32), 2)
    assert (s, z) == (0.0, 0) and not q.any()
    s, z, q = O.quantize_group(-np.zeros(16, np.float32), 4)
    assert (s, z) == (0.0, 0) and not q.any()
    # constant c != 0 reconstructs c within fp32 rounding
    for c in (0.75, -0.75, 3.0e-3, -1.0e4):
        for bits in (2, 4):
            qmax = (1 << bits) - 1
            s, z, q = O.quantize_group(np.full(32, c, np.float32), bits)
            assert s > 0
            deq = (int(q[0]) - z) * s
            assert abs(deq - c) <= abs(c) * 2.0 ** -20
            assert len(set(q.tolist())) == 1
            if c > 0:
                assert z == 0 and q[0] == qmax
            else:
                assert z == qmax and q[0] == 0


def test_nonfinite_rejected():
    for bad in (np.inf, -np.inf, np.nan):
        x = np.zeros(8, np.float32)
        x[3] = bad
        with pytest.raises(O.OracleError):
            O.quantize_group(x, 4)


# --------------------------------------------------------------------------
# brute force
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 4])
def test_brute_force_optimal_codes(bits):
    """Every code is a nearest point of the grid {(q - z) s}, ties to an even
    (q - z), except where the quotient sits within fp32 rounding of a tie."""
    qmax = (1 << bits) - 1
    vals = [Fraction(k, 8) for k in range(-12, 13)]
    rng = np.random.default_rng(7 + bits)
    for g in (2, 3, 4):
        for _ in range(400):
            xs = [vals[i] for i in rng.integers(0, len(vals), g)]
            x32 = np.array([float(v) for v in xs], np.float32)
            s, z, q = O.quantize_group(x32, bits)
            if s == 0:
                assert all(v == 0 for v in xs) and not q.any()
                continue
            S = Fraction(s)
            for xi, qi in zip(xs, q.tolist()):
                d = [abs((c - z) * S - xi) for c in range(qmax + 1)]
                best = min(d)
                cand = [c for c in range(qmax + 1) if d[c] == best]
                t = xi / S
                near_tie = abs((t - math.floor(t)) - Fraction(1, 2)) < Fraction(1, 2 ** 18)
                if near_tie and len(cand) == 1:
                    assert abs(qi - cand[0]) <= 1
                    continue
                assert qi in cand, (xs, s, z, q)
                if len(cand) == 2:
                    assert (qi - z) % 2 == 0


def test_exact_rational_arithmetic():
    """The fp32 steps agree with exact rational arithmetic followed by
    round-to-nearest-even, including constructed near-tie quotients."""
    rng = np.random.default_rng(99)
    groups = _random_groups(rng, 140, 16)
    # near ties: x = fp32 nearest to (k + 1/2) s, plus its neighbours
    for _ in range(200):
        bits = 4
        base = rng.normal(0, 1, 16).astype(np.float32)
        s_guess = np.float32((base.max() - min(base.min(), 0)) / 15)
        k = int(rng.integers(-7, 8))
        t = np.float32((k + 0.5) * float(s_guess))
        nb = np.nextafter(t, np.float32(np.inf)), np.nextafter(t, np.float32(-np.inf))
        base[3], base[5], base[7] = t, nb[0], nb[1]
        groups.append(base.astype(np.float32))
    for i, x in enumerate(groups):
        for bits in (2, 4):
            s, z, q = O.quantize_group(x, bits)
            es, ez, eq = exact_group(x, bits)
            assert (s, z, q.tolist()) == (es, ez, eq), (i, bits)


# --------------------------------------------------------------------------
# matrix-level quantize (row/group indexing, fp16 and bf16 inputs)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("wtype", ["f16", "bf16"])
def test_matrix_quantize_matches_groups(wtype):
    rng = np.random.default_rng(5)
    N, K, g = 6, 256, 64
    w = torch.from_numpy(rng.normal(0, 0.02, (N, K)).astype(np.float32)).to(
        torch.float16 if wtype == "f16" else torch.bfloat16)
    bits16 = w.view(torch.int16).numpy().view(np.uint16)
    codes, scales, zeros = O.quantize(bits16, wtype, 2, g, threads=3)
    wf = w.float().numpy()
    for n in range(N):
        for j in range(K // g):
            s, z, q = O.quantize_group(wf[n, j * g:(j + 1) * g], 2)
            assert scales[n, j] == np.float32(s) and zeros[n, j] == z
            assert (codes[n, j * g:(j + 1) * g] == q).all()


# --------------------------------------------------------------------------
# element decoding and bf16 rounding
# --------------------------------------------------------------------------

def test_decode_f16_all_patterns():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = O.decode_f64(pats, "f16")
    ref = pats.view(np.float16).astype(np.float64)
    both_nan = np.isnan(mine) & np.isnan(ref)
    assert ((mine == ref) | both_nan).all()
    assert (np.signbit(mine) == np.signbit(ref))[~both_nan].all()


def test_decode_bf16_all_patterns():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = O.decode_f64(pats, "bf16")
    ref = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).double().numpy()
    both_nan = np.isnan(mine) & np.isnan(ref)
    assert ((mine == ref) | both_nan).all()


def test_bf16_rounding():
    rng = np.random.default_rng(3)
    v = rng.normal(0, 10, 4000).astype(np.float32).astype(np.float64)
    mine = O.to_bf16_bits(v)
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (mine == ref).all()
    # direct rounding of doubles: an exact tie goes to even, just above goes up
    assert O.to_bf16_bits(np.array([1 + 2 ** -8]))[0] == 0x3F80
    assert O.to_bf16_bits(np.array([1 + 2 ** -8 + 2 ** -40]))[0] == 0x3F81
    assert O.to_bf16_bits(np.array([1 + 3 * 2 ** -8]))[0] == 0x3F82
    assert O.to_bf16_bits(np.array([-2.0]))[0] == 0xC000


# --------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------

def test_interleaved_positions_hand_derived():
    with open(os.path.join(GOLD, "interleaved_positions.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) >= 20
    for bits, nrows, cols, n, k, byte, bit in (map(int, r) for r in rows):
        assert O.code_position("interleaved", n, k, nrows, cols, bits) == (byte, bit), (bits, nrows, cols, n, k)


def test_meta_positions_hand_derived():
    with open(os.path.join(GOLD, "meta_positions.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) >= 11
    for layout, n, g, nrows, G, idx in rows:
        assert O.meta_index(layout, int(n), int(g), int(nrows), int(G)) == int(idx), (layout, n, g, nrows, G)


@pytest.mark.parametrize("layout", ["canonical", "interleaved"])
def test_meta_layout_bijection(layout):
    rows, G = 144, 24
    seen = {O.meta_index(layout, n, g, rows, G) for n in range(rows) for g in range(G)}
    assert seen == set(range(rows * G))
    rng = np.random.default_rng(1)
    sc = rng.normal(size=(rows, G)).astype(np.float32)
    ze = rng.integers(0, 16, (rows, G)).astype(np.uint8)
    ps, pz = O.pack_meta(sc, ze, layout)
    for n in range(rows):
        for g in range(G):
            i = O.meta_index(layout, n, g, rows, G)
            assert ps[i] == sc[n, g] and pz[i] == ze[n, g]


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("layout", ["canonical", "interleaved"])
def test_pack_bijection(bits, layout):
    N, K = 144, 256
    rng = np.random.default_rng(bits)
    seen = set()
    for n in range(N):
        for k in range(K):
            seen.add(O.code_position(layout, n, k, N, K, bits))
    assert len(seen) == N * K
    assert all(0 <= b < N * K * bits // 8 and o % bits == 0 and o < 8 for b, o in seen)
    codes = rng.integers(0, 1 << bits, (N, K), dtype=np.uint8)
    p = O.pack(codes, bits, layout)
    assert p.size == N * K * bits // 8
    assert (O.unpack(p, N, K, bits, layout) == codes).all()


def test_canonical_is_row_major_lsb_first():
    codes = np.array([[1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 0]], np.uint8)
    p = O.pack(codes, 4, "canonical")
    assert p.tobytes() == bytes([0x21, 0x43, 0x65, 0x87, 0xA9, 0xCB, 0xED, 0x0F])
    c2 = np.array([[3, 0, 1, 2] * 4], np.uint8)
    assert O.pack(c2, 2, "canonical").tobytes() == bytes([0b10010011] * 4)


def test_storage_sizes_match_page():
    # "低比特量化": a 70B-parameter model takes 35 GB at INT4 and 17.5 GB at INT2
    # (codes only, 1 GB = 1e9 bytes)
    for bits, gb in ((4, 35.0), (2, 17.5)):
        assert 70e9 * bits / 8 / 1e9 == gb


# --------------------------------------------------------------------------
# linear
# --------------------------------------------------------------------------

def _representable_matrix(rng, N, K, g, bits):
    """W whose groups are reproduced exactly by the quantizer: per group a
    power-of-two scale, a zero point, and codes that include both 0 and
    2^b - 1 so the range is exactly (2^b - 1) s."""
    qmax = (1 << bits) - 1
    G = K // g
    codes = rng.integers(0, qmax + 1, (N, K)).astype(np.uint8)
    for n in range(N):
        for j in range(G):
            i0, i1 = rng.choice(g, 2, replace=False)
            codes[n, j * g + i0] = 0
            codes[n, j * g + i1] = qmax
    zeros = rng.integers(0, qmax + 1, (N, G)).astype(np.uint8)
    scales = np.float32(2.0) ** rng.integers(-9, -4, (N, G)).astype(np.float32)
    W = np.empty((N, K), np.float64)
    for n in range(N):
        for j in range(G):
            W[n, j * g:(j + 1) * g] = (codes[n, j * g:(j + 1) * g].astype(np.float64) - zeros[n, j]) * scales[n, j]
    return W, codes, scales, zeros


@pytest.mark.parametrize("bits,g", [(4, 128), (2, 64)])
def test_linear_closed_form(bits, g):
    rng = np.random.default_rng(11 * bits)
    N, K, M = 24, 512, 5
    W, codes, scales, zeros = _representable_matrix(rng, N, K, g, bits)
    w16 = W.astype(np.float16)
    assert (w16.astype(np.float64) == W).all()
    c2, s2, z2 = O.quantize(w16.view(np.uint16), "f16", bits, g)
    assert (c2 == codes).all() and (s2 == scales).all() and (z2 == zeros).all()
    assert (O.dequant_f64(c2, s2, z2, g) == W).all()
    x = rng.normal(0, 1, (M, K)).astype(np.float16).astype(np.float64)
    y = O.linear_f64(x, c2, s2, z2, g, threads=2)
    ref = x @ W.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_linear_exact_sum():
    rng = np.random.default_rng(2)
    N, K, M, g = 4, 64, 3, 32
    w = rng.normal(0, 0.02, (N, K)).astype(np.float16)
    codes, scales, zeros = O.quantize(w.view(np.uint16), "f16", 4, g)
    x = rng.normal(0, 1, (M, K)).astype(np.float16).astype(np.float64)
    y = O.linear_f64(x, codes, scales, zeros, g)
    for m in range(M):
        for n in range(N):
            terms = [x[m, k] * ((int(codes[n, k]) - int(zeros[n, k // g])) * float(scales[n, k // g]))
                     for k in range(K)]
            exact = math.fsum(terms)
            assert abs(y[m, n] - exact) <= 1e-13 * math.fsum(abs(t) for t in terms) + 1e-300


@pytest.mark.parametrize("bits,g", [(4, 128), (2, 64)])
def test_grad_input_closed_form(bits, g):
    """dx = dy . W for a matrix the quantizer reproduces exactly, against
    numpy's matmul."""
    rng = np.random.default_rng(13 * bits)
    N, K, M = 40, 256, 3
    W, codes, scales, zeros = _representable_matrix(rng, N, K, g, bits)
    c2, s2, z2 = O.quantize(W.astype(np.float16).view(np.uint16), "f16", bits, g)
    assert (c2 == codes).all() and (s2 == scales).all() and (z2 == zeros).all()
    dy = rng.normal(0, 1, (M, N)).astype(np.float16).astype(np.float64)
    dx = O.linear_grad_input_f64(dy, c2, s2, z2, g, threads=2)
    assert dx.shape == (M, K)
    assert np.allclose(dx, dy @ W, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("bits,g", [(4, 32), (2, 64)])
def test_grad_input_adjoint(bits, g):
    """<dy, x . dequant(W)^T> = <dy . dequant(W), x>: the input gradient is the
    adjoint of the forward product (pinned on its own above), here for
    generic quantized weights."""
    rng = np.random.default_rng(5 + bits)
    N, K, M = 48, 256, 4
    w = rng.normal(0, 0.02, (N, K)).astype(np.float16)
    codes, scales, zeros = O.quantize(w.view(np.uint16), "f16", bits, g)
    x = rng.normal(0, 1, (M, K))
    dy = rng.normal(0, 1, (M, N))
    y = O.linear_f64(x, codes, scales, zeros, g)
    dx = O.linear_grad_input_f64(dy, codes, scales, zeros, g)
    lhs = math.fsum((dy * y).ravel())
    rhs = math.fsum((dx * x).ravel())
    Wd = np.abs(O.dequant_f64(codes, scales, zeros, g))
    bound = 1e-12 * float(np.sum(np.abs(dy) * (np.abs(x) @ Wd.T)))
    assert abs(lhs - rhs) <= bound


def test_grad_input_one_hot_rows():
    """dy = one-hot (token m, channel n) gives dx[m] = row n of dequant(W) and
    zero for every other token."""
    rng = np.random.default_rng(17)
    N, K, g = 20, 128, 32
    w = rng.normal(0, 0.02, (N, K)).astype(np.float16)
    codes, scales, zeros = O.quantize(w.view(np.uint16), "f16", 4, g)
    Wd = O.dequant_f64(codes, scales, zeros, g)
    for m, n in [(0, 0), (1, 7), (2, N - 1)]:
        dy = np.zeros((3, N))
        dy[m, n] = 1.0
        dx = O.linear_grad_input_f64(dy, codes, scales, zeros, g)
        assert (dx[m] == Wd[n]).all()
        assert (np.delete(dx, m, axis=0) == 0).all()


def test_mixed_offsets_hand_computed():
    code_off, group_off = O.mixed_offsets([4, 2, 4], 256)
    assert code_off == [0, 16384, 24576, 40960]
    assert group_off == [0, 256, 768, 1024]


@pytest.mark.parametrize("bits", [4, 2])
def test_interleaved_stacks_whole_blocks(bits):
    """Interleaved layout is 128-row-block major: stacking matrices of whole
    blocks along N concatenates their packed codes and their metadata, which
    is what running q/k/v (or gate/up) as one linear relies on."""
    rng = np.random.default_rng(bits)
    K = 256 if bits == 4 else 512
    G = K // (128 if bits == 4 else 64)
    parts = [rng.integers(0, 1 << bits, size=(n, K), dtype=np.uint8) for n in (256, 128, 128)]
    whole = np.concatenate(parts)
    assert (O.pack(whole, bits, "interleaved") ==
            np.concatenate([O.pack(p, bits, "interleaved") for p in parts])).all()
    scales = [rng.standard_normal((p.shape[0], G)).astype(np.float32) for p in parts]
    zeros = [rng.integers(0, 1 << bits, size=(p.shape[0], G), dtype=np.uint8) for p in parts]
    ms, mz = O.pack_meta(np.concatenate(scales), np.concatenate(zeros), "interleaved")
    pieces = [O.pack_meta(s, z, "interleaved") for s, z in zip(scales, zeros)]
    assert (ms.view(np.uint32) == np.concatenate([p[0] for p in pieces]).view(np.uint32)).all()
    assert (mz == np.concatenate([p[1] for p in pieces])).all()


# --------------------------------------------------------------------------
# symmetric abs-max scheme ("大模型量化实战", section 2.3)
# --------------------------------------------------------------------------

def exact_group_sym(x32: np.ndarray, bits: int):
    """The symmetric scheme's steps in exact rational arithmetic."""
    qmax, zc = (1 << bits) - 1, 1 << (bits - 1)
    xs = [Fraction(float(v)) for v in x32]
    amax = max(abs(v) for v in xs)
    s = rne_f32(amax / (zc - 1))
    if s == 0:
        return 0.0, zc, [zc] * len(xs)
    q = [min(max(rne_int(rne_f32(v / s)) + zc, 0), qmax) for v in xs]
    return float(s), zc, q


@pytest.mark.parametrize("name", ["sym_int4_g8_worked.txt", "sym_int2_g8_worked.txt"])
def test_sym_worked_examples(name):
    g = read_golden(name)
    bits = int(g["bits"][0])
    x = np.array([float(v) for v in g["x"]], dtype=np.float32)
    s, z, q = O.quantize_group(x, bits, scheme="symmetric")
    assert s == float(g["s"][0])
    assert z == int(g["z"][0])
    assert q.tolist() == [int(v) for v in g["q"]]
    assert ((q.astype(np.float64) - z) * s).tolist() == [float(v) for v in g["dequant"]]
    for key in ("canonical_word32", "canonical_word16"):
        if key in g:
            packed = O.pack(q.reshape(1, -1), bits, "canonical")
            assert int.from_bytes(packed.tobytes(), "little") == int(g[key][0], 16)


def test_sym_page_scale_example():
    """The page's 8-bit example: x_absmax = 5.0 gives s = 5.0 / 127 ~ 0.039."""
    x = np.array([-5.0, -0.1, 0.0, 0.05, 0.1, 1.0, 2.5, 4.0], dtype=np.float32)
    s, z, q = O.quantize_group(x, 8, scheme="symmetric")
    assert s == float(np.float32(5.0) / np.float32(127.0))
    assert abs(s - 0.039) < 5e-4
    assert z == 128 and int(q[0]) == 1 and int(q[2]) == 128


@pytest.mark.parametrize("bits", [2, 4])
def test_sym_invariants(bits):
    rng = np.random.default_rng(7 + bits)
    for trial in range(300):
        x = (rng.standard_normal(32) * rng.choice([1e-3, 0.02, 1.0, 30.0])).astype(np.float32)
        s, z, q = O.quantize_group(x, bits, scheme="symmetric")
        assert z == 1 << (bits - 1)
        assert q.min() >= 1 and q.max() <= (1 << bits) - 1       # the code 0 is never needed
        err = np.abs(x.astype(np.float64) - (q.astype(np.float64) - z) * s)
        assert err.max() <= s / 2 * (1 + 2.0 ** -20)
        # round half to even is odd-symmetric: negating the group negates q - z
        s2, z2, q2 = O.quantize_group(-x, bits, scheme="symmetric")
        assert s2 == s and ((q2.astype(int) - z2) == -(q.astype(int) - z)).all()


def test_sym_exact_rational_arithmetic():
    rng = np.random.default_rng(11)
    for bits in (2, 4, 8):
        for _ in range(200):
            x = (rng.standard_normal(16) * 0.02).astype(np.float16).astype(np.float32)
            s, z, q = O.quantize_group(x, bits, scheme="symmetric")
            es, ez, eq = exact_group_sym(x, bits)
            assert s == es and z == ez and q.tolist() == eq


def test_sym_all_zero_group():
    s, z, q = O.quantize_group(np.zeros(64, dtype=np.float32), 4, scheme="symmetric")
    assert s == 0.0 and z == 8 and (q == 8).all()


def test_sym_matrix_matches_groups():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((4, 256)) * 0.02).astype(np.float16)
    codes, scales, zeros = O.quantize(W.view(np.uint16), "f16", 4, 64, scheme="symmetric")
    for n in range(4):
        for j in range(4):
            s, z, q = O.quantize_group(W[n, 64 * j:64 * (j + 1)].astype(np.float32), 4, scheme="symmetric")
            assert scales[n, j] == s and zeros[n, j] == z and (codes[n, 64 * j:64 * (j + 1)] == q).all()


# --------------------------------------------------------------------------
# binary16 group scales (the fp16-scale format variant)
# --------------------------------------------------------------------------

def test_f16_scale_worked_example():
    g = read_golden("int4_f16scale_worked.txt")
    x = np.array([float(v) for v in g["x"]], dtype=np.float32)
    s, z, q = O.quantize_group(x, int(g["bits"][0]), "asymmetric_f16_scale")
    assert s == float(g["s"][0])
    assert int(O.f32_to_f16_bits(np.float32(s))) == int(g["s_f16_bits"][0], 16)
    assert z == int(g["z"][0])
    assert q.tolist() == [int(v) for v in g["q"]]


def test_f32_to_f16_matches_library_rounding():
    """The oracle's binary16 rounding against numpy's (IEEE round to nearest,
    ties to even): every binary16 value and its neighbours, the midpoints
    between consecutive binary16 values (ties), the subnormal range, the
    overflow boundary and random magnitudes over the whole range."""
    rng = np.random.default_rng(7)
    h = np.arange(0, 0x7C00, dtype=np.uint16)
    exact = h.view(np.float16).astype(np.float32)
    up = np.nextafter(exact, np.float32(np.inf))
    down = np.nextafter(exact, np.float32(0))
    mids = ((exact[:-1].astype(np.float64) + exact[1:].astype(np.float64)) / 2).astype(np.float32)
    edge = np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 65536.0, 1e10, 2.0 ** -24, 2.0 ** -25,
                     2.0 ** -25 * 1.0001, 2.0 ** -26, 1e-10, 6.1e-5], dtype=np.float32)
    rnd = (rng.uniform(-30, 17, 20000).astype(np.float64))
    rnd = (np.sign(rng.normal(size=rnd.size)) * 2.0 ** rnd).astype(np.float32)
    vals = np.concatenate([exact, up, down[1:], mids, edge, -mids[::97], rnd])
    got = O.f32_to_f16_bits(vals)
    with np.errstate(over="ignore"):  # the overflow cases are intended (-> infinity)
        want = vals.astype(np.float16).view(np.uint16)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (vals[bad[:5]], got[bad[:5]], want[bad[:5]])


def exact_group_f16_scale(x32: np.ndarray, bits: int):
    """R1-R3 in exact rational arithmetic, with the scale rounded to binary16
    by numpy (round to nearest, ties to even) and used for z and the codes."""
    qmax = (1 << bits) - 1
    xs = [Fraction(float(v)) for v in x32]
    lo = min(min(xs), Fraction(0))
    hi = max(max(xs), Fraction(0))
    s32 = rne_f32(rne_f32(hi - lo) / qmax)
    if s32 == 0:
        return 0.0, 0, [0] * len(xs)
    s16 = Fraction(float(np.float16(float(s32))))
    if s16 == 0:
        s16 = Fraction(1, 2 ** 24)
    z = rne_int(rne_f32(-lo / s16))
    q = [min(max(rne_int(rne_f32(v / s16)) + z, 0), qmax) for v in xs]
    return float(s16), z, q


def test_f16_scale_exact_rational_arithmetic():
    rng = np.random.default_rng(123)
    groups = [g.astype(np.float16).astype(np.float32) for g in _random_groups(rng, 120, 16)]
    # tiny groups whose scale falls into (or below) the binary16 subnormals
    for e in (-18, -22, -26, -30):
        groups.append((rng.normal(0, 2.0 ** e, 16)).astype(np.float16).astype(np.float32))
    # near ties of x / s16
    for _ in range(150):
        base = rng.normal(0, 1, 16).astype(np.float16).astype(np.float32)
        s16 = float(np.float16((float(base.max()) - min(float(base.min()), 0.0)) / 15))
        k = int(rng.integers(-7, 8))
        base[4] = np.float32(np.float16((k + 0.5) * s16))
        groups.append(base)
    for i, x in enumerate(groups):
        for bits in (2, 4):
            s, z, q = O.quantize_group(x, bits, "asymmetric_f16_scale")
            es, ez, eq = exact_group_f16_scale(x, bits)
            assert (s, z, q.tolist()) == (es, ez, eq), (i, bits)
