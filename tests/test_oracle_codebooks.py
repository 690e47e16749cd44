"""Pins for the oracle's codebooks (CPU only).

The pages fix only that the code is dynamic: a non-linear code that keeps small and large
magnitudes alike accurate ([BWQ] abstract, "8-bit Optimizers via Block-wise Quantization", as
reproduced on the blog.csdn.net bitsandbytes guide, section 2), and that NF4 is a 4-bit type fitted to normally
distributed weights ("Bitsandbytes" transformers docs, section "Normal Float 4 (NF4)").  The
construction read from them (dynamic tree; NF4 from normal quantiles) is pinned here by
properties that do not restate the oracle's formulas: counts per decade, equal spacing within
a decade, exact end points, symmetry, and scipy's normal distribution for NF4.
"""
from fractions import Fraction
import os

import numpy as np
import pytest
from scipy import special, stats

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _decade_counts(mags, top_decades):
    counts = []
    for E in range(top_decades):
        hi, lo = 10.0 ** (-E), 10.0 ** (-(E + 1))
        counts.append(int(np.sum((mags > lo * (1 + 1e-6)) & (mags <= hi * (1 + 1e-6)))))
    return counts


def test_unsigned_dynamic_structure(oracle_mod):
    c = oracle_mod.code_dynamic_unsigned()
    assert c.shape == (256,) and c.dtype == np.float32
    assert np.all(np.diff(c) > 0), "strictly increasing"
    assert c[0] == 0.0 and c[-1] == 1.0
    assert c[1] == np.float32(1e-7)
    # dynamic tree: one more fraction bit per decade towards 1 -> 2^(7-E) codes in decade E
    assert _decade_counts(c[1:].astype(np.float64), 8) == [128, 64, 32, 16, 8, 4, 2, 1]
    # within a decade the fraction bins are equal: spacing 0.9 * 10^-E / 2^(7-E)
    for E in range(7):
        hi, lo = 10.0 ** (-E), 10.0 ** (-(E + 1))
        sel = c[(c > lo * (1 + 1e-6)) & (c <= hi * (1 + 1e-6))].astype(np.float64)
        gaps = np.diff(sel)
        want = 0.9 * 10.0 ** (-E) / 2 ** (7 - E)
        # each end point carries at most half an ulp of binary32 rounding
        np.testing.assert_allclose(gaps, want, rtol=0, atol=float(np.spacing(np.float32(hi))))
        # the smallest code of the decade sits one bin above 10^-(E+1)
        assert abs(sel[0] - (lo + want)) <= 2e-7 * sel[0]


def test_signed_dynamic_structure(oracle_mod):
    c = oracle_mod.code_dynamic_signed()
    assert c.shape == (256,)
    assert np.all(np.diff(c) > 0)
    assert c[0] == -1.0 and c[-1] == 1.0
    assert np.count_nonzero(c == 0.0) == 1
    zero = int(np.where(c == 0.0)[0][0])
    assert zero == 127
    neg = c[:zero][::-1]
    pos = c[zero + 1:]
    # the extra code just above zero is the next tree level, 1e-7
    assert pos[0] == np.float32(1e-7)
    np.testing.assert_array_equal(-neg, pos[1:])  # symmetric apart from +1e-7
    assert _decade_counts(pos[1:].astype(np.float64), 7) == [64, 32, 16, 8, 4, 2, 1]
    for E in range(6):
        hi, lo = 10.0 ** (-E), 10.0 ** (-(E + 1))
        sel = pos[(pos > lo * (1 + 1e-6)) & (pos <= hi * (1 + 1e-6))].astype(np.float64)
        np.testing.assert_allclose(np.diff(sel), 0.9 * 10.0 ** (-E) / 2 ** (6 - E), rtol=0,
                                   atol=float(np.spacing(np.float32(hi))))


def _exact_float32(fr: Fraction) -> np.float32:
    """Binary32 nearest to a positive rational, ties to even (exact integer arithmetic)."""
    f = np.float32(float(fr))
    best = f
    for cand in (np.nextafter(f, np.float32(0)), f, np.nextafter(f, np.float32(2))):
        d_c, d_b = abs(Fraction(float(cand)) - fr), abs(Fraction(float(best)) - fr)
        if d_c < d_b or (d_c == d_b and (cand.view(np.uint32) & 1) == 0):
            best = cand
    return best


def test_dynamic_codes_correctly_rounded(oracle_mod):
    """Every code is the binary32 nearest to its decade/bin value 10^-E * (bin upper edge)."""
    u = oracle_mod.code_dynamic_unsigned()
    s = oracle_mod.code_dynamic_signed()
    for code, nbits in ((u, 7), (s, 6)):
        pos = code[code > 0]
        want = []
        for E in range(nbits + 1):
            nE = nbits - E
            for k in range(2 ** nE):
                edge = Fraction(1, 10) + Fraction(9, 10) * Fraction(k + 1, 2 ** nE)
                want.append(_exact_float32(edge / 10 ** E))
        if code is s:
            want.append(_exact_float32(Fraction(1, 10 ** 7)))
        np.testing.assert_array_equal(np.sort(np.array(want, np.float32)), pos)


def test_nf4_normal_quantiles(oracle_mod):
    c = oracle_mod.code_nf4().astype(np.float64)
    assert c.shape == (16,)
    assert np.all(np.diff(c) > 0)
    assert c[0] == -1.0 and c[7] == 0.0 and c[15] == 1.0
    delta = 0.5 * (1 / 30 + 1 / 32)
    scale = special.ndtri(1 - delta)
    probs = stats.norm.cdf(c * scale)
    # 7 negative codes at evenly spaced probabilities in [delta, 1/2), 8 positive in (1/2, 1-delta]
    np.testing.assert_allclose(probs[:7], delta + (0.5 - delta) * np.arange(7) / 7, atol=2e-7)
    np.testing.assert_allclose(probs[8:], 0.5 + (0.5 - delta) * np.arange(1, 9) / 8, atol=2e-7)
    # and each value is the binary32 rounding of scipy's quantile ratio
    want = np.concatenate([special.ndtri(delta + (0.5 - delta) * np.arange(7) / 7), [0.0],
                           special.ndtri(0.5 + (0.5 - delta) * np.arange(1, 9) / 8)]) / scale
    np.testing.assert_array_equal(c.astype(np.float32), want.astype(np.float32))


def test_fp4_e2m1_values(oracle_mod):
    """FP4 = E2M1 (page "Quantize 🤗 Transformers models", section "FP4 quantization"; OCP MX v1.0):
    written out by hand, the sixteen values are k/12 for k in {0, 1, 2, 3, 4, 6, 8, 12} with both
    signs, the spare negative zero replaced by 1/24, each rounded once to binary32."""
    c = oracle_mod.code_fp4()
    want = sorted({Fraction(s * k, 12) for s in (-1, 1) for k in (0, 1, 2, 3, 4, 6, 8, 12)} | {Fraction(1, 24)})
    assert len(want) == 16
    np.testing.assert_array_equal(c, np.array([float(w) for w in want]).astype(np.float32))
    assert c[0] == -1.0 and c[-1] == 1.0 and 0.0 in c
    # away from zero the table is symmetric: E2M1 has the same magnitudes for both signs
    np.testing.assert_array_equal(-c[:7][::-1], c[9:])


def test_linear_code(oracle_mod):
    c = oracle_mod.code_linear()
    assert c[0] == -1.0 and c[-1] == 1.0
    np.testing.assert_allclose(np.diff(c.astype(np.float64)), 2 / 255, rtol=0, atol=float(np.spacing(np.float32(1))))


def test_midpoints_exact_for_dynamic_codes(oracle_mod):
    """mid_j is the exact mean of neighbours whenever that mean is a binary32 number."""
    for code in (oracle_mod.code_dynamic_signed(), oracle_mod.code_dynamic_unsigned(), oracle_mod.code_nf4(),
                 oracle_mod.code_fp4()):
        for j in range(len(code) - 1):
            exact = (Fraction(float(code[j])) + Fraction(float(code[j + 1]))) / 2
            mid = oracle_mod.code_mid(code, j)
            assert code[j] < mid < code[j + 1] or code[j] == mid  # inside the gap
            assert abs(Fraction(float(mid)) - exact) <= abs(Fraction(float(np.spacing(np.float32(mid))))) / 2


def _read_hex(path):
    vals = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                vals.append(float.fromhex(line))
    return np.array(vals, np.float32)


@pytest.mark.parametrize("name,fn", [("code_dynamic_signed", "code_dynamic_signed"),
                                     ("code_dynamic_unsigned", "code_dynamic_unsigned"),
                                     ("code_nf4", "code_nf4"), ("code_fp4", "code_fp4"),
                                     ("code_linear", "code_linear")])
def test_golden_codebooks(oracle_mod, name, fn):
    path = os.path.join(GOLDEN, name + ".hex")
    with open(path) as f:
        head = f.read(600)
    assert "source:" in head, "each fixture states its citation"
    np.testing.assert_array_equal(_read_hex(path), getattr(oracle_mod, fn)())
