"""Pins for the oracle's nested (double) quantization of block scales (CPU only).

The page "Bitsandbytes" (transformers docs, Turkish), section "İç içe nicelleştirme", describes
nested quantization as a second quantization of the already quantized weights' constants that
saves about 0.4 bit per parameter.  The oracle follows QLoRA's double quantization: centre the
fp32 scales by their mean, quantize them block-wise to 8 bits in blocks of 256 with the signed
dynamic code, rebuild as code[q] * absmax2 + offset.
"""
from fractions import Fraction

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st


def _round_f32(fr: Fraction) -> np.float32:
    """Nearest binary32 to an exact rational (ties to even), by bracketing."""
    x = np.float32(float(fr))
    best = None
    for c in (np.nextafter(x, np.float32(-np.inf)), x, np.nextafter(x, np.float32(np.inf))):
        d = abs(Fraction(float(c)) - fr)
        key = (d, int(np.float32(c).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return np.float32(best[1])


@pytest.mark.parametrize("nb", [1, 7, 256, 4095, 4096, 4097, 20000])
def test_offset_is_the_correctly_rounded_mean(oracle_mod, nb):
    rng = np.random.default_rng(nb)
    a = (rng.lognormal(-4, 1.5, nb)).astype(np.float32)
    exact = sum((Fraction(float(v)) for v in a), Fraction(0)) / nb
    assert oracle_mod.absmax_mean(a) == _round_f32(exact)
    _, _, off = oracle_mod.nest_absmax(a, oracle_mod.code_dynamic_signed())
    assert off == _round_f32(exact)


def test_equal_scales_rebuild_exactly(oracle_mod):
    code = oracle_mod.code_dynamic_signed()
    a = np.full(1000, 0.0371, np.float32)
    q, a2, off = oracle_mod.nest_absmax(a, code)
    assert off == a[0]
    assert np.all(a2 == 0) and np.all(code[q] == 0)
    np.testing.assert_array_equal(oracle_mod.unnest_absmax(q, a2, off, code), a)


def test_two_scales_map_to_the_ends_of_the_code(oracle_mod):
    """[0, 2s]: mean s, centred -s and +s, block scale s, codes -1 and +1: rebuilt exactly."""
    code = oracle_mod.code_dynamic_signed()
    s = np.float32(2.0 ** -5)
    a = np.array([0.0, 2 * s], np.float32)
    q, a2, off = oracle_mod.nest_absmax(a, code)
    assert off == s and a2[0] == s
    assert code[q[0]] == -1.0 and code[q[1]] == 1.0
    np.testing.assert_array_equal(oracle_mod.unnest_absmax(q, a2, off, code), a)


@pytest.mark.parametrize("nb", [300, 4096 + 513, 70000])
def test_rebuild_error_within_half_the_code_gap(oracle_mod, nb):
    """P7 for the nested scales: |rebuilt - a| <= absmax2 * max gap / 2 plus the two roundings
    of the rebuild (mul, add)."""
    code = oracle_mod.code_dynamic_signed()
    rng = np.random.default_rng(nb + 1)
    a = (rng.lognormal(-5, 1.0, nb)).astype(np.float32)
    q, a2, off = oracle_mod.nest_absmax(a, code)
    assert a2.size == (nb + 255) // 256
    r = oracle_mod.unnest_absmax(q, a2, off, code).astype(np.float64)
    gap = np.max(np.diff(code.astype(np.float64)))
    blk = np.repeat(a2.astype(np.float64), 256)[:nb]
    tol = blk * gap / 2 * (1 + 1e-6) + 2 * np.spacing(np.abs(r).astype(np.float32)).astype(np.float64) \
        + np.spacing(np.float32(abs(off))).astype(np.float64)
    assert np.all(np.abs(r - a) <= tol)
    # every block scale is the largest |a - offset| of its block
    c = a.astype(np.float32) - off
    want = np.array([np.max(np.abs(c[i:i + 256])) for i in range(0, nb, 256)], np.float32)
    np.testing.assert_array_equal(a2, want)


def test_nested_saves_about_0p4_bit_per_parameter():
    """Blocksize 64 keeps one fp32 scale per 64 weights (0.5 bit/param); nested, one byte per
    64 weights plus one fp32 per 64*256 weights and the offset: about 0.373 bit saved, the
    "0,4 bit/parametre" of the page."""
    n, B, B2 = 13_000_000_000, 64, 256
    nb = n // B
    plain = 32 * nb / n
    nested = (8 * nb + 32 * ((nb + B2 - 1) // B2) + 32) / n
    assert abs(plain - 0.5) < 1e-9
    assert 0.35 < plain - nested < 0.4 + 1e-9


def test_dequantize_nested_composes(oracle_mod):
    """Nested dequantize = dequantize with the rebuilt scales (NF4, blocksize 64)."""
    rng = np.random.default_rng(3)
    n, B = 64 * 300 + 17, 64
    x = rng.standard_normal(n).astype(np.float32)
    nf4, code = oracle_mod.code_nf4(), oracle_mod.code_dynamic_signed()
    a, q = oracle_mod.quantize_blockwise(nf4, x, B)
    qa, a2, off = oracle_mod.nest_absmax(a, code)
    y = oracle_mod.dequantize_blockwise_nested(nf4, q, qa, a2, off, code, n, B)
    r = oracle_mod.unnest_absmax(qa, a2, off, code)
    np.testing.assert_array_equal(y, oracle_mod.dequantize_blockwise(nf4, q, r, n, B))
    # and it stays close to the plain dequantization
    y0 = oracle_mod.dequantize_blockwise(nf4, q, a, n, B)
    assert np.max(np.abs(y - y0)) <= np.max(np.abs(r - a)) * 1.0001


@settings(max_examples=80, deadline=None)
@given(nb=st.integers(1, 1500), mu=st.floats(-12, 2), sigma=st.floats(0, 3), seed=st.integers(0, 2**32 - 1))
def test_nested_random_scales(oracle_mod, nb, mu, sigma, seed):
    """Random counts (one block, full and ragged last blocks) and scale spreads: the offset is
    within one binary32 ulp of the exact mean, every second-level scale is its block's largest
    |a - offset|, and every rebuilt scale is within half the code's largest gap of the original
    (plus the rebuild's two roundings)."""
    code = oracle_mod.code_dynamic_signed()
    a = np.random.default_rng(seed).lognormal(mu, sigma, nb).astype(np.float32)
    q, a2, off = oracle_mod.nest_absmax(a, code)
    exact = sum((Fraction(float(v)) for v in a), Fraction(0)) / nb
    assert abs(Fraction(float(off)) - exact) <= Fraction(float(np.spacing(np.float32(float(exact)))))
    c = a - np.float32(off)
    want = np.array([np.max(np.abs(c[i:i + 256])) for i in range(0, nb, 256)], np.float32)
    np.testing.assert_array_equal(a2, want)
    r = oracle_mod.unnest_absmax(q, a2, off, code).astype(np.float64)
    gap = np.max(np.diff(code.astype(np.float64)))
    blk = np.repeat(a2.astype(np.float64), 256)[:nb]
    tol = blk * gap / 2 * (1 + 1e-6) + 2 * np.spacing(np.abs(r).astype(np.float32)).astype(np.float64) \
        + np.spacing(np.float32(abs(off))).astype(np.float64)
    assert np.all(np.abs(r - a) <= tol)
