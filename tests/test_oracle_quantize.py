"""Pins for the oracle's block-wise quantize / dequantize (CPU only).

Block-wise quantization, per the abstract of "8-bit Optimizers via Block-wise Quantization"
(quoted on the blog.csdn.net bitsandbytes guide, section 2): the tensor is cut into blocks that
are quantized independently.  The oracle normalises each block by its absolute maximum and
takes the nearest code.  These tests pin it by exact rational brute force (argmin of the
distance over every code, ties to the lower code), by round trips through the codebook, by the
error bound of a nearest-code rule, and by torch's own bf16 rounding.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st

RNG = np.random.default_rng(12345)


def _codes(o):
    return {"signed": o.code_dynamic_signed(), "unsigned": o.code_dynamic_unsigned(),
            "nf4": o.code_nf4(), "fp4": o.code_fp4(), "linear": o.code_linear()}


def _argmin_exact(code, xn):
    """Index of the code nearest to xn in exact arithmetic; a tie goes to the lower index."""
    x = Fraction(float(xn))
    best, bestd = 0, None
    for j, c in enumerate(code):
        d = abs(Fraction(float(c)) - x)
        if bestd is None or d < bestd:
            best, bestd = j, d
    return best


def _is_rounded_mid(code, xn):
    """xn equals fl32(mid) of a neighbour pair whose exact mean is not a binary32 number."""
    for j in range(len(code) - 1):
        exact = (Fraction(float(code[j])) + Fraction(float(code[j + 1]))) / 2
        fm = np.float32(float(exact))
        if Fraction(float(fm)) != exact and np.float32(xn) == fm:
            return True
    return False


def _adversarial_xn(code, rng, n_random):
    vals = [0.0, -0.0, 1.0, -1.0, np.float32(1e-45), -np.float32(1e-45)]
    vals += list(code)
    for j in range(len(code) - 1):
        m = (float(code[j]) + float(code[j + 1])) / 2
        fm = np.float32(m)
        vals += [fm, np.nextafter(fm, np.float32(2)), np.nextafter(fm, np.float32(-2))]
    vals += list(rng.uniform(-1, 1, n_random).astype(np.float32))
    vals += list((rng.standard_normal(n_random) * 10.0 ** rng.uniform(-9, 0, n_random)).astype(np.float32))
    vals = np.clip(np.array(vals, np.float32), -1, 1)
    if code.min() >= 0:
        vals = np.abs(vals)
    return vals


@pytest.mark.parametrize("name", ["signed", "unsigned", "nf4", "fp4", "linear"])
def test_nearest_code_exact_bruteforce(oracle_mod, name):
    code = _codes(oracle_mod)[name]
    xs = _adversarial_xn(code, np.random.default_rng(7), 400)
    n_rounded_mid = 0
    for xn in xs:
        q = oracle_mod.nearest_code(code, float(xn))
        want = _argmin_exact(code, xn)
        if q != want:
            assert _is_rounded_mid(code, xn), (name, float(xn), q, want)
            assert q == want - 1  # rounded-up midpoint decided towards the lower code
            n_rounded_mid += 1
    # the mismatches are exactly the enumerated fl(mid) != mid cases, and there are few
    assert n_rounded_mid <= len(code)


def _neighbour_argmin(code, xn):
    """Vectorised exact nearest code for xn inside [code[0], code[-1]] (code sorted)."""
    c64 = code.astype(np.float64)
    x64 = xn.astype(np.float64)
    hi = np.clip(np.searchsorted(c64, x64, side="left"), 1, len(code) - 1)
    lo = hi - 1
    dlo = x64 - c64[lo]
    dhi = c64[hi] - x64
    q = np.where(dhi < dlo, hi, lo)
    near_tie = np.abs(dhi - dlo) <= 1e-12 * np.maximum(np.abs(x64), 1e-30)
    for i in np.nonzero(near_tie)[0]:
        q[i] = _argmin_exact(code, xn[i])
    return q


def _blocks(x, B):
    n = x.size
    return [(s, min(n, s + B)) for s in range(0, n, B)]


@pytest.mark.parametrize("name", ["signed", "unsigned", "nf4", "fp4", "linear"])
@pytest.mark.parametrize("B", [64, 128, 256, 2048, 4096])
@pytest.mark.parametrize("bf16", [False, True])
def test_quantize_blockwise_matches_bruteforce(oracle_mod, name, B, bf16):
    code = _codes(oracle_mod)[name]
    n = 3 * B + 517  # several blocks and a ragged tail
    x = RNG.standard_normal(n).astype(np.float32)
    x[RNG.random(n) < 0.001] *= 50.0
    if code.min() >= 0:
        x = np.abs(x)
    if bf16:
        xin = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        xv = oracle_mod.bf16_bits_to_f32(xin)
    else:
        xin, xv = x, x
    absmax, q = oracle_mod.quantize_blockwise(code, xin, B)
    assert absmax.shape == ((n + B - 1) // B,)
    K = len(code)
    if K == 16:
        assert q.size == (n + 1) // 2
        qi = np.empty(n, np.int64)
        qi[0::2] = q[: (n + 1) // 2] >> 4
        qi[1::2] = (q & 0xF)[: n // 2]
        if n % 2:
            assert q[-1] & 0xF == 0
    else:
        qi = q.astype(np.int64)
    for b, (s, e) in enumerate(_blocks(xv, B)):
        blk = xv[s:e]
        assert absmax[b] == np.max(np.abs(blk)), "absmax over the elements present"
        xn = blk / absmax[b]  # binary32 division, the same precision the decision is taken in
        want = _neighbour_argmin(code, xn.astype(np.float32))
        got = qi[s:e]
        bad = np.nonzero(got != want)[0]
        for i in bad:
            assert _is_rounded_mid(code, xn[i]) and got[i] == want[i] - 1


def test_normalisation_is_the_correctly_rounded_quotient(oracle_mod):
    """x / absmax is one binary32 division (numpy's float32 division is IEEE's correctly rounded
    one), not x times a rounded reciprocal of absmax.  For scales whose reciprocal is inexact the
    inputs are chosen where the two normalisations fall on opposite sides of a decision
    midpoint.  The decision rule itself (xn above the binary32 midpoint of two neighbouring
    codes, ties to the lower code) is pinned against exact nearest-code brute force above; here
    it is taken as given, so that only the quotient is under test."""
    code = oracle_mod.code_dynamic_signed()
    c64 = code.astype(np.float64)
    mid32 = np.float32((c64[:-1] + c64[1:]) / 2)

    def decide(xn):
        return np.searchsorted(mid32, xn, side="left")  # number of midpoints strictly below xn

    for a in (3.0, 7.0, 0.3):
        a32 = np.float32(a)
        r32 = np.float32(1) / a32
        picks = []
        for m in mid32:
            near = (np.float32(m * a32).view(np.int32) + np.arange(-64, 65)).astype(np.int32).view(np.float32)
            near = near[np.abs(near) < a32]
            picks.extend(near[decide(near / a32) != decide(near * r32)].tolist())
        assert len(picks) >= 40
        x = np.array(picks + [float(a32)], np.float32)  # the last element sets the block's absmax
        absmax, q = oracle_mod.quantize_blockwise(code, x, 4096)
        assert absmax[0] == a32
        np.testing.assert_array_equal(q.astype(np.int64), decide(x / a32))


@pytest.mark.parametrize("name", ["signed", "unsigned", "linear", "nf4", "fp4"])
def test_round_trip_every_code(oracle_mod, name):
    """P1: a block {code_j * A, A} quantizes back to j, and dequantizes to code_j * A exactly."""
    code = _codes(oracle_mod)[name]
    K = len(code)
    top = int(np.argmax(code))
    for A in (2.0 ** -20, 0.25, 1.0, 64.0, 2.0 ** 40):
        x = np.concatenate([code * np.float32(A), [np.float32(A)]]).astype(np.float32)
        B = 2048  # all K codes and the absmax element share one block
        absmax, q = oracle_mod.quantize_blockwise(code, x, B)
        assert absmax[0] == np.float32(A)
        if K == 16:
            qi = np.empty(x.size, np.int64)
            qi[0::2] = q >> 4
            qi[1::2] = (q & 0xF)[: x.size // 2]
        else:
            qi = q.astype(np.int64)
        np.testing.assert_array_equal(qi[:K], np.arange(K))
        assert qi[K] == top  # the absmax element maps to code +1 (P3)
        y = oracle_mod.dequantize_blockwise(code, q, absmax, x.size, B)
        np.testing.assert_array_equal(y[:K], code * np.float32(A))


@pytest.mark.parametrize("name", ["signed", "unsigned", "linear"])
def test_quantize_of_dequantize_is_identity(oracle_mod, name):
    """P2: for random q whose block holds the +-1 code, quantize(dequantize(q)) == q."""
    code = _codes(oracle_mod)[name]
    rng = np.random.default_rng(3)
    B, n = 2048, 2048 * 4 + 100
    q = rng.integers(0, 256, n).astype(np.uint8)
    one = int(np.argmax(code))
    q[::B] = one  # each block contains the +1 code
    for A in ([2.0 ** -3] * 5, list(2.0 ** rng.integers(-30, 30, 5))):
        absmax = np.array(A, np.float32)
        y = oracle_mod.dequantize_blockwise(code, q, absmax, n, B)
        a2, q2 = oracle_mod.quantize_blockwise(code, y, B)
        np.testing.assert_array_equal(a2, absmax)
        np.testing.assert_array_equal(q2, q)
    # with arbitrary (non power of two) scales the round trip still holds: report and require 0
    absmax = rng.uniform(0.01, 10, 5).astype(np.float32)
    y = oracle_mod.dequantize_blockwise(code, q, absmax, n, B)
    _, q2 = oracle_mod.quantize_blockwise(code, y, B)
    assert np.mean(q2 != q) == 0.0


def test_negative_absmax_element_maps_to_minus_one(oracle_mod):
    """P3 for a block whose largest magnitude is negative."""
    code = oracle_mod.code_dynamic_signed()
    x = RNG.uniform(-0.5, 0.5, 4096).astype(np.float32)
    x[1234] = -3.0
    absmax, q = oracle_mod.quantize_blockwise(code, x, 4096)
    assert absmax[0] == 3.0 and q[1234] == 0 and code[0] == -1.0


@pytest.mark.parametrize("name", ["signed", "nf4", "linear"])
def test_error_bound(oracle_mod, name):
    """P7: |dequant(quant(x)) - x| <= absmax * (half the widest gap) + rounding."""
    code = _codes(oracle_mod)[name]
    B, n = 256, 256 * 50 + 3
    x = (RNG.standard_normal(n) * 3).astype(np.float32)
    absmax, q = oracle_mod.quantize_blockwise(code, x, B)
    y = oracle_mod.dequantize_blockwise(code, q, absmax, n, B)
    gap = np.max(np.diff(code.astype(np.float64))) / 2
    bound = np.repeat(absmax.astype(np.float64), B)[:n] * (gap + 2 ** -22)
    assert np.all(np.abs(y.astype(np.float64) - x) <= bound)


def test_zero_block_and_empty(oracle_mod):
    code = oracle_mod.code_dynamic_signed()
    x = np.zeros(300, np.float32)
    x[:5] = -0.0
    absmax, q = oracle_mod.quantize_blockwise(code, x, 256)
    assert np.all(absmax == 0) and np.all(q == 127)
    y = oracle_mod.dequantize_blockwise(code, q, absmax, 300, 256)
    assert np.all(y == 0)
    u = oracle_mod.code_dynamic_unsigned()
    _, qu = oracle_mod.quantize_blockwise(u, np.zeros(10, np.float32), 256)
    assert np.all(qu == 0)
    a, qq = oracle_mod.quantize_blockwise(code, np.zeros(0, np.float32), 256)
    assert a.size == 0 and qq.size == 0


def test_subnormal_absmax(oracle_mod):
    code = oracle_mod.code_dynamic_signed()
    x = np.array([1e-45, -2e-45, 3e-45, 0.0], np.float32)  # subnormal block
    absmax, q = oracle_mod.quantize_blockwise(code, x, 256)
    assert absmax[0] == np.float32(3e-45)
    xn = (x / absmax[0]).astype(np.float32)
    np.testing.assert_array_equal(q, [_argmin_exact(code, v) for v in xn])


def test_nf4_nibble_order(oracle_mod):
    code = oracle_mod.code_nf4()
    x = np.array([1.0, -1.0] * 4 + [1.0], np.float32)  # odd length
    absmax, q = oracle_mod.quantize_blockwise(code, x, 256)
    np.testing.assert_array_equal(q, [0xF0, 0xF0, 0xF0, 0xF0, 0xF0])  # even element -> high nibble
    y = oracle_mod.dequantize_blockwise(code, q, absmax, x.size, 256)
    np.testing.assert_array_equal(y, x)


def test_bf16_input_is_exact_widening(oracle_mod):
    code = oracle_mod.code_dynamic_signed()
    x = torch.randn(5000, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    a1, q1 = oracle_mod.quantize_blockwise(code, bits, 2048)
    a2, q2 = oracle_mod.quantize_blockwise(code, x.float().numpy(), 2048)
    np.testing.assert_array_equal(a1, a2)
    np.testing.assert_array_equal(q1, q2)


def test_dequantize_bf16_matches_torch_rounding(oracle_mod):
    code = oracle_mod.code_dynamic_signed()
    rng = np.random.default_rng(9)
    n, B = 4096 + 7, 256
    q = rng.integers(0, 256, n).astype(np.uint8)
    absmax = rng.uniform(0.1, 100, (n + B - 1) // B).astype(np.float32)
    y32 = oracle_mod.dequantize_blockwise(code, q, absmax, n, B)
    y16 = oracle_mod.dequantize_blockwise(code, q, absmax, n, B, out_bf16=True)
    want = torch.from_numpy(y32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(y16, want)
    # the fp32 output is code[q] scaled: exact whenever absmax is a power of two
    absmax2 = (2.0 ** rng.integers(-10, 10, absmax.size)).astype(np.float32)
    y = oracle_mod.dequantize_blockwise(code, q, absmax2, n, B)
    np.testing.assert_array_equal(y / np.repeat(absmax2, B)[:n], code[q])


def test_dequantize_bf16_ties_to_even(oracle_mod):
    """bf16 output rounds to nearest with ties to even, as torch's float32 -> bfloat16
    conversion does.  A codebook made of exact halfway cases (low 16 bits 0x8000) with both
    parities of the kept bits, dequantized with absmax 1, puts every tie through the narrowing."""
    his = np.arange(0x3E00, 0x3E00 + 127, dtype=np.uint32)  # both parities, values in [0.125, 0.25)
    ties = ((his << 16) | 0x8000).view(np.float32)
    code = np.sort(np.concatenate([ties, -ties, np.float32([0.0, 1.0])]).astype(np.float32))
    assert code.size == 256 and np.all(np.diff(code) > 0)
    q = np.arange(256, dtype=np.uint8)
    y = oracle_mod.dequantize_blockwise(code, q, np.ones(1, np.float32), 256, 256, out_bf16=True)
    want = torch.from_numpy(code).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(y, want)
    kept = (code.view(np.uint32) >> 16).astype(np.uint16)
    assert np.any(want == kept) and np.any(want != kept)  # some ties stay, some round away


def test_rejects_bad_arguments(oracle_mod):
    code = oracle_mod.code_dynamic_signed()
    with pytest.raises(ValueError):
        oracle_mod.quantize_blockwise(code, np.zeros(10, np.float32), 1000)
    with pytest.raises(ValueError):
        oracle_mod.quantize_blockwise(code[:100], np.zeros(10, np.float32), 256)


_VALUES = st.one_of(st.floats(-1e4, 1e4, width=32, allow_subnormal=True),
                    st.sampled_from([0.0, -0.0, 1e-45, -1e-45, 3.4e38, -3.4e38, 1.0, -1.0]))


@settings(max_examples=150, deadline=None)
@given(x=st.lists(_VALUES, max_size=300), B=st.sampled_from([64, 128, 256]),
       name=st.sampled_from(["signed", "nf4", "fp4", "unsigned"]))
def test_quantize_random_blocks_match_bruteforce(oracle_mod, x, B, name):
    """Random lengths (empty and ragged included), blocksizes, codebooks and values (zeros,
    subnormals, huge values, exact codes): each block's scale is its largest magnitude and each
    element takes the exact nearest code of its binary32 quotient (ties and rounded midpoints to
    the lower code), packed two per byte for 4-bit codes; dequantizing gives code * scale in
    binary32 within half a code gap of x, and bf16 output is that value rounded as torch does."""
    code = _codes(oracle_mod)[name]
    xs = np.array(x, np.float32)
    if code.min() >= 0:
        xs = np.abs(xs)
    n = xs.size
    absmax, q = oracle_mod.quantize_blockwise(code, xs, B)
    assert absmax.shape == ((n + B - 1) // B,)
    if len(code) == 16:
        assert q.size == (n + 1) // 2
        qi = np.empty(n, np.int64)
        qi[0::2] = q[: (n + 1) // 2] >> 4
        qi[1::2] = (q & 0xF)[: n // 2]
    else:
        qi = q.astype(np.int64)
    for b, (s, e) in enumerate(_blocks(xs, B)):
        blk = xs[s:e]
        a = np.max(np.abs(blk))
        assert absmax[b] == a
        xn = blk / a if a > 0 else np.zeros_like(blk)
        for i in range(e - s):
            want = _argmin_exact(code, xn[i])
            got = int(qi[s + i])
            assert got == want or (_is_rounded_mid(code, xn[i]) and got == want - 1), (b, i, xn[i], got, want)
    # dequantize: within half the code's largest gap of x (times the block scale), and the bf16
    # output is torch's rounding of the fp32 output
    y = oracle_mod.dequantize_blockwise(code, q, absmax, n, B)
    np.testing.assert_array_equal(y, (code[qi] * np.repeat(absmax, B)[:n]).astype(np.float32))
    gap = np.max(np.diff(code.astype(np.float64)))
    scale = np.repeat(absmax.astype(np.float64), B)[:n]
    assert np.all(np.abs(y.astype(np.float64) - xs) <= scale * gap / 2 * (1 + 1e-6) + np.spacing(np.abs(y)))
    yb = oracle_mod.dequantize_blockwise(code, q, absmax, n, B, out_bf16=True)
    np.testing.assert_array_equal(yb, torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
