"""GPU parity: nested (double) quantization of block scales through the C ABI against the CPU
oracle (page "Bitsandbytes", section "İç içe nicelleştirme"; QLoRA's double quantization).

Workloads: log-normal scale arrays of several lengths (chunk and block edges of the mean and
of the 256-scale blocks), and the 4-bit weight setting end to end -- NF4, blocksize 64, fp32
and bf16 weights ~N(0, 0.02) with 0.1% outliers x50 -- quantized, its scales nested, then
dequantized in one pass with the scales rebuilt on the fly.  Bar: bit-exact offset, codes, second
level scales, rebuilt scales and dequantized values.
"""
import numpy as np
import pytest
import torch

import block_wise_bit_b200 as bq
from block_wise_bit_b200 import workloads as W

from . import parity
import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    bq.lib()
    bq.bnbq_device_flags(clear=True)
    yield
    assert bq.bnbq_device_flags(clear=True) == 0


def _scales(nb, tag):
    return W.log_uniform(nb, 1e-4, 1.0, DEV, "nested", tag)


@pytest.mark.parametrize("nb", [1, 255, 256, 257, 4095, 4096, 4097, 70001, 1 << 20])
def test_nest_absmax_bit_exact(nb):
    code2 = bq.bnbq_codebook("dynamic_signed")
    a = _scales(nb, nb)
    qabs, a2, off = bq.bnbq_quantize_absmax_nested(code2.to(DEV), a)
    q_or, a2_or, off_or = oracle.nest_absmax(parity.to_np(a), code2.numpy())
    assert parity.to_np(off).view(np.uint32)[0] == np.float32(off_or).view(np.uint32)
    np.testing.assert_array_equal(parity.to_np(a2).view(np.uint32), a2_or.view(np.uint32))
    np.testing.assert_array_equal(parity.to_np(qabs), q_or)
    r = bq.bnbq_dequantize_absmax_nested(code2.to(DEV), qabs, a2, off)
    r_or = oracle.unnest_absmax(q_or, a2_or, off_or, code2.numpy())
    np.testing.assert_array_equal(parity.to_np(r).view(np.uint32), r_or.view(np.uint32))


@pytest.mark.parametrize("nb", [4096, 70001])
def test_nest_absmax_mean_any_spread(nb):
    """The mean's chunk sums: chunks whose scales span at most 2^17 in ulp size are added in
    parallel (the index-order sum is then exact), wider ones in index order.  Chunks of both kinds,
    zeros and subnormal scales: the offset must still equal the oracle's index-order sum."""
    code2 = bq.bnbq_codebook("dynamic_signed")
    a = W.log_uniform(nb, 1e-4, 1.0, DEV, "nested-spread", nb)
    a[4096:8192] = W.log_uniform(min(4096, max(0, nb - 4096)), 1e-44, 1.0, DEV, "nested-wide", nb)  # subnormals too
    a[::97] = 0.0
    a[5] = 2.0 ** -130  # a subnormal in the first (narrow) chunk
    qabs, a2, off = bq.bnbq_quantize_absmax_nested(code2.to(DEV), a)
    q_or, a2_or, off_or = oracle.nest_absmax(parity.to_np(a), code2.numpy())
    assert parity.to_np(off).view(np.uint32)[0] == np.float32(off_or).view(np.uint32)
    np.testing.assert_array_equal(parity.to_np(qabs), q_or)
    np.testing.assert_array_equal(parity.to_np(a2).view(np.uint32), a2_or.view(np.uint32))


@pytest.mark.parametrize("nb", [8192 + 5, 70001, 1 << 20])
def test_nest_absmax_mean_narrow_scales(nb):
    """Scales within a factor 8 of each other (ulps spanning at most 2^3): the sum over the whole
    array is exact, so the last CTA adds the chunk sums in parallel; with zeros mixed in.  The
    offset must equal the oracle's index-order sum."""
    code2 = bq.bnbq_codebook("dynamic_signed")
    a = W.log_uniform(nb, 0.5, 4.0, DEV, "nested-narrow", nb)
    a[::61] = 0.0
    qabs, a2, off = bq.bnbq_quantize_absmax_nested(code2.to(DEV), a)
    q_or, a2_or, off_or = oracle.nest_absmax(parity.to_np(a), code2.numpy())
    assert parity.to_np(off).view(np.uint32)[0] == np.float32(off_or).view(np.uint32)
    np.testing.assert_array_equal(parity.to_np(qabs), q_or)
    np.testing.assert_array_equal(parity.to_np(a2).view(np.uint32), a2_or.view(np.uint32))


def test_nest_absmax_staged_centred_quantize(monkeypatch):
    """The centred 8-bit quantize of the scales through the shared-memory stages (forced at this
    size; by default staging starts at 2^26 scales), with the grid capped so that every CTA takes
    several tiles."""
    monkeypatch.setenv("BNBQ_QUANT_STAGE_FROM", "0")
    monkeypatch.setenv("BNBQ_QUANT_MAX_CTAS", "4")
    code2 = bq.bnbq_codebook("dynamic_signed")
    nb = 70001
    a = _scales(nb, "staged")
    qabs, a2, off = bq.bnbq_quantize_absmax_nested(code2.to(DEV), a)
    q_or, a2_or, off_or = oracle.nest_absmax(parity.to_np(a), code2.numpy())
    assert parity.to_np(off).view(np.uint32)[0] == np.float32(off_or).view(np.uint32)
    np.testing.assert_array_equal(parity.to_np(a2).view(np.uint32), a2_or.view(np.uint32))
    np.testing.assert_array_equal(parity.to_np(qabs), q_or)


def test_nest_empty_and_equal_scales():
    code2 = bq.bnbq_codebook("dynamic_signed").to(DEV)
    qabs, a2, off = bq.bnbq_quantize_absmax_nested(code2, torch.empty(0, device=DEV))
    assert qabs.numel() == 0 and float(off) == 0.0
    a = torch.full((1000,), 0.0371, device=DEV)
    qabs, a2, off = bq.bnbq_quantize_absmax_nested(code2, a)
    assert float(off) == float(a[0]) and bool((a2 == 0).all())
    assert torch.equal(bq.bnbq_dequantize_absmax_nested(code2, qabs, a2, off), a)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("n", [64 * 1000 + 33, 1 << 24])
def test_nf4_blocksize64_nested_end_to_end(dtype, n):
    B = 64
    nf4 = bq.bnbq_codebook("nf4")
    code2 = bq.bnbq_codebook("dynamic_signed")
    x = W.normal(n, 0.02, DEV, "nested-w", n, str(dtype))
    W.outliers_(x, 0.001, 50.0, DEV, "nested-w", n, str(dtype))
    x = x.to(dtype)
    a, q = bq.bnbq_quantize_blockwise(nf4.to(DEV), x, B)
    qabs, a2, off = bq.bnbq_quantize_absmax_nested(code2.to(DEV), a)
    a_or, q_or = oracle.quantize_blockwise(nf4.numpy(), parity.to_np(x), B)
    np.testing.assert_array_equal(parity.to_np(q), q_or)
    q2_or, a2_or, off_or = oracle.nest_absmax(a_or, code2.numpy())
    np.testing.assert_array_equal(parity.to_np(qabs), q2_or)
    for out_dtype in (torch.float32, torch.bfloat16):
        y = bq.bnbq_dequantize_blockwise_nested(nf4.to(DEV), q, qabs, a2, off, code2.to(DEV), n, B,
                                                out_dtype=out_dtype)
        y_or = oracle.dequantize_blockwise_nested(nf4.numpy(), q_or, q2_or, a2_or, off_or, code2.numpy(), n, B,
                                                  out_bf16=(out_dtype == torch.bfloat16))
        gy = parity.to_np(y)
        if out_dtype == torch.float32:
            np.testing.assert_array_equal(gy.view(np.uint32), y_or.view(np.uint32))
        else:
            np.testing.assert_array_equal(gy, y_or)
    # the rebuilt scales stay within half a code gap of the plain ones
    r = parity.to_np(bq.bnbq_dequantize_absmax_nested(code2.to(DEV), qabs, a2, off)).astype(np.float64)
    gap = np.max(np.diff(code2.numpy().astype(np.float64)))
    blk = np.repeat(a2_or.astype(np.float64), 256)[: r.size]
    assert np.all(np.abs(r - a_or) <= blk * gap / 2 * (1 + 1e-6) + 4 * np.spacing(np.float32(1.0)) * np.abs(r) + 1e-30)
