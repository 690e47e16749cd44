"""GPU parity: block-wise quantize / dequantize through the C ABI against the CPU oracle.

Workload: the standalone quantize + dequantize sweep -- fp32 and bf16 tensors, N(0,1) with 0.1%
of positions scaled x50, blocksize 256/2048/4096 (and 64/128, the 4-bit weight setting), 8-bit
signed dynamic code and NF4 (seed 1).
2^20-element tensors (plus a ragged tail) are compared element by element; the 2^24 and 2^28
tensors are run whole, in the launch configuration of the benchmark, and compared on sampled
blocks that the oracle recomputes one by one (blocks are independent).  Bar: bit-exact codes,
block scales and dequantized values.
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


def _codes():
    return {"signed": bq.bnbq_codebook("dynamic_signed"), "nf4": bq.bnbq_codebook("nf4"), "fp4": bq.bnbq_codebook("fp4"),
            "unsigned": bq.bnbq_codebook("dynamic_unsigned"), "linear": bq.bnbq_codebook("linear")}


def sweep_input(n, dtype, seed_tag, device=DEV):
    x = W.normal(n, 1.0, device, "quant-sweep", 1, seed_tag)
    W.outliers_(x, 0.001, 50.0, device, "quant-sweep", 1, seed_tag)
    return x.to(dtype)


def _with_canary(n, dtype, pad=64):
    """Device buffer of n elements followed by a canary region; returns (view, full)."""
    full = torch.empty(n + pad, dtype=dtype, device=DEV)
    if dtype == torch.uint8:
        full.fill_(0xA5)
    else:
        full.fill_(-12345.0)
    return full[:n], full


def _canary_ok(full, n):
    tail = full[n:]
    return bool((tail == (0xA5 if full.dtype == torch.uint8 else -12345.0)).all())


def _run_quant(code, x, B):
    n = x.numel()
    K = code.numel()
    nq = n if K == 256 else (n + 1) // 2
    nb = (n + B - 1) // B
    q, qfull = _with_canary(nq, torch.uint8)
    a, afull = _with_canary(nb, torch.float32)
    bq.bnbq_quantize_blockwise(code.to(DEV), x, B, absmax=a, out=q)
    torch.cuda.synchronize()
    assert _canary_ok(qfull, nq) and _canary_ok(afull, nb), "write past the end of an output"
    return a, q


def _check_full(code_cpu, x, B):
    a, q = _run_quant(code_cpu, x, B)
    a_or, q_or = oracle.quantize_blockwise(code_cpu.numpy(), parity.to_np(x), B)
    np.testing.assert_array_equal(parity.to_np(a).view(np.uint32), a_or.view(np.uint32))
    np.testing.assert_array_equal(parity.to_np(q), q_or)
    # dequantize both dtypes
    n = x.numel()
    for dt in (torch.float32, torch.bfloat16):
        y = bq.bnbq_dequantize_blockwise(code_cpu.to(DEV), q, a, n, B, out_dtype=dt)
        y_or = oracle.dequantize_blockwise(code_cpu.numpy(), q_or, a_or, n, B, out_bf16=(dt == torch.bfloat16))
        gy = parity.to_np(y)
        np.testing.assert_array_equal(gy.view(np.uint32) if dt == torch.float32 else gy,
                                      y_or.view(np.uint32) if dt == torch.float32 else y_or)
    return a, q


@pytest.mark.parametrize("code_name", ["signed", "nf4", "fp4"])
@pytest.mark.parametrize("B", [64, 128, 256, 2048, 4096])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_sweep_2p20_elementwise(code_name, B, dtype):
    code = _codes()[code_name]
    n = 2 ** 20 + 517  # several tiles per CTA and a ragged tail
    x = sweep_input(n, dtype, f"{code_name}-{B}-{dtype}")
    _check_full(code, x, B)


@pytest.mark.parametrize("n", [2 ** 20 + 517, 2 ** 20])
@pytest.mark.parametrize("code_name", ["signed", "nf4"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_staged_tiles_many_per_cta(code_name, dtype, n, monkeypatch):
    """Aligned fp32 input goes through the shared-memory stages (forced at this size).  With
    the grid capped at 3 CTAs every CTA takes 43 tiles (each stage refilled about 20 times, its
    barrier phase flipping each time) and one CTA also quantizes the ragged last tile; bf16 input
    (plain loads) takes 21 passes per CTA.  Compared element by element with the oracle, at
    blocksizes with 4 to 128 threads per block; and a size of whole tiles (no ragged tile)."""
    monkeypatch.setenv("BNBQ_QUANT_MAX_CTAS", "3")
    monkeypatch.setenv("BNBQ_QUANT_STAGE_FROM", "0")  # staged at this size too (by default from 2^26)
    code = _codes()[code_name]
    x = sweep_input(n, dtype, f"staged-{code_name}-{dtype}-{n}")
    for B in (64, 128, 2048):
        _check_full(code, x, B)


@pytest.mark.parametrize("cap,stage_from", [("abc", "-5"), ("0", "x1"), ("", "")])
def test_testing_aids_ignore_malformed_values(cap, stage_from, monkeypatch):
    """Malformed or empty values of the quantize kernel's testing variables leave the defaults in
    force; results as the oracle's."""
    monkeypatch.setenv("BNBQ_QUANT_MAX_CTAS", cap)
    monkeypatch.setenv("BNBQ_QUANT_STAGE_FROM", stage_from)
    x = sweep_input(50_000 + 11, torch.float32, f"aids-{cap}-{stage_from}")
    _check_full(_codes()["signed"], x, 2048)


@pytest.mark.parametrize("code_name", ["unsigned", "linear"])
def test_other_codebooks(code_name):
    """Unsigned dynamic code (non-negative data) and the linear code (it has a zero midpoint, so
    the kernel takes the IEEE-division path)."""
    code = _codes()[code_name]
    x = sweep_input(300_001, torch.float32, code_name)
    if code_name == "unsigned":
        x = x.abs()
    _check_full(code, x, 2048)


@pytest.mark.parametrize("kind", ["crowded", "crowded11", "tiny"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_16_codes_outside_the_prefix_table(kind, dtype):
    """16-entry codebooks the 11-bit-prefix search cannot take: two midpoints in one of its
    buckets (codes 0.5, 0.505, 0.51, which a 12-bit prefix would not separate either, or 0.5,
    0.53, 0.6, which it would), where the kernel falls back to the 16-bit-prefix table or the
    midpoint walk; and a midpoint below 2^-41 (outside the FMA quotient's safe range), where it
    divides with IEEE division.  Results as the oracle's."""
    base = np.concatenate([-np.linspace(1.0, 0.125, 7), [0.0]])
    if kind == "crowded":
        pos = [0.25, 0.5, 0.505, 0.51, 0.75, 0.875, 0.9375, 1.0]
    elif kind == "crowded11":
        pos = [0.25, 0.5, 0.53, 0.6, 0.75, 0.875, 0.9375, 1.0]
    else:
        pos = [2.0 ** -45, 0.125, 0.25, 0.375, 0.5, 0.625, 0.75, 1.0]
    code = torch.tensor(np.concatenate([base, pos]).astype(np.float32))
    assert bq.bnbq_check_codebook(code) is None and code.numel() == 16
    x = sweep_input(64 * 3000 + 19, dtype, f"16codes-{kind}")
    for B in (64, 2048):
        _check_full(code, x, B)


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 255, 256, 257, 2047, 2049, 4097, 8191])
@pytest.mark.parametrize("code_name", ["signed", "nf4"])
def test_small_and_ragged(n, code_name):
    code = _codes()[code_name]
    x = sweep_input(n, torch.float32, f"ragged-{n}")
    for B in (256, 2048, 4096):
        _check_full(code, x, B)


@pytest.mark.parametrize("n", [1, 5, 7, 8, 9, 31, 33, 63, 64, 65, 127, 129, 2049, 65 * 64 + 3])
@pytest.mark.parametrize("code_name", ["signed", "nf4"])
def test_small_and_ragged_bf16(n, code_name):
    """bf16 input, whose full blocks take 8-element chunks: ragged tails inside a chunk and a
    block, for the 4-bit weight blocksize and the optimizer-state ones."""
    code = _codes()[code_name]
    x = sweep_input(n, torch.bfloat16, f"ragged-bf16-{n}")
    for B in (64, 256, 2048):
        _check_full(code, x, B)


@pytest.mark.parametrize("code_name", ["signed", "nf4"])
def test_bf16_input_and_codes_at_narrow_alignment(code_name):
    """bf16 input only 8-byte aligned and codes only as aligned as the interface asks (4 bytes for
    8-bit codes, 2 for 4-bit): quantize falls back to 4-element chunks and dequantize to 16-bit
    code loads; results as the oracle's."""
    code = _codes()[code_name]
    n, B = 64 * 1000 + 37, 64
    K = code.numel()
    xf = sweep_input(n + 4, torch.bfloat16, "narrow")
    x = xf[4:]                                  # 8 bytes past a 16-byte boundary
    assert x.data_ptr() % 16 == 8
    nq = n if K == 256 else (n + 1) // 2
    step = 4 if K == 256 else 2
    qf = torch.full((nq + step + 64,), 0xA5, dtype=torch.uint8, device=DEV)
    q = qf[step:step + nq]                      # 4 (8-bit) or 2 (4-bit) bytes past an 8-byte boundary
    a = torch.empty((n + B - 1) // B, dtype=torch.float32, device=DEV)
    bq.bnbq_quantize_blockwise(code.to(DEV), x, B, absmax=a, out=q)
    torch.cuda.synchronize()
    assert bool((qf[:step] == 0xA5).all()) and bool((qf[step + nq:] == 0xA5).all()), "write outside the codes"
    a_or, q_or = oracle.quantize_blockwise(code.numpy(), parity.to_np(x), B)
    np.testing.assert_array_equal(parity.to_np(a).view(np.uint32), a_or.view(np.uint32))
    np.testing.assert_array_equal(parity.to_np(q), q_or)
    for dt in (torch.float32, torch.bfloat16):
        y = bq.bnbq_dequantize_blockwise(code.to(DEV), q, a, n, B, out_dtype=dt)
        y_or = oracle.dequantize_blockwise(code.numpy(), q_or, a_or, n, B, out_bf16=(dt == torch.bfloat16))
        gy = parity.to_np(y)
        np.testing.assert_array_equal(gy.view(np.uint32) if dt == torch.float32 else gy,
                                      y_or.view(np.uint32) if dt == torch.float32 else y_or)


def test_empty_is_noop():
    code = _codes()["signed"].to(DEV)
    x = torch.empty(0, device=DEV)
    a, q = bq.bnbq_quantize_blockwise(code, x, 2048)
    assert a.numel() == 0 and q.numel() == 0
    y = bq.bnbq_dequantize_blockwise(code, q, a, 0, 2048)
    assert y.numel() == 0


def test_edge_values():
    """Zero blocks, subnormal blocks, negative absmax elements, huge values, exact codes and
    exact midpoints (ties go to the lower code), codes scaled by powers of two."""
    sc = _codes()["signed"]
    c = sc.numpy()
    B = 256
    blocks = []
    blocks.append(np.zeros(B, np.float32))
    blocks.append(np.full(B, -0.0, np.float32))
    sub = np.zeros(B, np.float32)
    sub[:4] = [1e-45, -2e-45, 3e-45, 1e-40]
    blocks.append(sub)
    neg = np.linspace(-0.5, 0.5, B).astype(np.float32)
    neg[17] = -3.0
    blocks.append(neg)
    blocks.append(np.linspace(-3e38, 3e38, B).astype(np.float32))
    A = np.float32(2.0 ** -7)
    blocks.append(np.concatenate([c[::2] * A, [A]]).astype(np.float32)[:B])
    mids = ((c[:-1].astype(np.float64) + c[1:]) / 2).astype(np.float32)
    m = np.concatenate([mids[:B - 1] * A, [A]]).astype(np.float32)
    blocks.append(m)
    blocks.append((np.nextafter(mids, 2)[:B - 1] * A).tolist() + [A])
    tiny_scale = np.concatenate([c[:B - 1] * np.float32(2.0 ** -100), [np.float32(2.0 ** -100)]])
    blocks.append(tiny_scale.astype(np.float32))
    big_scale = np.concatenate([c[:B - 1] * np.float32(2.0 ** 110), [np.float32(2.0 ** 110)]])
    blocks.append(big_scale.astype(np.float32))
    x = torch.from_numpy(np.concatenate([np.asarray(b, np.float32) for b in blocks])).to(DEV)
    for code in (sc, _codes()["nf4"]):
        _check_full(code, x, B)


def test_bad_codebook_sets_flag_and_writes_nothing():
    bad = _codes()["signed"].flip(0).contiguous().to(DEV)
    x = sweep_input(10000, torch.float32, "bad")
    q = torch.full((10000,), 7, dtype=torch.uint8, device=DEV)
    a = torch.full((5,), 3.0, device=DEV)
    bq.bnbq_device_flags(clear=True)
    bq.bnbq_quantize_blockwise(bad, x, 2048, absmax=a, out=q)
    flags = bq.bnbq_device_flags(clear=True)
    assert flags & 0x1
    assert bool((q == 7).all()) and bool((a == 3.0).all())


def test_nonfinite_input_sets_flag():
    x = sweep_input(5000, torch.float32, "nan")
    x[123] = float("nan")
    bq.bnbq_device_flags(clear=True)
    bq.bnbq_quantize_blockwise(_codes()["signed"].to(DEV), x, 2048)
    assert bq.bnbq_device_flags(clear=True) & 0x2


@pytest.mark.parametrize("log2n", [24, 28])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_sweep_full_size_sampled(log2n, dtype):
    """Whole 2^24 / 2^28 tensors through the kernel; 24 sampled blocks per blocksize recomputed
    by the oracle, plus a full-array property check (every code within range, every absmax the
    max of its block, computed by torch)."""
    n = 2 ** log2n
    x = sweep_input(n, dtype, f"full-{log2n}")
    rng = np.random.default_rng(log2n)
    for code_name in ("signed", "nf4"):
        code = _codes()[code_name]
        for B in (256, 2048, 4096):
            a, q = bq.bnbq_quantize_blockwise(code.to(DEV), x, B)
            nb = n // B
            want_a = x.float().view(nb, B).abs().amax(dim=1)
            assert torch.equal(a, want_a)
            if code_name == "nf4":
                assert q.numel() == n // 2
            else:
                assert int(q.max()) <= 255
            sample = np.unique(np.concatenate([[0, nb - 1], rng.integers(0, nb, 22)]))
            for b in sample:
                xs = parity.to_np(x[b * B:(b + 1) * B])
                a_or, q_or = oracle.quantize_blockwise(code.numpy(), xs, B)
                assert parity.to_np(a[b:b + 1]).view(np.uint32)[0] == a_or.view(np.uint32)[0]
                lo, hi = (b * B, (b + 1) * B) if code_name != "nf4" else (b * B // 2, (b + 1) * B // 2)
                np.testing.assert_array_equal(parity.to_np(q[lo:hi]), q_or)
            y = bq.bnbq_dequantize_blockwise(code.to(DEV), q, a, n, B, out_dtype=dtype)
            for b in sample[:6]:
                lo, hi = (b * B, (b + 1) * B) if code_name != "nf4" else (b * B // 2, (b + 1) * B // 2)
                y_or = oracle.dequantize_blockwise(code.numpy(), parity.to_np(q[lo:hi]), parity.to_np(a[b:b + 1]),
                                                   B, B, out_bf16=(dtype == torch.bfloat16))
                np.testing.assert_array_equal(parity.to_np(y[b * B:(b + 1) * B]), y_or)
            del a, q, y
    torch.cuda.empty_cache()


@pytest.mark.parametrize("code_name", ["signed", "nf4"])
def test_beyond_2p31_elements_sampled(code_name):
    """Maximum sizes: a bf16 tensor of 2^31 + 4099 elements (element and byte offsets past 32
    bits, a ragged last block).  Blocks at the start, around element 2^31 and at the end are
    recomputed by the oracle; every block scale is checked against torch's block maxima."""
    if torch.cuda.get_device_properties(0).total_memory < 40e9:
        pytest.skip("needs a GPU with >= 40 GB")
    n, B = 2 ** 31 + 4099, 4096
    x = W.normal(n, 1.0, DEV, "huge", code_name).to(torch.bfloat16)
    code = _codes()[code_name]
    a, q = bq.bnbq_quantize_blockwise(code.to(DEV), x, B)
    nb = (n + B - 1) // B
    full = n // B
    want_a = x[:full * B].float().view(full, B).abs().amax(dim=1)
    assert torch.equal(a[:full], want_a)
    assert float(a[-1]) == float(x[full * B:].float().abs().max())
    edge = (2 ** 31) // B
    for b in (0, 1, edge - 1, edge, edge + 1, nb - 2, nb - 1):
        e0, e1 = b * B, min(n, (b + 1) * B)
        xs = x[e0:e1].view(torch.int16).cpu().numpy().view(np.uint16)
        a_or, q_or = oracle.quantize_blockwise(code.numpy(), xs, B)
        assert parity.to_np(a[b:b + 1]).view(np.uint32)[0] == a_or.view(np.uint32)[0]
        lo, hi = (e0, e1) if code_name != "nf4" else (e0 // 2, (e1 + 1) // 2)
        np.testing.assert_array_equal(parity.to_np(q[lo:hi]), q_or)
    del want_a
    y = bq.bnbq_dequantize_blockwise(code.to(DEV), q, a, n, B, out_dtype=torch.bfloat16)
    for b in (0, edge, nb - 1):
        e0, e1 = b * B, min(n, (b + 1) * B)
        lo, hi = (e0, e1) if code_name != "nf4" else (e0 // 2, (e1 + 1) // 2)
        y_or = oracle.dequantize_blockwise(code.numpy(), parity.to_np(q[lo:hi]), parity.to_np(a[b:b + 1]), e1 - e0, B,
                                           out_bf16=True)
        np.testing.assert_array_equal(y[e0:e1].view(torch.int16).cpu().numpy().view(np.uint16), y_or)
    del x, a, q, y
    torch.cuda.empty_cache()
