"""Helpers shared by the GPU parity tests: run the oracle on host copies of the same seeded
inputs and compare element by element.

Bars (from the method's requirements for this library):
  * quantize / dequantize: code indices, absmax and dequantized values bit-exact;
  * optimizer step: p within 1e-6 relative or 1e-9 absolute per element; requantized state
    indices equal except where the pre-quantization value lies within 2 ulp of a decision
    boundary, and that fraction must stay below 1e-5; absmax mismatches are reported.
With the floating-point rules both sides follow, the expected outcome is fully bit-exact; the
tolerances are the stated bar, and the tests also report how many elements differ at all.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

P_RTOL, P_ATOL = 1e-6, 1e-9
Q_BOUNDARY_FRACTION = 1e-5


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()


def assert_p_close(p_gpu: np.ndarray, p_or: np.ndarray, what: str = "p"):
    diff = np.abs(p_gpu.astype(np.float64) - p_or.astype(np.float64))
    ok = (diff <= P_RTOL * np.abs(p_or.astype(np.float64))) | (diff <= P_ATOL)
    assert ok.all(), f"{what}: {np.count_nonzero(~ok)} of {ok.size} outside 1e-6 rel / 1e-9 abs; first at " \
                     f"{np.nonzero(~ok)[0][:5]}"
    return int(np.count_nonzero(p_gpu.view(np.uint32) != p_or.view(np.uint32)))


def near_boundary(code: np.ndarray, xn: np.ndarray, ulps: int = 2) -> np.ndarray:
    """xn within ``ulps`` binary32 ulps of a decision midpoint of ``code``."""
    mids = np.array([oracle.code_mid(code, j) for j in range(len(code) - 1)], np.float32)
    x = xn.astype(np.float32)
    idx = np.clip(np.searchsorted(mids, x), 1, len(mids) - 1)
    d = np.minimum(np.abs(x - mids[idx - 1]), np.abs(x - mids[idx]))
    return d <= ulps * np.spacing(np.abs(x)).astype(np.float32) + 1e-45


def compare_state(q_gpu, q_or, a_gpu, a_or, code, xn_or=None, what="state"):
    """Compare requantized codes and block scales.  ``xn_or``: the oracle's normalised
    pre-quantization values (for classifying mismatches as near-boundary)."""
    a_mis = int(np.count_nonzero(a_gpu.view(np.uint32) != a_or.view(np.uint32)))
    mis = q_gpu != q_or
    n_mis = int(np.count_nonzero(mis))
    if n_mis:
        assert xn_or is not None, f"{what}: {n_mis} code mismatches"
        nb = near_boundary(code, xn_or[mis])
        assert nb.all(), f"{what}: {np.count_nonzero(~nb)} code mismatches away from a decision boundary"
        assert n_mis / q_gpu.size < Q_BOUNDARY_FRACTION, f"{what}: boundary mismatch fraction {n_mis / q_gpu.size}"
    return n_mis, a_mis


def oracle_step_numpy(optim, p, g, s1, s2, a1, a2, code1, code2, B, hp, t):
    """Run the oracle in place on numpy copies (bf16 gradients given as uint16 bits)."""
    oracle.step_tensor(optim, p, g, s1, s2, a1, a2, code1, code2, B, step=t, **hp)


def oracle_new_moments(optim, p, g, s1, s2, a1, a2, code1, code2, B, hp, t):
    """The oracle's fp32 moments m', v' of one step (via its 32-bit path from the dequantized
    state), for classifying code mismatches."""
    n = p.size
    if s1.dtype == np.uint8:
        m = oracle.dequantize_blockwise(code1, s1, a1, n, B)
        v = oracle.dequantize_blockwise(code2, s2, a2, n, B) if s2 is not None else None
    else:
        m, v = s1.copy(), (s2.copy() if s2 is not None else None)
    pp = p.copy()
    oracle.step_tensor(optim, pp, g, m, v, None, None, None, None, B, step=t, **hp)
    return m, v


def blockwise_normalised(x: np.ndarray, a: np.ndarray, B: int) -> np.ndarray:
    sc = np.repeat(a, B)[: x.size]
    with np.errstate(divide="ignore", invalid="ignore"):
        xn = np.where(sc == 0, 0, x / np.where(sc == 0, 1, sc)).astype(np.float32)
    return xn
