"""bnbq_step_8bit_noalloc: the optimizer step for callers that cannot let the library allocate
device memory (all device memory owned by their own pool, or no allocation allowed between steps).

It must give the same results as bnbq_step_8bit, the allocating entry point, call after call:
both run the same kernel and only the home of the descriptor table differs (a fixed array inside
the library instead of cached allocations).  This file is collected last so that a run stopping at
its first failure has already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_wise_bit_b200 as bq
from block_wise_bit_b200 import bindings as B
from block_wise_bit_b200 import workloads as W

from . import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"
HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
SIZES = [3, 4095, 4096, 2048 * 5 + 17, 65536, 100003]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    bq.lib()
    yield


def _list(seed, sizes, blocksize):
    """Two identical copies of a tensor list with a synthetic non-zero state (8-bit state for
    tensors of 4096 elements or more, 32-bit below)."""
    copies = ([], [])
    for i, n in enumerate(sizes):
        p = W.normal(n, 0.02, DEV, "noalloc", seed, i, "p")
        g = W.normal(n, 1e-3, DEV, "noalloc", seed, i, "g").to(torch.bfloat16)
        if n >= 4096:
            nb = (n + blocksize - 1) // blocksize
            s1 = W.random_codes(n, DEV, "noalloc", seed, i, "q1")
            s2 = W.random_codes(n, DEV, "noalloc", seed, i, "q2")
            a1 = W.log_uniform(nb, 1e-4, 1e-2, DEV, "noalloc", seed, i, "a1")
            a2 = W.log_uniform(nb, 1e-8, 1e-5, DEV, "noalloc", seed, i, "a2")
        else:
            s1 = W.normal(n, 1e-3, DEV, "noalloc", seed, i, "m")
            s2 = W.normal(n, 1e-3, DEV, "noalloc", seed, i, "v").square_()
            a1 = a2 = None
        for c in copies:
            c.append(bq.TensorState(p.clone(), g, s1.clone(), s2.clone(), None if a1 is None else a1.clone(),
                                    None if a2 is None else a2.clone()))
    return copies


def _same(ref, got):
    for i, (r, t) in enumerate(zip(ref, got)):
        parity.assert_p_close(parity.to_np(t.p), parity.to_np(r.p), f"tensor {i} p")
        if r.absmax1 is not None:
            np.testing.assert_array_equal(parity.to_np(t.state1), parity.to_np(r.state1))
            np.testing.assert_array_equal(parity.to_np(t.state2), parity.to_np(r.state2))
            np.testing.assert_array_equal(parity.to_np(t.absmax1), parity.to_np(r.absmax1))
            np.testing.assert_array_equal(parity.to_np(t.absmax2), parity.to_np(r.absmax2))
        else:
            np.testing.assert_allclose(parity.to_np(t.state1), parity.to_np(r.state1), rtol=1e-6, atol=1e-12)
            np.testing.assert_allclose(parity.to_np(t.state2), parity.to_np(r.state2), rtol=1e-6, atol=1e-18)


@pytest.mark.parametrize("blocksize", [2048, 256])
def test_noalloc_step_matches_allocating_step_on_consecutive_calls(blocksize):
    c1 = bq.bnbq_codebook("dynamic_signed").to(DEV)
    c2 = bq.bnbq_codebook("dynamic_unsigned").to(DEV)
    ref, got = _list(7, SIZES, blocksize)
    for t in (1, 2):  # two calls in a row share the library's fixed table
        B.bnbq_step_8bit("adamw", ref, step=t, code1=c1, code2=c2, blocksize=blocksize, **HP)
        B.bnbq_step_8bit_noalloc("adamw", got, step=t, code1=c1, code2=c2, blocksize=blocksize, **HP)
        torch.cuda.synchronize()
        _same(ref, got)
    # a different, shorter list next: the fixed table is rewritten, not appended to
    ref2, got2 = _list(8, SIZES[2:4], blocksize)
    B.bnbq_step_8bit("adamw", ref2, step=3, code1=c1, code2=c2, blocksize=blocksize, **HP)
    B.bnbq_step_8bit_noalloc("adamw", got2, step=3, code1=c1, code2=c2, blocksize=blocksize, **HP)
    torch.cuda.synchronize()
    _same(ref2, got2)
    assert bq.bnbq_device_flags(clear=True) == 0


def test_noalloc_rejects_lists_beyond_its_table():
    """More non-empty tensors than the fixed table holds: a clear error, nothing launched."""
    n = 4097
    arr = (B.CTensor * n)()
    for i in range(n):
        arr[i] = B.CTensor(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000, 4096, 1, 8)
    hp = B.CHParams(1e-3, 0.9, 0.999, 1e-8, 0.0)
    rc = B.lib().bnbq_step_8bit_noalloc(0, arr, n, ctypes.byref(hp), 1, 0x7000, 0x8000, 2048, None)
    assert rc == B.EINVAL
    assert "at most 4096" in B.bnbq_last_error()


def test_noalloc_step_takes_no_device_memory():
    """After one call on the device (which may load the library's device code), further calls
    with lists of different lengths leave the device's free memory unchanged: the entry point
    allocates nothing, not even the descriptor table that the allocating entry point caches."""
    c1 = bq.bnbq_codebook("dynamic_signed").to(DEV)
    c2 = bq.bnbq_codebook("dynamic_unsigned").to(DEV)
    _, lists = _list(9, SIZES, 2048)
    subsets = [lists, lists[:2], lists[3:], lists[1:5]]
    B.bnbq_step_8bit_noalloc("adamw", lists, step=1, code1=c1, code2=c2, blocksize=2048, **HP)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for t, sub in enumerate(subsets, start=2):
        B.bnbq_step_8bit_noalloc("adamw", sub, step=t, code1=c1, code2=c2, blocksize=2048, **HP)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert bq.bnbq_device_flags(clear=True) == 0
