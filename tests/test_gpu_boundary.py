"""C-ABI checks that need a GPU: a codebook must be device memory of the current device, or the
entry point returns BNBQ_EINVAL before it launches anything (the kernel would otherwise read a
host pointer)."""
import ctypes

import pytest
import torch

import block_wise_bit_b200 as bq
from block_wise_bit_b200 import bindings as B
from block_wise_bit_b200 import optim as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    bq.lib()
    yield


def _one_tensor(n=8192, B_=2048):
    p = torch.randn(n, device=DEV) * 0.02
    g = (torch.randn(n, device=DEV) * 1e-3).to(torch.bfloat16)
    st = O.new_state(p, True, 8, B_, O.device_codebook("dynamic_signed", DEV), O.device_codebook("dynamic_unsigned", DEV))
    return bq.TensorState(p, g, st["state1"], st["state2"], st["absmax1"], st["absmax2"])


def _raw_step(fn, t, c1, c2):
    arr = B.pack_tensor_list([t])
    hp = B.CHParams(1e-3, 0.9, 0.999, 1e-8, 0.0)
    return getattr(B.lib(), fn)(0, arr, 1, ctypes.byref(hp), 1, c1, c2, 2048, None)


@pytest.mark.parametrize("fn", ["bnbq_step_8bit", "bnbq_step_8bit_noalloc"])
def test_step_refuses_host_codebooks(fn):
    t = _one_tensor()
    before = [x.clone() for x in (t.p, t.state1, t.state2, t.absmax1, t.absmax2)]
    host = bq.bnbq_codebook("dynamic_signed")              # what bnbq_codebook returns: host memory
    pinned = bq.bnbq_codebook("dynamic_unsigned").pin_memory()
    dev2 = O.device_codebook("dynamic_unsigned", DEV)
    for c1, c2, name in ((host.data_ptr(), dev2.data_ptr(), "code1"),
                         (O.device_codebook("dynamic_signed", DEV).data_ptr(), pinned.data_ptr(), "code2")):
        assert _raw_step(fn, t, c1, c2) == B.EINVAL
        err = B.bnbq_last_error()
        assert name in err and "device memory" in err, err
    torch.cuda.synchronize()
    for a, b in zip(before, (t.p, t.state1, t.state2, t.absmax1, t.absmax2)):
        assert torch.equal(a, b)                             # nothing was launched
    assert bq.bnbq_device_flags(clear=True) == 0


def test_quantize_refuses_host_codebook():
    x = torch.randn(4096, device=DEV)
    absmax = torch.zeros(2, device=DEV)
    out = torch.zeros(4096, dtype=torch.uint8, device=DEV)
    host = bq.bnbq_codebook("dynamic_signed")
    rc = B.lib().bnbq_quantize_blockwise(host.data_ptr(), 256, x.data_ptr(), B.F32, 4096, 2048, absmax.data_ptr(),
                                         out.data_ptr(), None)
    assert rc == B.EINVAL and "device memory" in B.bnbq_last_error()
    rc = B.lib().bnbq_dequantize_blockwise(host.data_ptr(), 256, out.data_ptr(), absmax.data_ptr(), 4096, 2048,
                                           x.data_ptr(), B.F32, None)
    assert rc == B.EINVAL and "device memory" in B.bnbq_last_error()
    torch.cuda.synchronize()
    assert torch.count_nonzero(absmax).item() == 0 and torch.count_nonzero(out).item() == 0

