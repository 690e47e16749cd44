"""The bulk-copy helpers behind the staged quantize kernel (tests/gpu_checks/bulk_copy_wait.cu,
built from the library's own bulk-copy header): a 32 KB copy into shared memory completes its
barrier with the right bytes, and a wait on a barrier that nothing arrives on gives up after its
budget (about a second) and returns, the context staying usable."""
import os
import subprocess

import pytest
import torch

from block_wise_bit_b200 import build as B

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_bulk_copy_lands_and_wait_is_bounded(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    exe = tmp_path / "bulk_copy_wait"
    subprocess.run([B.nvcc()] + B.ARCH + ["-O3", "-std=c++17", "-o", str(exe),
                                          os.path.join(HERE, "gpu_checks", "bulk_copy_wait.cu")], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and "result ok" in out.stdout, out.stdout + out.stderr
    assert "copy landed 128 of 128 waits, bytes equal" in out.stdout
    assert "wait gave up 32 of 32" in out.stdout
