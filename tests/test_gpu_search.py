"""Exhaustive check of the nearest-code search used by the quantize and step kernels: for each
built-in codebook, every binary32 in [-1, 1] goes through the bucket search in each mode that
applies (including the quantize kernel's FMA-pipe form of the signed search) and is compared with
a plain count of the midpoints below it (tests/gpu_checks/search_exhaustive.cu, built from the
library's own device headers); about a second per codebook on a B200."""
import os
import subprocess

import numpy as np
import pytest
import torch

from block_wise_bit_b200 import bindings as BQ
from block_wise_bit_b200 import build as B

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    exe = tmp_path_factory.mktemp("search") / "search_exhaustive"
    subprocess.run([B.nvcc()] + B.ARCH + ["-O3", "-std=c++17", "--fmad=false", "-o", str(exe),
                                          os.path.join(HERE, "gpu_checks", "search_exhaustive.cu")], check=True)
    return exe


@pytest.mark.parametrize("kind", ["dynamic_signed", "dynamic_unsigned", "nf4", "fp4", "linear"])
def test_search_exhaustive(checker, tmp_path, kind):
    code = BQ.bnbq_codebook(kind).numpy().astype(np.float32)
    f = tmp_path / f"{kind}.f32"
    code.tofile(f)
    out = subprocess.run([str(checker), str(f), str(code.size)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0 and "result ok" in out.stdout, out.stdout + out.stderr
    assert "midpoints equal" in out.stdout and "mode general status no error mismatches 0" in out.stdout
    if code.size == 16:  # the quantize kernel's search for 16 codes
        assert "mode prefix11 status no error mismatches 0" in out.stdout, out.stdout
    if "mode signed status" in out.stdout:  # the quantize kernel's form of the signed search
        assert "mode signed-fma status no error mismatches 0" in out.stdout, out.stdout
