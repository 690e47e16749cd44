"""CPU-only checks of the C ABI boundary (no kernel runs here).

* the shared library loads and exports every entry point declared in include/bnbq.h;
* its host-side codebooks equal the oracle's and the golden fixtures (independent builds);
* argument checks reject bad input synchronously, before any CUDA call, with a message;
* the launcher policy (which tensors keep 32-bit state) and the workload shapes.
"""
import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest

from block_wise_bit_b200 import bindings as B
from block_wise_bit_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bnbq.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bnbq_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = B.lib()
    declared = _declared()
    assert len(declared) >= 10, declared
    for name in declared:
        assert hasattr(L, name), f"{name} declared in bnbq.h but not exported"
    assert set(declared) == set(B.EXPORTED)
    assert B.bnbq_version() == "0.1.0"


def test_flag_bits_match_the_header():
    """The binding's flag constants and the device code's flag bits are the header's."""
    src = open(HEADER).read()
    defs = {m.group(1): int(m.group(2), 16) for m in re.finditer(r"#define BNBQ_FLAG_([A-Z_]+) (0x[0-9a-fA-F]+)u", src)}
    assert defs == {"BAD_CODE": B.FLAG_BAD_CODE, "NONFINITE": B.FLAG_NONFINITE, "TIMEOUT": B.FLAG_TIMEOUT}
    dev = ""
    for f in ("bnbq_device.cuh", "bnbq_async.cuh"):
        dev += open(os.path.join(ROOT, "block_wise_bit_b200", "csrc", f)).read()
    kdefs = {m.group(1): int(m.group(2), 16) for m in re.finditer(r"constexpr unsigned kFlag(\w+) = (0x[0-9a-fA-F]+)u", dev)}
    assert kdefs == {"BadCode": defs["BAD_CODE"], "NonFinite": defs["NONFINITE"], "Timeout": defs["TIMEOUT"]}


def test_only_bnbq_symbols_exported():
    out = os.popen(f"nm -D --defined-only {B.library_path()}").read().split("\n")
    funcs = [ln.split()[-1] for ln in out if " T " in ln]
    assert funcs and all(f.startswith("bnbq_") for f in funcs), funcs


@pytest.mark.parametrize("kind", ["dynamic_signed", "dynamic_unsigned", "nf4", "fp4", "linear"])
def test_library_codebooks_match_oracle_and_golden(oracle_mod, kind):
    lib_code = B.bnbq_codebook(kind).numpy()
    np.testing.assert_array_equal(lib_code, getattr(oracle_mod, "code_" + kind)())
    path = os.path.join(ROOT, "tests", "golden", f"code_{kind}.hex")
    gold = [float.fromhex(x.strip()) for x in open(path) if x.strip() and not x.startswith("#")]
    np.testing.assert_array_equal(lib_code, np.array(gold, np.float32))
    B.bnbq_check_codebook(B.bnbq_codebook(kind))


def test_check_codebook_rejects():
    import torch
    good = B.bnbq_codebook("dynamic_signed")
    for bad in (good.flip(0), torch.cat([good[:-1], torch.tensor([2.0])]),
                torch.cat([good[:-1], torch.tensor([float("nan")])]), good[:100]):
        with pytest.raises(B.BnbqError) as e:
            B.bnbq_check_codebook(bad)
        assert e.value.status == B.EINVAL and B.bnbq_last_error()


def _q(code=0x1000, K=256, A=0x2000, dt=0, n=100, Bs=2048, am=0x3000, out=0x4000):
    return B.lib().bnbq_quantize_blockwise(code, K, A, dt, n, Bs, am, out, None)


def test_quantize_argument_checks():
    assert _q(code=None) == B.EINVAL
    assert _q(K=17) == B.EINVAL
    assert _q(Bs=1024) == B.EINVAL
    assert _q(n=-1) == B.EINVAL
    assert _q(dt=7) == B.EINVAL
    assert _q(A=None) == B.EINVAL
    assert _q(A=0x2004) == B.EINVAL          # fp32 input must be 16-byte aligned
    assert _q(out=0x4001) == B.EINVAL
    assert _q(K=16, out=0x4001) == B.EINVAL
    assert _q(am=0x3002) == B.EINVAL
    assert "aligned" in B.bnbq_last_error()
    assert _q(n=0, A=None, am=None, out=None) == B.OK  # empty: no-op, no CUDA call


def test_dequantize_argument_checks():
    L = B.lib()
    assert L.bnbq_dequantize_blockwise(0x1000, 256, 0x2000, 0x3000, 10, 100, 0x4000, 0, None) == B.EINVAL
    assert L.bnbq_dequantize_blockwise(0x1000, 256, 0x2002, 0x3000, 10, 256, 0x4000, 0, None) == B.EINVAL
    assert L.bnbq_dequantize_blockwise(0x1000, 16, 0x2002, 0x3000, 10, 256, 0x4008, 0, None) == B.EINVAL
    assert L.bnbq_dequantize_blockwise(0x1000, 256, 0x2000, 0x3000, 10, 256, 0x4000, 5, None) == B.EINVAL
    assert L.bnbq_dequantize_blockwise(0x1000, 256, None, None, 0, 256, None, 0, None) == B.OK


def test_nested_argument_checks():
    """Nested quantization of block scales: checks before any CUDA call."""
    L = B.lib()
    assert L.bnbq_nested_workspace_bytes(0) == 0
    assert L.bnbq_nested_workspace_bytes(1) == 24          # chunk sum, exponent range, counter
    assert L.bnbq_nested_workspace_bytes(4096) == 24 and L.bnbq_nested_workspace_bytes(4097) == 40
    q = L.bnbq_quantize_absmax_nested
    assert q(0x1000, -1, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None) == B.EINVAL
    assert q(0x1000, 10, None, 0x3000, 0x4000, 0x5000, 0x6000, None) == B.EINVAL        # no code2
    assert q(0x1000, 10, 0x2000, 0x3000, 0x4000, 0x5000, None, None) == B.EINVAL        # no workspace
    assert q(0x1004, 10, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, None) == B.EINVAL      # absmax alignment
    assert q(0x1000, 10, 0x2000, 0x3000, 0x4000, 0x5000, 0x6004, None) == B.EINVAL      # workspace alignment
    assert "aligned" in B.bnbq_last_error()
    d = L.bnbq_dequantize_absmax_nested
    assert d(0x1000, 0x2000, 0x3000, 0x4000, -1, 0x5000, None) == B.EINVAL
    assert d(None, None, None, None, 0, None, None) == B.OK                               # empty: no-op
    dn = L.bnbq_dequantize_blockwise_nested
    assert dn(0x1000, 16, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 100, 32, 0x7000, 0, None) == B.EINVAL  # blocksize
    assert dn(0x1000, 16, 0x2000, 0x3000, 0x4000, 0x5000, None, 100, 64, 0x7000, 0, None) == B.EINVAL    # no code2
    assert dn(0x1000, 16, 0x2001, 0x3000, 0x4000, 0x5000, 0x6000, 100, 64, 0x7000, 0, None) == B.EINVAL  # q alignment
    assert dn(0x1000, 16, None, None, None, None, 0x6000, 0, 64, None, 0, None) == B.OK


def _t(**kw):
    d = dict(p=0x10000, g=0x20000, state1=0x30000, state2=0x40000, absmax1=0x50000, absmax2=0x60000, n=5000,
             g_dtype=1, state_bits=8)
    d.update(kw)
    return B.CTensor(**d)


def _step(opt=0, tensors=None, hp=(1e-3, 0.9, 0.999, 1e-8, 0.0), step=1, c1=0x7000, c2=0x8000, Bs=2048):
    tensors = [_t()] if tensors is None else tensors
    arr = (B.CTensor * max(1, len(tensors)))(*tensors)
    h = B.CHParams(*hp)
    return B.lib().bnbq_step_8bit(opt, arr, len(tensors), ctypes.byref(h), step, c1, c2, Bs, None)


def test_step_tensor_count_limits():
    """More than 2^20 tensors, a negative count, or a NULL list: rejected before any CUDA call."""
    h = B.CHParams(1e-3, 0.9, 0.999, 1e-8, 0.0)
    arr = (B.CTensor * 1)(_t())
    L = B.lib()
    assert L.bnbq_step_8bit(0, arr, (1 << 20) + 1, ctypes.byref(h), 1, 0x7000, 0x8000, 2048, None) == B.EINVAL
    assert "2^20" in B.bnbq_last_error()
    assert L.bnbq_step_8bit(0, arr, -1, ctypes.byref(h), 1, 0x7000, 0x8000, 2048, None) == B.EINVAL
    assert L.bnbq_step_8bit(0, None, 3, ctypes.byref(h), 1, 0x7000, 0x8000, 2048, None) == B.EINVAL
    assert L.bnbq_step_8bit(0, None, 0, ctypes.byref(h), 1, 0x7000, 0x8000, 2048, None) == B.OK  # empty list
    assert L.bnbq_step_8bit(4, arr, 1, ctypes.byref(B.CHParams(1e-3, 1.0, 0.0, 1e-8, 0.0)), 1, 0x7000, None,
                            2048, None) == B.EINVAL  # RMSprop alpha must be < 1


def test_step_argument_checks():
    assert _step(opt=9) == B.EINVAL
    assert _step(step=0) == B.EINVAL
    assert _step(Bs=512) == B.EINVAL
    assert _step(hp=(1e-3, 1.0, 0.999, 1e-8, 0.0)) == B.EINVAL   # Adam beta1 must be < 1
    assert _step(hp=(float("nan"), 0.9, 0.999, 1e-8, 0.0)) == B.EINVAL
    assert _step(tensors=[_t(n=-5)]) == B.EINVAL
    assert _step(tensors=[_t(state_bits=16)]) == B.EINVAL
    assert _step(tensors=[_t(g_dtype=3)]) == B.EINVAL
    assert _step(tensors=[_t(p=0x10004)]) == B.EINVAL
    assert _step(tensors=[_t(g=0x20004)]) == B.EINVAL           # bf16 needs 8-byte alignment
    assert _step(tensors=[_t(state1=0x30002)]) == B.EINVAL
    assert _step(tensors=[_t(state_bits=32, state1=0x30008)]) == B.EINVAL
    assert _step(tensors=[_t(absmax2=None)]) == B.EINVAL
    assert _step(tensors=[_t(state2=None)]) == B.EINVAL
    assert _step(c2=None) == B.EINVAL                           # Adam 8-bit needs the unsigned code
    assert "code" in B.bnbq_last_error()
    # empty entries and empty lists are no-ops (no CUDA call)
    assert _step(tensors=[_t(n=0)]) == B.OK
    assert _step(tensors=[]) == B.OK
    # one-state optimizers ignore state2 / absmax2 / code2
    assert _step(opt=2, tensors=[_t(n=-1)]) == B.EINVAL
    h = B.CHParams(1e-3, 0.9, 0.999, 1e-8, 0.0)
    assert B.lib().bnbq_step_8bit(0, None, 3, ctypes.byref(h), 1, 0x7000, 0x8000, 2048, None) == B.EINVAL
    assert B.lib().bnbq_step_8bit(0, None, 0, None, 1, 0x7000, 0x8000, 2048, None) == B.EINVAL


def test_state_policy_and_shapes():
    assert W.state_bits_for(W.ParamSpec("a", 4095)) == 32
    assert W.state_bits_for(W.ParamSpec("a", 4096)) == 8       # "fewer than 4096" is strict
    assert W.state_bits_for(W.ParamSpec("e", 10 ** 8, embedding=True)) == 32
    assert W.state_bits_for(W.ParamSpec("a", 10000), min_8bit_size=16384) == 32
    g = W.gpt2_1p5b()
    assert len(g) == 580 and sum(s.numel for s in g) == 1_557_611_200
    lay = W.Layout.build(g, 2048)
    assert lay.state_bits.count(32) == 291 and lay.n32 == 80_875_200
    assert sum(1 for s, b in zip(g, lay.state_bits) if b == 8 and s.numel % 2048) == 96
    ll = W.llama7b()
    assert len(ll) == 291 and sum(s.numel for s in ll) == 6_738_415_616
    lay = W.Layout.build(ll, 2048)
    assert lay.state_bits.count(32) == 1 and lay.n32 == 131_072_000
    assert lay.n8 == 6_607_343_616 and lay.n_blocks8 == 3_226_242
    assert sum(s.numel for s in W.llama7b_layer()) == 202_383_360
    # every flat offset keeps 16-byte alignment for fp32 and 4-byte alignment for codes
    assert all(o % 4 == 0 for o in lay.off + [x for x in lay.off8 if x >= 0] + [x for x in lay.off32 if x >= 0])


def test_algorithmic_bytes_model():
    """Bytes per step of the 7B AdamW list: 14 B per 8-bit-state param (bf16 grads), 26 B per
    32-bit-state param, 16 B per block of scales."""
    from bench import algorithmic_bytes
    lay = W.Layout.build(W.llama7b(), 2048)
    assert algorithmic_bytes(lay, "adamw", g_bytes=2) == 6_607_343_616 * 14 + 3_226_242 * 16 + 131_072_000 * 26
    assert algorithmic_bytes(lay, "lion", g_bytes=2) == 6_607_343_616 * 12 + 3_226_242 * 8 + 131_072_000 * 18


def test_e2e_slices_cover_the_list_in_order():
    """The end-to-end leg of bench.py steps the list in contiguous, element-balanced slices."""
    from bench import e2e_slices
    lay = W.Layout.build(W.SHAPES["llama7b"](), 2048)
    for k in (1, 2, 4, 7):
        sl = e2e_slices(lay, k)
        assert sl[0][0] == 0 and sl[-1][1] == len(lay.specs) and len(sl) <= k
        assert all(a[1] == b[0] and a[3] <= b[2] for a, b in zip(sl, sl[1:]))
        for i0, i1, a, b in sl:
            assert a == lay.off[i0] and b == lay.off[i1 - 1] + lay.specs[i1 - 1].numel
        sizes = [sum(s.numel for s in lay.specs[i0:i1]) for i0, i1, _, _ in sl]
        assert max(sizes) <= 2 * lay.n_params / k


def test_traffic_record_hash_ignores_comments_only():
    """bench.py keys the committed ncu traffic on a hash of the step kernel's sources with
    comments removed and spaces folded (line breaks kept): editing a comment keeps the key,
    editing code changes it."""
    from bench import _code_only
    src = ('#include "a.h"\n#define N 16 // elements\nint f(int x) { /* twice */ return 2 * x; }\n'
           'const char* s = "a // b /* c */";\nchar c = \'/\';\n')
    same = ('#include "a.h"\n\n// a comment line\n#define N 16   // per thread\nint f(int x) {  return 2 * x; }'
            '\nconst char* s = "a // b /* c */";\nchar c = \'/\';  /* slash */\n')
    assert _code_only(src) == _code_only(same)
    assert _code_only(src) != _code_only(src.replace("2 * x", "3 * x"))
    assert _code_only(src) != _code_only(src.replace("#define N 16 // elements\n", "#define N 16 int\n"))
    assert "a // b /* c */" in _code_only(src)  # string contents are code
    assert _code_only("#define A 1\nint y;") != _code_only("#define A 1 int y;")  # line ends kept


C_CLIENT = r"""
#include <stdio.h>
#include "bnbq.h"

int main(void)
{
    static const bnbq_code_kind kinds[] = {BNBQ_CODE_DYNAMIC_SIGNED, BNBQ_CODE_DYNAMIC_UNSIGNED, BNBQ_CODE_NF4,
                                           BNBQ_CODE_FP4, BNBQ_CODE_LINEAR};
    float code[256];
    printf("%s\n", bnbq_version());
    for (unsigned k = 0; k < sizeof kinds / sizeof kinds[0]; k++) {
        int K = bnbq_code_size(kinds[k]);
        if (bnbq_codebook(kinds[k], code) != K || bnbq_check_codebook(code, K) != BNBQ_OK) return 1;
        for (int j = 0; j < K; j++) printf("%a%c", code[j], j + 1 < K ? ' ' : '\n');
    }
    code[1] = code[0];  /* not strictly increasing */
    if (bnbq_check_codebook(code, 16) != BNBQ_EINVAL || bnbq_last_error()[0] == '\0') return 2;
    return 0;
}
"""


def test_header_is_plain_c_and_links(tmp_path):
    """A C11 program that includes only bnbq.h and links the shared library builds with warnings
    as errors, and its host-side calls give the same codebooks as the Python binding."""
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(B.library_path())
    cuda_lib = "/usr/local/cuda/lib64"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.dirname(HEADER),
                    str(src), "-o", str(exe), "-L", libdir, "-lbnbq", f"-Wl,-rpath,{libdir}:{cuda_lib}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    assert out[0] == B.bnbq_version()
    for line, kind in zip(out[1:6], ["dynamic_signed", "dynamic_unsigned", "nf4", "fp4", "linear"]):
        got = np.array([float.fromhex(t) for t in line.split()], np.float32)
        np.testing.assert_array_equal(got, B.bnbq_codebook(kind).numpy())


def test_bench_reference_arm_prints_the_contract_line():
    """``bench.py --impl reference`` (the oracle timed on the host) prints one JSON line with the
    benchmark's metric, unit and workload, the oracle as cpu_baseline and a host-only e2e."""
    import json
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "3", "--cpu-sample", "65536"], capture_output=True, text=True, check=True,
                         cwd=ROOT, timeout=600).stdout.strip().split("\n")
    line = json.loads(out[-1])
    assert line["impl"] == "reference" and line["unit"] == "params/s" and line["higher_is_better"] is True
    assert line["steps"] == 2 and line["warmup"] == 3 and line["n_gpus"] == 1 and line["value"] > 0
    assert line["config"]["workload"] == "llama7b_adamw8bit" and line["config"]["params"] == 6738415616
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "params/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_gpu_check_programs_build_for_sm100a(tmp_path):
    """The stand-alone GPU check programs under tests/gpu_checks build for sm_100a from the
    library's own device header (compiled here, run only by the -m gpu tests)."""
    from block_wise_bit_b200 import build as BLD
    checks = os.path.join(ROOT, "tests", "gpu_checks")
    for name in sorted(os.listdir(checks)):
        if name.endswith(".cu"):
            subprocess.run([BLD.nvcc()] + BLD.ARCH + ["-O3", "-std=c++17", "--fmad=false", "-c", "-o",
                                                      str(tmp_path / (name + ".o")), os.path.join(checks, name)],
                           check=True)


def test_host_tensors_are_refused_without_fallback():
    """The compute wrappers take CUDA tensors only: host tensors are refused in Python before the
    library is called (there is no CPU path to fall back to), for the standalone calls and the
    optimizer front end alike."""
    import torch
    from block_wise_bit_b200 import optim as O
    code = B.bnbq_codebook("dynamic_signed")
    x = torch.zeros(4096)
    with pytest.raises(TypeError, match="CUDA tensor"):
        B.bnbq_quantize_blockwise(code, x, 2048, absmax=torch.zeros(2), out=torch.zeros(4096, dtype=torch.uint8))
    with pytest.raises(TypeError, match="CUDA tensor"):
        B.bnbq_dequantize_blockwise(code, torch.zeros(4096, dtype=torch.uint8), torch.ones(2), 2048,
                                    out=torch.zeros(4096))
    p = torch.nn.Parameter(torch.zeros(8192))
    p.grad = torch.zeros(8192)
    with pytest.raises((TypeError, RuntimeError, AssertionError)):
        O.AdamW8bit([p], lr=1e-3).step()
    assert torch.equal(p.detach(), torch.zeros(8192))


def test_front_end_keeps_a_step_count_per_parameter(monkeypatch):
    """As in torch.optim, each parameter counts its own steps: a parameter whose first gradient
    arrives later starts its bias correction at step 1, so the front end makes one library call
    per distinct count (recorded here in place of the CUDA call)."""
    import torch
    from block_wise_bit_b200 import optim as O
    calls = []
    monkeypatch.setattr(O.B, "bnbq_step_8bit",
                        lambda kind, entries, step, **kw: calls.append((kind, step, [e.p.numel() for e in entries])))
    p1, p2 = torch.nn.Parameter(torch.zeros(5000)), torch.nn.Parameter(torch.zeros(6000))
    opt = O.AdamW8bit([p1, p2], lr=1e-3)
    p1.grad = torch.ones(5000)
    opt.step()
    p2.grad = torch.ones(6000)
    opt.step()
    opt.step()
    assert calls == [("adamw", 1, [5000]), ("adamw", 2, [5000]), ("adamw", 1, [6000]),
                     ("adamw", 3, [5000]), ("adamw", 2, [6000])]
    assert opt.state[p1]["step"] == 3 and opt.state[p2]["step"] == 2


def test_front_end_refuses_a_group_on_several_devices(monkeypatch):
    import torch
    from block_wise_bit_b200 import optim as O
    monkeypatch.setattr(O.B, "bnbq_step_8bit", lambda *a, **kw: pytest.fail("must not be called"))
    p1 = torch.nn.Parameter(torch.zeros(5000))
    p2 = torch.nn.Parameter(torch.zeros(5000, device="meta"))
    p1.grad = torch.ones(5000)
    p2.grad = torch.ones(5000, device="meta")
    with pytest.raises(ValueError, match="one device"):
        O.AdamW8bit([p1, p2], lr=1e-3).step()


def test_step_codebooks_are_checked_before_the_library_is_called(monkeypatch):
    """The step wrappers pass a codebook to the library only if it is a contiguous float32 CUDA
    tensor of 256 codes on the current device: a host codebook (what bnbq_codebook returns) or a
    16-entry one is refused in Python, so the kernel never reads a host pointer or past the end
    of a short table."""
    import torch
    arr = (B.CTensor * 1)(_t())

    class NoLib:
        def __getattr__(self, name):
            pytest.fail(f"library called ({name})")

    monkeypatch.setattr(B, "lib", lambda *a, **kw: NoLib())
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=1, blocksize=2048)
    for fn in (B.bnbq_step_8bit, B.bnbq_step_8bit_noalloc):
        with pytest.raises(TypeError, match="CUDA tensor"):
            fn("adamw", arr, ntensors=1, code1=torch.zeros(256), code2=torch.zeros(256), **hp)
        with pytest.raises(ValueError, match="256 float32 codes"):
            fn("adamw", arr, ntensors=1, code1=torch.zeros(16), code2=torch.zeros(256), **hp)
        with pytest.raises(ValueError, match="256 float32 codes"):
            fn("adamw", arr, ntensors=1, code1=torch.zeros(256, dtype=torch.float64), code2=torch.zeros(256), **hp)
        with pytest.raises(TypeError, match="torch.Tensor"):
            fn("lion", arr, ntensors=1, code1=[0.0] * 256, code2=None, **hp)
