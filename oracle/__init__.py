"""CPU oracle for block-wise dynamic quantization and the 8-bit optimizer step.

TEST INFRASTRUCTURE, NOT PART OF THE LIBRARY.  Only the test suite, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference legs may import this package.  It wraps the plain C
restatement in ``bnbq_oracle.c`` (see that file and ``bnbq_oracle.h`` for the sources it
follows) through ctypes on numpy arrays.  It shares no code with ``block_wise_bit_b200``.

The shared object is compiled with gcc on first use (or by ``build()``) with
``-ffp-contract=off`` so that every binary32 operation is rounded on its own.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bnbq_oracle.c")
_HDR = os.path.join(_HERE, "bnbq_oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

ADAMW, ADAM, LION, MOMENTUM, RMSPROP = 0, 1, 2, 3, 4
F32, BF16 = 0, 1
OPTIMS = {"adamw": ADAMW, "adam": ADAM, "lion": LION, "momentum": MOMENTUM, "rmsprop": RMSPROP}

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, plain -O2, no FMA contraction)."""
    stale = (not os.path.exists(_LIB)) or max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)) > os.path.getmtime(_LIB)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


class _HP(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float)]


def _declare(L):
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    for name in ("oracle_code_dynamic_unsigned", "oracle_code_dynamic_signed",
                 "oracle_code_nf4", "oracle_code_fp4", "oracle_code_linear"):
        getattr(L, name).argtypes = [vp]
        getattr(L, name).restype = None
    L.oracle_code_mid.argtypes = [vp, i32]
    L.oracle_code_mid.restype = ctypes.c_float
    L.oracle_nearest_code.argtypes = [vp, i32, ctypes.c_float]
    L.oracle_nearest_code.restype = i32
    L.oracle_quantize_blockwise.argtypes = [vp, i32, vp, i32, i64, i32, vp, vp]
    L.oracle_quantize_blockwise.restype = i32
    L.oracle_dequantize_blockwise.argtypes = [vp, i32, vp, vp, i64, i32, vp, i32]
    L.oracle_dequantize_blockwise.restype = i32
    L.oracle_step_blocks.argtypes = [i32, i32, vp, vp, i32, i64, vp, vp, vp, vp, vp, vp, i32,
                                     ctypes.POINTER(_HP), i32, i64, i64]
    L.oracle_step_blocks.restype = i32
    L.oracle_absmax_mean.argtypes = [vp, i64]
    L.oracle_absmax_mean.restype = ctypes.c_float
    L.oracle_nest_absmax.argtypes = [vp, i64, vp, vp, vp, vp]
    L.oracle_nest_absmax.restype = i32
    L.oracle_unnest_absmax.argtypes = [vp, vp, ctypes.c_float, vp, i64, vp]
    L.oracle_unnest_absmax.restype = i32
    return L


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _declare(ctypes.CDLL(_LIB))
    return _lib


def swap_library(path):
    """Test hook: load another build of this oracle's source (the mutation tests plant a mistake
    in a copy of it) in place of the real one; returns the previous library handle, which
    ``restore_library`` puts back."""
    global _lib
    with _lock:
        prev = _lib
        _lib = _declare(ctypes.CDLL(path))
    return prev


def restore_library(prev):
    global _lib
    with _lock:
        _lib = prev


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.float32, a.dtype
    return a


# ---------------------------------------------------------------- codebooks
def code_dynamic_unsigned() -> np.ndarray:
    out = np.zeros(256, np.float32)
    lib().oracle_code_dynamic_unsigned(_ptr(out))
    return out


def code_dynamic_signed() -> np.ndarray:
    out = np.zeros(256, np.float32)
    lib().oracle_code_dynamic_signed(_ptr(out))
    return out


def code_nf4() -> np.ndarray:
    out = np.zeros(16, np.float32)
    lib().oracle_code_nf4(_ptr(out))
    return out


def code_fp4() -> np.ndarray:
    out = np.zeros(16, np.float32)
    lib().oracle_code_fp4(_ptr(out))
    return out


def code_linear() -> np.ndarray:
    out = np.zeros(256, np.float32)
    lib().oracle_code_linear(_ptr(out))
    return out


def code_mid(code: np.ndarray, j: int) -> np.float32:
    code = _f32(code)
    return np.float32(lib().oracle_code_mid(_ptr(code), j))


def nearest_code(code: np.ndarray, xn: float) -> int:
    code = _f32(code)
    return int(lib().oracle_nearest_code(_ptr(code), len(code), ctypes.c_float(xn)))


# ---------------------------------------------------------------- quantize / dequantize
def _dtype_id(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:  # bf16 bit patterns
        return BF16
    raise TypeError(f"oracle takes float32 or uint16 (bf16 bits), got {a.dtype}")


def quantize_blockwise(code: np.ndarray, x: np.ndarray, blocksize: int):
    """Return (absmax float32[ceil(n/B)], q uint8[n] or packed uint8[ceil(n/2)] for K == 16).

    ``x`` is float32, or uint16 holding bf16 bit patterns."""
    code = _f32(code)
    x = np.ascontiguousarray(x).reshape(-1)
    n = x.size
    nb = (n + blocksize - 1) // blocksize
    absmax = np.zeros(nb, np.float32)
    out = np.zeros(n if len(code) == 256 else (n + 1) // 2, np.uint8)
    rc = lib().oracle_quantize_blockwise(_ptr(code), len(code), _ptr(x), _dtype_id(x), n, blocksize,
                                         _ptr(absmax), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_quantize_blockwise rejected its arguments")
    return absmax, out


def dequantize_blockwise(code: np.ndarray, q: np.ndarray, absmax: np.ndarray, n: int, blocksize: int,
                         out_bf16: bool = False) -> np.ndarray:
    """Return float32[n] (or uint16 bf16 bits[n] when ``out_bf16``)."""
    code = _f32(code)
    q = np.ascontiguousarray(q, dtype=np.uint8)
    absmax = _f32(absmax)
    y = np.zeros(n, np.uint16 if out_bf16 else np.float32)
    rc = lib().oracle_dequantize_blockwise(_ptr(code), len(code), _ptr(q), _ptr(absmax), n, blocksize,
                                           _ptr(y), BF16 if out_bf16 else F32)
    if rc != 0:
        raise ValueError("oracle_dequantize_blockwise rejected its arguments")
    return y


# ---------------------------------------------------------------- nested quantization of scales
NEST_B = 256
NEST_CHUNK = 4096


def absmax_mean(absmax: np.ndarray) -> np.float32:
    absmax = _f32(absmax)
    return np.float32(lib().oracle_absmax_mean(_ptr(absmax), absmax.size))


def nest_absmax(absmax: np.ndarray, code2: np.ndarray):
    """Return (qabs uint8[nb], absmax2 float32[ceil(nb/256)], offset float32)."""
    absmax = _f32(absmax)
    code2 = _f32(code2)
    nb = absmax.size
    qabs = np.zeros(nb, np.uint8)
    absmax2 = np.zeros((nb + NEST_B - 1) // NEST_B, np.float32)
    off = np.zeros(1, np.float32)
    rc = lib().oracle_nest_absmax(_ptr(absmax), nb, _ptr(code2), _ptr(qabs), _ptr(absmax2), _ptr(off))
    if rc != 0:
        raise ValueError("oracle_nest_absmax rejected its arguments")
    return qabs, absmax2, np.float32(off[0])


def unnest_absmax(qabs: np.ndarray, absmax2: np.ndarray, offset, code2: np.ndarray) -> np.ndarray:
    qabs = np.ascontiguousarray(qabs, dtype=np.uint8)
    absmax2 = _f32(absmax2)
    code2 = _f32(code2)
    out = np.zeros(qabs.size, np.float32)
    rc = lib().oracle_unnest_absmax(_ptr(qabs), _ptr(absmax2), ctypes.c_float(float(offset)), _ptr(code2),
                                    qabs.size, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_unnest_absmax rejected its arguments")
    return out


def dequantize_blockwise_nested(code: np.ndarray, q: np.ndarray, qabs: np.ndarray, absmax2: np.ndarray, offset,
                                code2: np.ndarray, n: int, blocksize: int, out_bf16: bool = False) -> np.ndarray:
    """Dequantize with block scales rebuilt from their nested quantization."""
    return dequantize_blockwise(code, q, unnest_absmax(qabs, absmax2, offset, code2), n, blocksize, out_bf16)


# ---------------------------------------------------------------- optimizer step
def step_tensor(optim: str | int, p: np.ndarray, g: np.ndarray, s1: np.ndarray, s2: np.ndarray | None,
                absmax1: np.ndarray | None, absmax2: np.ndarray | None, code1: np.ndarray | None,
                code2: np.ndarray | None, blocksize: int, *, lr: float, beta1: float, beta2: float,
                eps: float, weight_decay: float, step: int, block_range: tuple[int, int] | None = None):
    """In-place oracle step on one tensor.  State is uint8 (8-bit) or float32 (32-bit);
    ``g`` is float32 or uint16 bf16 bits.  All arrays must be C-contiguous numpy arrays and
    are modified in place (p, s1, s2, absmax1, absmax2)."""
    opt = OPTIMS[optim] if isinstance(optim, str) else int(optim)
    bits = 8 if s1.dtype == np.uint8 else 32
    for a in (p, g, s1, s2, absmax1, absmax2):
        if a is not None and not a.flags["C_CONTIGUOUS"]:
            raise ValueError("oracle step needs C-contiguous arrays")
    assert p.dtype == np.float32
    n = p.size
    nb = (n + blocksize - 1) // blocksize
    b0, b1 = (0, nb) if block_range is None else block_range
    hp = _HP(lr, beta1, beta2, eps, weight_decay)
    rc = lib().oracle_step_blocks(opt, bits, _ptr(p), _ptr(g), _dtype_id(g), n, _ptr(s1), _ptr(s2),
                                  _ptr(absmax1), _ptr(absmax2),
                                  _ptr(None if code1 is None else _f32(code1)),
                                  _ptr(None if code2 is None else _f32(code2)),
                                  blocksize, ctypes.byref(hp), step, b0, b1)
    if rc != 0:
        raise ValueError("oracle_step_blocks rejected its arguments")


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
