"""ctypes binding of include/bnbq.h (libbnbq.so, built for sm_100a).

Argument marshalling only: every step of quantization, dequantization and the optimizer step
runs in the CUDA kernels of the library.  torch supplies device memory and the current stream.
There is no fallback: if the library is missing or the tensors are not on a CUDA device, the
calls raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

from . import build as _build

OK, EINVAL, EUNSUPPORTED, ECUDA = 0, 1, 2, 3
F32, BF16 = 0, 1
ADAMW, ADAM, LION, MOMENTUM, RMSPROP = 0, 1, 2, 3, 4
OPTIMS = {"adamw": ADAMW, "adam": ADAM, "lion": LION, "momentum": MOMENTUM, "rmsprop": RMSPROP}
CODE_DYNAMIC_SIGNED, CODE_DYNAMIC_UNSIGNED, CODE_NF4, CODE_LINEAR, CODE_FP4 = 0, 1, 2, 3, 4
CODE_KINDS = {"dynamic_signed": CODE_DYNAMIC_SIGNED, "dynamic_unsigned": CODE_DYNAMIC_UNSIGNED,
              "nf4": CODE_NF4, "linear": CODE_LINEAR, "fp4": CODE_FP4}
FLAG_BAD_CODE, FLAG_NONFINITE, FLAG_TIMEOUT = 0x1, 0x2, 0x4

EXPORTED = ["bnbq_quantize_blockwise", "bnbq_dequantize_blockwise", "bnbq_step_8bit", "bnbq_step_8bit_noalloc",
            "bnbq_nested_workspace_bytes", "bnbq_quantize_absmax_nested", "bnbq_dequantize_absmax_nested",
            "bnbq_dequantize_blockwise_nested", "bnbq_codebook",
            "bnbq_code_size", "bnbq_check_codebook", "bnbq_device_flags", "bnbq_last_error", "bnbq_release",
            "bnbq_version"]


class BnbqError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"bnbq status {status}: {msg}")
        self.status = status


class CTensor(ctypes.Structure):
    """bnbq_tensor"""
    _fields_ = [("p", ctypes.c_void_p), ("g", ctypes.c_void_p), ("state1", ctypes.c_void_p),
                ("state2", ctypes.c_void_p), ("absmax1", ctypes.c_void_p), ("absmax2", ctypes.c_void_p),
                ("n", ctypes.c_int64), ("g_dtype", ctypes.c_int32), ("state_bits", ctypes.c_int32)]


class CHParams(ctypes.Structure):
    """bnbq_hparams"""
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float)]


_lib = None


def library_path() -> str:
    return _build.LIB


def lib(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libbnbq.so (building it with nvcc first if it is missing or stale and nvcc exists).
    The environment variable BNBQ_LIBRARY names another build of the same library to load."""
    global _lib
    if _lib is None:
        path = os.environ.get("BNBQ_LIBRARY") or _build.LIB
        if build_if_missing and not os.environ.get("BNBQ_LIBRARY"):
            try:
                path = _build.build()
            except RuntimeError:
                if not os.path.exists(path):
                    raise
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library {path} is not built (python -m block_wise_bit_b200.build)")
        L = ctypes.CDLL(path)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.bnbq_quantize_blockwise.argtypes = [vp, i32, vp, i32, i64, i32, vp, vp, vp]
        L.bnbq_dequantize_blockwise.argtypes = [vp, i32, vp, vp, i64, i32, vp, i32, vp]
        L.bnbq_step_8bit.argtypes = [i32, ctypes.POINTER(CTensor), i32, ctypes.POINTER(CHParams), i32, vp, vp,
                                     i32, vp]
        L.bnbq_step_8bit_noalloc.argtypes = L.bnbq_step_8bit.argtypes
        L.bnbq_step_8bit_noalloc.restype = i32
        L.bnbq_nested_workspace_bytes.argtypes = [i64]
        L.bnbq_nested_workspace_bytes.restype = i64
        L.bnbq_quantize_absmax_nested.argtypes = [vp, i64, vp, vp, vp, vp, vp, vp]
        L.bnbq_quantize_absmax_nested.restype = i32
        L.bnbq_dequantize_absmax_nested.argtypes = [vp, vp, vp, vp, i64, vp, vp]
        L.bnbq_dequantize_absmax_nested.restype = i32
        L.bnbq_dequantize_blockwise_nested.argtypes = [vp, i32, vp, vp, vp, vp, vp, i64, i32, vp, i32, vp]
        L.bnbq_dequantize_blockwise_nested.restype = i32
        for f in ("bnbq_quantize_blockwise", "bnbq_dequantize_blockwise", "bnbq_step_8bit",
                  "bnbq_check_codebook", "bnbq_device_flags"):
            getattr(L, f).restype = i32
        L.bnbq_codebook.argtypes = [i32, vp]
        L.bnbq_codebook.restype = i32
        L.bnbq_code_size.argtypes = [i32]
        L.bnbq_code_size.restype = i32
        L.bnbq_check_codebook.argtypes = [vp, i32]
        L.bnbq_device_flags.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
        L.bnbq_last_error.restype = ctypes.c_char_p
        L.bnbq_last_error.argtypes = []
        L.bnbq_release.restype = None
        L.bnbq_release.argtypes = []
        L.bnbq_version.restype = ctypes.c_char_p
        L.bnbq_version.argtypes = []
        _lib = L
    return _lib


def _check(status: int):
    if status != OK:
        raise BnbqError(status, lib().bnbq_last_error().decode())


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_id(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _dev(t: torch.Tensor, name: str, device: Optional[int] = None) -> int:
    """Device pointer of ``t``, which must be a contiguous CUDA tensor on the current device (the
    library launches on the current device; ``device`` passes it in when already known)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    cur = torch.cuda.current_device() if device is None else device
    if t.device.index != cur:
        raise ValueError(f"{name} is on {t.device} but the current device is cuda:{cur}; "
                         f"call inside torch.cuda.device({t.device.index})")
    return t.data_ptr()


def _step_code(code: Optional[torch.Tensor], name: str, device: Optional[int]) -> Optional[int]:
    """Device pointer of a step codebook: None stays None; otherwise a contiguous float32 CUDA
    tensor of exactly 256 values on the current device (the kernel reads 256 codes)."""
    if code is None:
        return None
    if not isinstance(code, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if code.dtype != torch.float32 or code.numel() != 256:
        raise ValueError(f"{name} must hold 256 float32 codes (got {code.numel()} values of {code.dtype})")
    return _dev(code, name, device)


# ------------------------------------------------------------------------------------ codebooks
def bnbq_codebook(kind: str | int) -> torch.Tensor:
    """Host-side construction of a codebook (CPU float32 tensor)."""
    k = CODE_KINDS[kind] if isinstance(kind, str) else int(kind)
    size = lib().bnbq_code_size(k)
    if size < 0:
        raise ValueError(f"unknown codebook kind {kind}")
    out = torch.empty(size, dtype=torch.float32)
    if lib().bnbq_codebook(k, ctypes.c_void_p(out.data_ptr())) != size:
        raise ValueError(f"codebook {kind} failed")
    return out


def bnbq_check_codebook(code: torch.Tensor) -> None:
    c = code.detach().to("cpu", torch.float32).contiguous()
    _check(lib().bnbq_check_codebook(ctypes.c_void_p(c.data_ptr()), c.numel()))


# --------------------------------------------------------------------------- quantize / dequant
def bnbq_quantize_blockwise(code: torch.Tensor, A: torch.Tensor, blocksize: int = 2048,
                            absmax: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                            stream=None):
    """Return (absmax float32[ceil(n/B)], codes uint8[n] or packed uint8[ceil(n/2)] for 16 codes)."""
    n = A.numel()
    K = code.numel()
    nb = (n + blocksize - 1) // blocksize
    if absmax is None:
        absmax = torch.empty(nb, dtype=torch.float32, device=A.device)
    if out is None:
        out = torch.empty(n if K == 256 else (n + 1) // 2, dtype=torch.uint8, device=A.device)
    _check(lib().bnbq_quantize_blockwise(_dev(code, "code"), K, _dev(A, "A") if n else None, _dtype_id(A), n,
                                         blocksize, _dev(absmax, "absmax") if n else None,
                                         _dev(out, "out") if n else None, _stream(stream)))
    return absmax, out


def bnbq_dequantize_blockwise(code: torch.Tensor, q: torch.Tensor, absmax: torch.Tensor, n: int,
                              blocksize: int = 2048, out_dtype=torch.float32,
                              out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(n, dtype=out_dtype, device=q.device)
    _check(lib().bnbq_dequantize_blockwise(_dev(code, "code"), code.numel(), _dev(q, "q") if n else None,
                                           _dev(absmax, "absmax") if n else None, n, blocksize,
                                           _dev(out, "out") if n else None, _dtype_id(out), _stream(stream)))
    return out


# ------------------------------------------------------------------------- nested block scales
NEST_BLOCK = 256


def bnbq_quantize_absmax_nested(code2: torch.Tensor, absmax: torch.Tensor, stream=None,
                                qabs: Optional[torch.Tensor] = None, absmax2: Optional[torch.Tensor] = None,
                                offset: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """Nested quantization of a block-scale array: returns (qabs uint8[nb], absmax2 float32
    [ceil(nb/256)], offset float32[1]), all on absmax's device.  Outputs and the workspace
    (``bnbq_nested_workspace_bytes(nb)`` bytes) may be passed in to reuse them; missing ones are
    torch allocations made here."""
    nb = absmax.numel()
    dev = absmax.device
    if qabs is None:
        qabs = torch.empty(nb, dtype=torch.uint8, device=dev)
    if absmax2 is None:
        absmax2 = torch.empty((nb + NEST_BLOCK - 1) // NEST_BLOCK, dtype=torch.float32, device=dev)
    if offset is None:
        offset = torch.empty(1, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(1, lib().bnbq_nested_workspace_bytes(nb)), dtype=torch.uint8, device=dev)
    _check(lib().bnbq_quantize_absmax_nested(_dev(absmax, "absmax") if nb else None, nb, _dev(code2, "code2"),
                                             _dev(qabs, "qabs") if nb else None,
                                             _dev(absmax2, "absmax2") if nb else None, _dev(offset, "offset"),
                                             _dev(workspace, "workspace"), _stream(stream)))
    return qabs, absmax2, offset


def bnbq_dequantize_absmax_nested(code2: torch.Tensor, qabs: torch.Tensor, absmax2: torch.Tensor,
                                  offset: torch.Tensor, stream=None) -> torch.Tensor:
    nb = qabs.numel()
    out = torch.empty(nb, dtype=torch.float32, device=qabs.device)
    if nb:
        _check(lib().bnbq_dequantize_absmax_nested(_dev(qabs, "qabs"), _dev(absmax2, "absmax2"),
                                                   _dev(offset, "offset"), _dev(code2, "code2"), nb,
                                                   _dev(out, "absmax_out"), _stream(stream)))
    return out


def bnbq_dequantize_blockwise_nested(code: torch.Tensor, q: torch.Tensor, qabs: torch.Tensor, absmax2: torch.Tensor,
                                     offset: torch.Tensor, code2: torch.Tensor, n: int, blocksize: int = 64,
                                     out_dtype=torch.float32, out: Optional[torch.Tensor] = None,
                                     stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(n, dtype=out_dtype, device=q.device)
    _check(lib().bnbq_dequantize_blockwise_nested(_dev(code, "code"), code.numel(), _dev(q, "q") if n else None,
                                                  _dev(qabs, "qabs") if n else None,
                                                  _dev(absmax2, "absmax2") if n else None,
                                                  _dev(offset, "offset") if n else None, _dev(code2, "code2"), n,
                                                  blocksize, _dev(out, "out") if n else None, _dtype_id(out),
                                                  _stream(stream)))
    return out


# ------------------------------------------------------------------------------- optimizer step
@dataclass
class TensorState:
    """One parameter tensor and its optimizer state (device tensors, contiguous)."""
    p: torch.Tensor                   # float32
    g: torch.Tensor                   # float32 or bfloat16
    state1: torch.Tensor              # uint8 (8-bit) or float32 (32-bit)
    state2: Optional[torch.Tensor] = None
    absmax1: Optional[torch.Tensor] = None
    absmax2: Optional[torch.Tensor] = None

    @property
    def state_bits(self) -> int:
        return 8 if self.state1.dtype == torch.uint8 else 32


def pack_tensor_list(tensors: Sequence[TensorState]):
    arr = (CTensor * max(1, len(tensors)))()
    cur = None  # the current device, looked up once the first tensor is known to be on CUDA
    for i, t in enumerate(tensors):
        if t.p.dtype != torch.float32:
            raise TypeError("parameters must be float32")
        c = arr[i]
        c.p = _dev(t.p, "p", cur)
        if cur is None:
            cur = t.p.device.index
        c.g = _dev(t.g, "g", cur)
        c.state1 = _dev(t.state1, "state1", cur)
        c.state2 = _dev(t.state2, "state2", cur) if t.state2 is not None else None
        c.absmax1 = _dev(t.absmax1, "absmax1", cur) if t.absmax1 is not None else None
        c.absmax2 = _dev(t.absmax2, "absmax2", cur) if t.absmax2 is not None else None
        c.n = t.p.numel()
        c.g_dtype = _dtype_id(t.g)
        c.state_bits = t.state_bits
    return arr


def bnbq_step_8bit(opt: str | int, tensors: Sequence[TensorState] | ctypes.Array, *, lr: float, beta1: float,
                   beta2: float, eps: float, weight_decay: float, step: int,
                   code1: Optional[torch.Tensor], code2: Optional[torch.Tensor], blocksize: int = 2048,
                   stream=None, ntensors: Optional[int] = None) -> None:
    """One fused optimizer step over the list (one kernel launch).  ``tensors`` may be a list of
    TensorState or an array already packed by ``pack_tensor_list`` (then give ``ntensors``)."""
    o = OPTIMS[opt] if isinstance(opt, str) else int(opt)
    if isinstance(tensors, ctypes.Array):
        arr, nt = tensors, ntensors
    else:
        arr, nt = pack_tensor_list(tensors), len(tensors)
    hp = CHParams(lr, beta1, beta2, eps, weight_decay)
    c1, c2 = _step_code(code1, "code1", None), _step_code(code2, "code2", None)
    _check(lib().bnbq_step_8bit(o, arr, nt, ctypes.byref(hp), step, c1, c2, blocksize, _stream(stream)))


def bnbq_step_8bit_noalloc(opt: str | int, tensors: Sequence[TensorState] | ctypes.Array, *, lr: float,
                           beta1: float, beta2: float, eps: float, weight_decay: float, step: int,
                           code1: Optional[torch.Tensor], code2: Optional[torch.Tensor], blocksize: int = 2048,
                           stream=None, ntensors: Optional[int] = None) -> None:
    """The same step as ``bnbq_step_8bit`` without any device allocation by the library (for
    callers whose device memory all belongs to their own pool, or that must not allocate between
    steps): the descriptor table lives in a fixed array inside the library (at most 4096
    non-empty tensors per call).  All calls on a device share that array, so calls that can
    overlap on the GPU must be ordered.  Like ``bnbq_step_8bit`` it refuses a stream that is
    being captured into a CUDA graph."""
    o = OPTIMS[opt] if isinstance(opt, str) else int(opt)
    if isinstance(tensors, ctypes.Array):
        arr, nt = tensors, ntensors
    else:
        arr, nt = pack_tensor_list(tensors), len(tensors)
    hp = CHParams(lr, beta1, beta2, eps, weight_decay)
    c1, c2 = _step_code(code1, "code1", None), _step_code(code2, "code2", None)
    _check(lib().bnbq_step_8bit_noalloc(o, arr, nt, ctypes.byref(hp), step, c1, c2, blocksize, _stream(stream)))


def bnbq_device_flags(clear: bool = False) -> int:
    """The calling device's flag word (synchronizes the device): FLAG_BAD_CODE (a codebook failed
    the device-side check), FLAG_NONFINITE (a block scale came out NaN or Inf), FLAG_TIMEOUT (a
    kernel's bounded wait for its own bulk copy ran out); ``clear`` resets it."""
    v = ctypes.c_uint32(0)
    _check(lib().bnbq_device_flags(ctypes.byref(v), int(clear)))
    return int(v.value)


def bnbq_release() -> None:
    lib().bnbq_release()


def bnbq_version() -> str:
    return lib().bnbq_version().decode()


def bnbq_last_error() -> str:
    return lib().bnbq_last_error().decode()
