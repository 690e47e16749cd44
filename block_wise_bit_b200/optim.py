"""Host-side launcher policy and optimizer front ends over ``bnbq_step_8bit``.

The pages present the 8-bit optimizers as drop-in replacements for torch.optim classes
(``bnb.optim.AdamW8bit(params, lr, betas, eps)``; page "bitsandbytes - Quantização de LLM",
section "Workflow 3"; page "Py之bitsandbytes…详细攻略", section "使用8位优化器"), with tensors of
fewer than ``min_8bit_size`` (default 4096) elements keeping 32-bit state, and per-parameter
32-bit overrides for unstable parameters such as embeddings (same page, sections
"如果需要高精度的参数" and "更改单个参数的位数和其他超参数").

This module only decides which tensors are 8-bit, allocates their state, and packs the tensor
list; each ``step()`` is one call of the CUDA library per parameter group.
"""
from __future__ import annotations

import contextlib
from typing import Dict, List, Optional

import torch

from . import bindings as B

_CODE_CACHE: Dict[tuple, torch.Tensor] = {}


def device_codebook(kind: str, device) -> torch.Tensor:
    """Codebook ``kind`` as a float32 tensor on ``device`` (built once per device)."""
    key = (kind, str(torch.device(device)))
    if key not in _CODE_CACHE:
        _CODE_CACHE[key] = B.bnbq_codebook(kind).to(device)
    return _CODE_CACHE[key]


def zero_state_index(code: torch.Tensor) -> int:
    """Index of the code nearest 0 (lowest on a tie): the code a zero state is stored as."""
    return int(torch.argmin(code.detach().cpu().abs()).item())


def new_state(p: torch.Tensor, two_states: bool, state_bits: int, blocksize: int, code1: torch.Tensor,
              code2: Optional[torch.Tensor]) -> dict:
    """Zero optimizer state for parameter p: 8-bit codes + block scales, or fp32 moments."""
    n = p.numel()
    st = {}
    if state_bits == 8:
        nb = (n + blocksize - 1) // blocksize
        st["state1"] = torch.full((n,), zero_state_index(code1), dtype=torch.uint8, device=p.device)
        st["absmax1"] = torch.zeros(nb, dtype=torch.float32, device=p.device)
        if two_states:
            st["state2"] = torch.full((n,), zero_state_index(code2), dtype=torch.uint8, device=p.device)
            st["absmax2"] = torch.zeros(nb, dtype=torch.float32, device=p.device)
    else:
        st["state1"] = torch.zeros(n, dtype=torch.float32, device=p.device)
        if two_states:
            st["state2"] = torch.zeros(n, dtype=torch.float32, device=p.device)
    return st


class Optimizer8bit(torch.optim.Optimizer):
    """torch.optim-style optimizer whose state is kept 8-bit block-wise (see module docstring)."""

    _KIND = "adamw"

    def __init__(self, params, lr: float, betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 0.0,
                 min_8bit_size: int = 4096, blocksize: int = 2048, optim_bits: int = 8):
        if optim_bits not in (8, 32):
            raise ValueError("optim_bits must be 8 or 32")
        defaults = dict(lr=lr, betas=tuple(betas), eps=eps, weight_decay=weight_decay)
        super().__init__(params, defaults)
        self.min_8bit_size = min_8bit_size
        self.blocksize = blocksize
        self.optim_bits = optim_bits
        self._force32: set = set()

    @property
    def two_states(self) -> bool:
        return self._KIND in ("adamw", "adam")

    @property
    def code1_kind(self) -> str:
        """Codebook of the first state: signed, except RMSprop's non-negative mean of squares."""
        return "dynamic_unsigned" if self._KIND == "rmsprop" else "dynamic_signed"

    def override_32bit(self, param: torch.Tensor) -> None:
        """Keep ``param``'s state in 32 bits (e.g. an embedding table)."""
        self._force32.add(id(param))

    def state_bits_for(self, p: torch.Tensor) -> int:
        if self.optim_bits == 32 or id(p) in self._force32 or p.numel() < self.min_8bit_size:
            return 32
        return 8

    @torch.no_grad()
    def step(self, closure=None):
        loss = None
        if closure is not None:
            with torch.enable_grad():
                loss = closure()
        for group in self.param_groups:
            params = [p for p in group["params"] if p.grad is not None]
            if not params:
                continue
            dev = params[0].device
            if any(p.device != dev for p in params):
                raise ValueError("the parameters of one group must be on one device")
            code1 = device_codebook(self.code1_kind, dev)
            code2 = device_codebook("dynamic_unsigned", dev) if self.two_states else None
            # Each parameter keeps its own step count, as in torch.optim (a parameter whose first
            # gradient comes later starts its bias correction at 1); one call per distinct count.
            by_step: Dict[int, List[B.TensorState]] = {}
            for p in params:
                if p.dtype != torch.float32 or not p.is_contiguous():
                    raise TypeError("8-bit optimizers here step contiguous float32 parameters")
                st = self.state[p]
                if not st:
                    st.update(new_state(p, self.two_states, self.state_bits_for(p), self.blocksize, code1, code2))
                    st["step"] = 0
                st["step"] += 1
                g = p.grad if p.grad.is_contiguous() else p.grad.contiguous()
                by_step.setdefault(st["step"], []).append(
                    B.TensorState(p.view(-1), g.view(-1), st["state1"], st.get("state2"), st.get("absmax1"),
                                  st.get("absmax2")))
            b1, b2 = group["betas"]
            with torch.cuda.device(dev) if dev.type == "cuda" else contextlib.nullcontext():
                for t, entries in by_step.items():
                    B.bnbq_step_8bit(self._KIND, entries, lr=group["lr"], beta1=b1, beta2=b2, eps=group["eps"],
                                     weight_decay=group["weight_decay"], step=t, code1=code1, code2=code2,
                                     blocksize=self.blocksize)
        return loss


class AdamW8bit(Optimizer8bit):
    _KIND = "adamw"

    def __init__(self, params, lr=1e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=1e-2, **kw):
        super().__init__(params, lr, betas, eps, weight_decay, **kw)


class Adam8bit(Optimizer8bit):
    _KIND = "adam"

    def __init__(self, params, lr=1e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0, **kw):
        super().__init__(params, lr, betas, eps, weight_decay, **kw)


class Lion8bit(Optimizer8bit):
    _KIND = "lion"

    def __init__(self, params, lr=1e-4, betas=(0.9, 0.99), weight_decay=0.0, **kw):
        super().__init__(params, lr, betas, 0.0, weight_decay, **kw)


class SGD8bit(Optimizer8bit):
    """SGD with momentum (dampening 0); ``momentum`` is passed to the kernel as beta1."""
    _KIND = "momentum"

    def __init__(self, params, lr, momentum=0.9, weight_decay=0.0, **kw):
        super().__init__(params, lr, (momentum, 0.0), 0.0, weight_decay, **kw)


class RMSprop8bit(Optimizer8bit):
    """RMSprop without momentum (torch.optim.RMSprop's default form); ``alpha`` is passed to the
    kernel as beta1 and the one state uses the unsigned dynamic code."""
    _KIND = "rmsprop"

    def __init__(self, params, lr=1e-2, alpha=0.99, eps=1e-8, weight_decay=0.0, **kw):
        super().__init__(params, lr, (alpha, 0.0), eps, weight_decay, **kw)


class FlatStateList:
    """A whole parameter list laid out in flat device buffers (see ``workloads.Layout``), with
    its 8-bit / 32-bit state and the tensor list packed once for repeated steps."""

    def __init__(self, layout, optim: str, device, g_dtype=torch.bfloat16):
        self.layout = layout
        self.optim = optim
        self.two = optim in ("adamw", "adam")
        self.device = torch.device(device)
        self.code1 = device_codebook("dynamic_unsigned" if optim == "rmsprop" else "dynamic_signed", self.device)
        self.code2 = device_codebook("dynamic_unsigned", self.device) if self.two else None
        lay = layout
        self.p = torch.empty(lay.total, dtype=torch.float32, device=self.device)
        self.g = torch.empty(lay.total, dtype=g_dtype, device=self.device)
        self.q1 = torch.full((lay.total8,), zero_state_index(self.code1), dtype=torch.uint8, device=self.device)
        self.q2 = (torch.full((lay.total8,), zero_state_index(self.code2), dtype=torch.uint8, device=self.device)
                   if self.two else None)
        self.a1 = torch.zeros(lay.totala, dtype=torch.float32, device=self.device)
        self.a2 = torch.zeros(lay.totala, dtype=torch.float32, device=self.device) if self.two else None
        self.m32 = torch.zeros(lay.total32, dtype=torch.float32, device=self.device)
        self.v32 = torch.zeros(lay.total32, dtype=torch.float32, device=self.device) if self.two else None
        self.entries = [self.entry(i) for i in range(len(lay.specs))]
        self.packed = B.pack_tensor_list(self.entries)

    def entry(self, i: int) -> B.TensorState:
        lay = self.layout
        n = lay.specs[i].numel
        o = lay.off[i]
        p, g = self.p[o:o + n], self.g[o:o + n]
        if lay.state_bits[i] == 8:
            o8, oa = lay.off8[i], lay.offa[i]
            nb = (n + lay.blocksize - 1) // lay.blocksize
            return B.TensorState(p, g, self.q1[o8:o8 + n], self.q2[o8:o8 + n] if self.two else None,
                                 self.a1[oa:oa + nb], self.a2[oa:oa + nb] if self.two else None)
        o32 = lay.off32[i]
        return B.TensorState(p, g, self.m32[o32:o32 + n], self.v32[o32:o32 + n] if self.two else None)

    def step(self, t: int, lr: float, beta1: float, beta2: float, eps: float, weight_decay: float, stream=None):
        B.bnbq_step_8bit(self.optim, self.packed, lr=lr, beta1=beta1, beta2=beta2, eps=eps,
                         weight_decay=weight_decay, step=t, code1=self.code1, code2=self.code2,
                         blocksize=self.layout.blocksize, stream=stream, ntensors=len(self.entries))
