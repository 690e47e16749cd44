"""Seeded synthetic workloads: parameter-list shapes and their inputs.

This module holds none of the method's arithmetic.  It only describes parameter lists (names,
sizes, which tensors keep 32-bit state) and draws seeded random inputs with torch's generators;
the CUDA library and the CPU oracle both consume what it produces.

Shapes (stand-ins for the models the 8-bit optimizer pages train; no weights are loaded):
  * GPT-2 1.5B: 48 layers, d_model 1600, d_ff 6400, vocab 50257, 1024 positions -- 580 tensors,
    1,557,611,200 parameters.
  * Llama 7B: 32 layers, d_model 4096, d_ff 11008, vocab 32000, untied lm_head -- 291 tensors,
    6,738,415,616 parameters.
  * tiny: one tensor of 65,536 elements.
Which tensors keep 32-bit state: those with fewer than 4096 elements and the token-embedding
table (page "Py之bitsandbytes：bitsandbytes的简介、安装、使用方法之详细攻略", sections
"如果需要高精度的参数" and "更改单个参数的位数和其他超参数"; the embedding override follows the
stable-embedding advice of the same page).
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field
from typing import List, Optional

import torch


@dataclass(frozen=True)
class ParamSpec:
    name: str
    numel: int
    embedding: bool = False  # token-embedding table


def state_bits_for(spec: ParamSpec, min_8bit_size: int = 4096) -> int:
    """32-bit state for tensors with fewer than ``min_8bit_size`` elements and for the
    token-embedding table; 8-bit state otherwise."""
    return 32 if (spec.numel < min_8bit_size or spec.embedding) else 8


def gpt2_1p5b() -> List[ParamSpec]:
    d, f, vocab, pos, L = 1600, 6400, 50257, 1024, 48
    specs = [ParamSpec("wte", vocab * d, embedding=True), ParamSpec("wpe", pos * d)]
    for i in range(L):
        h = f"h{i}."
        specs += [ParamSpec(h + "ln_1.w", d), ParamSpec(h + "ln_1.b", d),
                  ParamSpec(h + "attn.c_attn.w", d * 3 * d), ParamSpec(h + "attn.c_attn.b", 3 * d),
                  ParamSpec(h + "attn.c_proj.w", d * d), ParamSpec(h + "attn.c_proj.b", d),
                  ParamSpec(h + "ln_2.w", d), ParamSpec(h + "ln_2.b", d),
                  ParamSpec(h + "mlp.c_fc.w", d * f), ParamSpec(h + "mlp.c_fc.b", f),
                  ParamSpec(h + "mlp.c_proj.w", f * d), ParamSpec(h + "mlp.c_proj.b", d)]
    specs += [ParamSpec("ln_f.w", d), ParamSpec("ln_f.b", d)]
    return specs


def llama7b() -> List[ParamSpec]:
    d, f, vocab, L = 4096, 11008, 32000, 32
    specs = [ParamSpec("embed_tokens", vocab * d, embedding=True)]
    for i in range(L):
        h = f"layers.{i}."
        specs += [ParamSpec(h + n, d * d) for n in ("q_proj", "k_proj", "v_proj", "o_proj")]
        specs += [ParamSpec(h + n, d * f) for n in ("gate_proj", "up_proj", "down_proj")]
        specs += [ParamSpec(h + "input_layernorm", d), ParamSpec(h + "post_attention_layernorm", d)]
    specs += [ParamSpec("norm", d), ParamSpec("lm_head", vocab * d)]
    return specs


def llama7b_layer() -> List[ParamSpec]:
    """One decoder layer of the Llama-7B list (202,383,360 parameters)."""
    return [s for s in llama7b() if s.name.startswith("layers.0.")]


def tiny() -> List[ParamSpec]:
    return [ParamSpec("w", 65536)]


SHAPES = {"gpt2_1p5b": gpt2_1p5b, "llama7b": llama7b, "llama7b_layer": llama7b_layer, "tiny": tiny}


def seed_of(*parts) -> int:
    """Stable 63-bit seed from any tuple of ints / strings."""
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def generator(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed_of(*parts))
    return g


def normal(n: int, std: float, device, *seed_parts, dtype=torch.float32) -> torch.Tensor:
    """N(0, std^2) samples drawn in fp32, then rounded to ``dtype`` (bf16: round to nearest even)."""
    x = torch.randn(n, generator=generator(device, *seed_parts), device=device, dtype=torch.float32)
    x.mul_(std)
    return x.to(dtype) if dtype != torch.float32 else x


def outliers_(x: torch.Tensor, fraction: float, scale: float, device, *seed_parts) -> torch.Tensor:
    """Multiply a seeded random ``fraction`` of the entries of x by ``scale`` (in place)."""
    if fraction <= 0:
        return x
    u = torch.rand(x.numel(), generator=generator(device, *seed_parts, "outliers"), device=device)
    sel = u < fraction
    x[sel] = (x[sel].float() * scale).to(x.dtype)
    return x


def grad_fill_(g: torch.Tensor, std: float, outlier_fraction: float, outlier_scale: float, *seed_parts) -> None:
    """Fill a gradient buffer in place (same distribution as ``normal`` + ``outliers_``)."""
    src = normal(g.numel(), std, g.device, *seed_parts, dtype=g.dtype)
    outliers_(src, outlier_fraction, outlier_scale, g.device, *seed_parts)
    g.copy_(src.view_as(g))


def random_codes(n: int, device, *seed_parts, zero_index: Optional[int] = None) -> torch.Tensor:
    """Uniform random 8-bit code indices (a synthetic non-zero optimizer state)."""
    return torch.randint(0, 256, (n,), generator=generator(device, *seed_parts), device=device,
                         dtype=torch.int32).to(torch.uint8)


def log_uniform(n: int, lo: float, hi: float, device, *seed_parts) -> torch.Tensor:
    """n fp32 values log-uniform in [lo, hi] (synthetic block scales)."""
    u = torch.rand(n, generator=generator(device, *seed_parts), device=device, dtype=torch.float64)
    return torch.exp(torch.log(torch.tensor(lo, dtype=torch.float64)) * (1 - u)
                     + torch.log(torch.tensor(hi, dtype=torch.float64)) * u).float()


@dataclass
class Layout:
    """Offsets of each tensor inside flat buffers (every offset keeps 16-byte alignment)."""
    specs: List[ParamSpec]
    state_bits: List[int]
    blocksize: int
    off: List[int] = field(default_factory=list)          # element offset in the p / g flats
    off8: List[int] = field(default_factory=list)         # element offset in the 8-bit state flats
    off32: List[int] = field(default_factory=list)        # element offset in the 32-bit state flats
    offa: List[int] = field(default_factory=list)         # block offset in the absmax flats
    total: int = 0
    total8: int = 0
    total32: int = 0
    totala: int = 0

    @staticmethod
    def build(specs: List[ParamSpec], blocksize: int, min_8bit_size: int = 4096) -> "Layout":
        bits = [state_bits_for(s, min_8bit_size) for s in specs]
        lay = Layout(specs, bits, blocksize)
        up4 = lambda x: (x + 3) // 4 * 4  # noqa: E731
        for s, b in zip(specs, bits):
            lay.off.append(lay.total)
            lay.total += up4(s.numel)
            if b == 8:
                lay.off8.append(lay.total8)
                lay.off32.append(-1)
                lay.offa.append(lay.totala)
                lay.total8 += up4(s.numel)
                lay.totala += up4((s.numel + blocksize - 1) // blocksize)
            else:
                lay.off8.append(-1)
                lay.offa.append(-1)
                lay.off32.append(lay.total32)
                lay.total32 += up4(s.numel)
        return lay

    @property
    def n_params(self) -> int:
        return sum(s.numel for s in self.specs)

    @property
    def n8(self) -> int:
        return sum(s.numel for s, b in zip(self.specs, self.state_bits) if b == 8)

    @property
    def n32(self) -> int:
        return sum(s.numel for s, b in zip(self.specs, self.state_bits) if b == 32)

    @property
    def n_blocks8(self) -> int:
        B = self.blocksize
        return sum((s.numel + B - 1) // B for s, b in zip(self.specs, self.state_bits) if b == 8)
