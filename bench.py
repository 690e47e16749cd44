#!/usr/bin/env python
"""Benchmark of the fused 8-bit optimizer step (one JSON line on rank 0).

Default workload: 8-bit AdamW on the 7B Llama-shaped list (291 tensors, 6,738,415,616 fp32
parameters, bf16 gradients ~N(0,1e-3), signed / unsigned dynamic codes for m / v, blocksize 2048,
32-bit state for the token embedding; seed 4).  One step = one ``bnbq_step_8bit`` call = one
kernel launch over the whole list.  Inputs live in HBM (about 96 GB of traffic per step, far
above the 126 MB L2, so no L2 flush is needed between steps).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

``value``: parameters stepped per second over all ranks (each rank steps its own list: weak
scaling, no collective on the data path).  ``e2e``: the same metric through the public API with
the step's gradients copied from pinned host memory every step and the device flag word read
back.  ``roofline``: algorithmic bytes of one launch / the launch's average CUDA-event duration,
against the measured HBM copy bandwidth.  ``cpu_baseline``: the CPU oracle on a bounded sample.
``--impl reference`` times that oracle alone (the slow reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "8-bit AdamW step params/s and achieved HBM GB/s (% of B200 HBM roofline), 1 GPU"
WORKLOADS = {
    # name: (shape, optimizer, seed, hyper-parameters, (outlier fraction, outlier scale))
    "llama7b_adamw": ("llama7b", "adamw", 4, dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01),
                      (0.0, 1.0)),
    "gpt2_adamw": ("gpt2_1p5b", "adamw", 2, dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01),
                   (0.0, 1.0)),
    "llama7b_lion": ("llama7b", "lion", 3, dict(lr=1e-4, beta1=0.9, beta2=0.99, eps=0.0, weight_decay=0.1),
                     (1e-4, 100.0)),
    "llama7b_momentum": ("llama7b", "momentum", 3, dict(lr=1e-2, beta1=0.9, beta2=0.0, eps=0.0, weight_decay=0.0),
                         (1e-4, 100.0)),
    "llama7b_rmsprop": ("llama7b", "rmsprop", 3, dict(lr=1e-3, beta1=0.99, beta2=0.0, eps=1e-8, weight_decay=0.0),
                        (1e-4, 100.0)),
    # one decoder layer (202M params, ~3 GB): the size used for ncu captures
    "llama7b_layer_adamw": ("llama7b_layer", "adamw", 4,
                            dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01), (0.0, 1.0)),
}

# Standalone quantize / dequantize sweep points (development measurements of those kernels):
# name: (log2 n, input dtype, codebook, blocksize, nested block scales)
QUANT_WORKLOADS = {
    "quant_2p28_f32_signed_b2048": (28, "f32", "dynamic_signed", 2048, False),
    "quant_2p28_bf16_signed_b2048": (28, "bf16", "dynamic_signed", 2048, False),
    "quant_2p28_f32_nf4_b2048": (28, "f32", "nf4", 2048, False),
    "quant_2p28_f32_signed_b256": (28, "f32", "dynamic_signed", 256, False),
    "quant_2p28_f32_signed_b4096": (28, "f32", "dynamic_signed", 4096, False),
    # 4-bit weights as QLoRA stores them: blocksize 64, NF4 or FP4, bf16 weights
    "quant_2p28_bf16_nf4_b64": (28, "bf16", "nf4", 64, False),
    "quant_2p28_bf16_fp4_b64": (28, "bf16", "fp4", 64, False),
    # ... with the block scales nested (quantize + nest; dequantize rebuilding the scales)
    "quant_2p28_bf16_nf4_b64_nested": (28, "bf16", "nf4", 64, True),
}


# The sweep of standalone quantize / dequantize measurements: every combination of these.
QUANT_SWEEP = dict(log2n=(20, 24, 28), dtype=("f32", "bf16"), code=("dynamic_signed", "nf4"),
                   blocksize=(256, 2048, 4096))
L2_BYTES = 126 << 20


def quant_point(point, steps, warmup, seed_tag):
    """Time bnbq_quantize_blockwise and bnbq_dequantize_blockwise on one point (log2 n, input dtype,
    codebook, blocksize, nested scales); inputs ~N(0,1) with 0.1% of positions x50 (seed 1).  When
    a call's inputs and outputs are less than twice the L2 size, a 512 MB buffer is written before
    every timed call so that each one starts from HBM.  Returns a dict of timings and fractions of the HBM peak."""
    import torch
    import block_wise_bit_b200 as bq
    from block_wise_bit_b200 import workloads as W
    log2n, dt, code_name, B, nested = point
    n = 1 << log2n
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    dtype = torch.float32 if dt == "f32" else torch.bfloat16
    x = W.normal(n, 1.0, dev, "quant-sweep", 1, seed_tag)
    W.outliers_(x, 0.001, 50.0, dev, "quant-sweep", 1, seed_tag)
    x = x.to(dtype)
    code = bq.bnbq_codebook(code_name).to(dev)
    K = code.numel()
    absmax = torch.empty((n + B - 1) // B, dtype=torch.float32, device=dev)
    q = torch.empty(n if K == 256 else (n + 1) // 2, dtype=torch.uint8, device=dev)
    y = torch.empty(n, dtype=dtype, device=dev)
    esz = x.element_size()
    qbytes = n if K == 256 else n / 2
    nb = absmax.numel()
    alg_q = n * esz + qbytes + 4 * nb
    alg_dq = qbytes + 4 * nb + n * esz
    stream = torch.cuda.current_stream(dev)
    code2 = nest_bufs = None
    if nested:  # nest: read the scales twice (mean, quantize), write codes + second-level scales
        code2 = bq.bnbq_codebook("dynamic_signed").to(dev)
        nb2 = (nb + 255) // 256
        alg_q += 8 * nb + nb + 4 * nb2
        alg_dq = qbytes + nb + 4 * nb2 + n * esz
        nest_bufs = dict(qabs=torch.empty(nb, dtype=torch.uint8, device=dev),
                         absmax2=torch.empty(nb2, dtype=torch.float32, device=dev),
                         offset=torch.empty(1, dtype=torch.float32, device=dev),
                         workspace=torch.empty(max(1, bq.lib().bnbq_nested_workspace_bytes(nb)), dtype=torch.uint8,
                                               device=dev))
    # each call's bytes well above L2, or L2 is overwritten before every timed call
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if min(alg_q, alg_dq) < 2 * L2_BYTES else None

    def quantize():
        bq.bnbq_quantize_blockwise(code, x, B, absmax=absmax, out=q)
        return bq.bnbq_quantize_absmax_nested(code2, absmax, **nest_bufs) if nested else None

    def dequantize(nest):
        if nested:
            bq.bnbq_dequantize_blockwise_nested(code, q, *nest, code2, n, B, out=y)
        else:
            bq.bnbq_dequantize_blockwise(code, q, absmax, n, B, out=y)

    for _ in range(warmup):
        dequantize(quantize())
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for k in range(steps):
        if flush is not None:
            flush.zero_()
        evs[k][0].record(stream)
        nest = quantize()
        evs[k][1].record(stream)
        if flush is not None:
            flush.zero_()
        evs[k][2].record(stream)
        dequantize(nest)
        evs[k][3].record(stream)
    torch.cuda.synchronize()
    tq = sorted(e[0].elapsed_time(e[1]) for e in evs)
    td = sorted(e[2].elapsed_time(e[3]) for e in evs)
    mq, md = statistics.median(tq), statistics.median(td)
    peak, _ = measured_peaks()
    return dict(n=n, dtype=dt, codebook=code_name, blocksize=B, nested_scales=nested,
                l2="L2 overwritten before each call" if flush is not None else "each call moves over twice the L2 size",
                quantize={"ms": round(mq, 4), "GB/s": round(alg_q / mq / 1e6, 1),
                          "frac": round(alg_q / mq / 1e6 / peak, 4), "bytes": int(alg_q)},
                dequantize={"ms": round(md, 4), "GB/s": round(alg_dq / md / 1e6, 1),
                            "frac": round(alg_dq / md / 1e6 / peak, 4), "bytes": int(alg_dq)},
                elements_per_s=n / ((mq + md) / 1e3), launches=(5 if nested else 2) * steps)


def bench_quant(args, base):
    """One sweep point (--workload quant_*) or the whole sweep (--workload quant_sweep): one JSON
    line per point with GB/s of quantize and dequantize against the HBM peak."""
    import itertools
    if args.workload == "quant_sweep":
        points = [(l, d, c, b, False) for l, d, c, b in itertools.product(*QUANT_SWEEP.values())]
    else:
        points = [QUANT_WORKLOADS[args.workload]]
    peak, kind = measured_peaks()
    for pt in points:
        r = quant_point(pt, args.steps, args.warmup, args.workload if len(points) == 1 else "sweep")
        out = dict(base, metric="block-wise quantize + dequantize elements/s", unit="elements/s",
                   value=r.pop("elements_per_s"), n_gpus=1, steps=args.steps, warmup=args.warmup,
                   ms_per_step=round(r["quantize"]["ms"] + r["dequantize"]["ms"], 4), dtype=pt[1],
                   config={"workload": args.workload, **{k: r.pop(k) for k in ("n", "dtype", "codebook", "blocksize",
                                                                                "nested_scales", "l2")}},
                   quantize=r["quantize"], dequantize=r["dequantize"], peak_gbs=peak, peak_source=kind,
                   gpu_launches=r["launches"], quantize_src_sha=quant_source_sha())
        print(json.dumps(out), flush=True)


def bench_hbm_mix(args, base):
    """Context for the rooflines of write-heavy kernels (--workload hbm_mix): the HBM rate that
    torch's own kernels reach on 512 MiB buffers for a write-only stream (fill) and a 50/50
    read-write stream (copy), CUDA events, median over the timed calls.  None of this library's
    kernels run."""
    import torch
    dev = torch.device("cuda", 0)
    n = 1 << 28
    a = torch.empty(n, dtype=torch.bfloat16, device=dev).normal_()
    b = torch.empty_like(a)
    stream = torch.cuda.current_stream(dev)
    peak, kind = measured_peaks()
    res = {}
    for name, fn, nbytes in (("write_only_fill", lambda: b.fill_(1.5), 2 * n), ("copy", lambda: b.copy_(a), 4 * n)):
        for _ in range(args.warmup):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        torch.cuda.synchronize()
        for e0, e1 in evs:
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)
        res[name] = {"ms": round(ms, 4), "GB/s": round(nbytes / ms / 1e6, 1), "frac": round(nbytes / ms / 1e6 / peak, 4),
                     "bytes": nbytes}
    out = dict(base, metric="HBM rate of torch fill / copy (context)", unit="GB/s", value=res["write_only_fill"]["GB/s"],
               n_gpus=1, steps=args.steps, warmup=args.warmup, ms_per_step=res["write_only_fill"]["ms"], dtype="bf16",
               config={"workload": "hbm_mix", "bytes_per_buffer": 2 * n}, peak_gbs=peak, peak_source=kind,
               gpu_launches=0, **res)
    print(json.dumps(out), flush=True)


def bench_zero1(args, base, shape, optim, seed, hp, outlier):
    """ZeRO-1 data-parallel step over the whole list on ``world`` ranks: every rank holds the full
    flat parameters and its own full bf16 gradient; per step the gradients are reduce-scattered in
    place, each rank steps its block-aligned share (optimizer state exists only for it), and the
    parameters are all-gathered in place.  ``value``: parameters of the list stepped per second
    (the list is stepped once per step by all ranks together: strong scaling), with the two
    collectives and the step kernel timed separately (CUDA events, slowest rank)."""
    import torch
    import torch.distributed as dist
    import block_wise_bit_b200 as bq
    from block_wise_bit_b200 import optim as O
    from block_wise_bit_b200 import workloads as W
    from block_wise_bit_b200 import zero
    from datetime import timedelta
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if "MASTER_ADDR" not in os.environ:  # one process without a launcher
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(29500 + os.getpid() % 1000))
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=timedelta(seconds=120),
                            device_id=dev)
    B = 2048
    lay = W.Layout.build(W.SHAPES[shape](), B)
    numels = [sp.numel for sp in lay.specs]
    ex = zero.ZeroOneExchange(numels, B, world, rank)
    P = torch.zeros(ex.total, device=dev)
    G = torch.zeros(ex.total, device=dev, dtype=torch.bfloat16)
    for i, spec in enumerate(lay.specs):
        ex.views(P, i).copy_(W.normal(spec.numel, 0.02, dev, shape, seed, i, "p"))
        W.grad_fill_(ex.views(G, i), 1e-3, outlier[0], outlier[1], shape, seed, rank, i, "g")
    two = optim in ("adamw", "adam")
    code1 = O.device_codebook("dynamic_unsigned" if optim == "rmsprop" else "dynamic_signed", dev)
    code2 = O.device_codebook("dynamic_unsigned", dev) if two else None
    entries = []
    for pc, pv, gv in ex.piece_views(P, G):
        st = O.new_state(pv, two, lay.state_bits[pc.tensor], B, code1, code2)
        entries.append(bq.TensorState(pv, gv, st["state1"], st.get("state2"), st.get("absmax1"), st.get("absmax2")))
    packed = bq.pack_tensor_list(entries)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)

    def one_step(t, ev=None):
        if ev is not None:
            ev[0].record(stream)
        ex.reduce_scatter_grads(G)
        if ev is not None:
            ev[1].record(stream)
        if entries:
            bq.bnbq_step_8bit(optim, packed, ntensors=len(entries), step=t, code1=code1, code2=code2, blocksize=B,
                              **hp)
        if ev is not None:
            ev[2].record(stream)
        ex.all_gather_params(P)
        if ev is not None:
            ev[3].record(stream)

    t = 0
    for _ in range(args.warmup):
        t += 1
        one_step(t)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    dist.barrier()
    torch.cuda.synchronize()
    for k in range(args.steps):
        t += 1
        one_step(t, evs[k])
    torch.cuda.synchronize()
    dist.barrier()
    parts = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps for i in range(3)]
    total_ms = evs[0][0].elapsed_time(evs[-1][3])
    total_ms = max_over_ranks(total_ms, dev, world)
    parts = [max_over_ranks(x, dev, world) for x in parts]
    flags = bq.bnbq_device_flags(clear=True)
    if rank == 0:
        cfg = dict(base["config"], workload=f"{args.workload}8bit_zero1", parallelism=f"zero1 x{world}",
                   rank_share_params=sum(pc.numel for pc in ex.pieces[0]))
        out = dict(base, config=cfg, scaling="strong", value=lay.n_params * args.steps / (total_ms / 1e3),
                   n_gpus=world, steps=args.steps, warmup=args.warmup, ms_per_step=round(total_ms / args.steps, 4),
                   zero1={"reduce_scatter_ms": round(parts[0], 4), "step_ms": round(parts[1], 4),
                          "all_gather_ms": round(parts[2], 4), "grad_bytes": 2 * ex.total, "param_bytes": 4 * ex.total},
                   cpu_baseline=None, e2e=None, gpu_launches=args.steps, device_flags=flags)
        print(json.dumps(out))
    dist.destroy_process_group()


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
KERNEL_SOURCES = [os.path.join(ROOT, "block_wise_bit_b200", "csrc", f) for f in
                  ("bnbq_step.cu", "bnbq_device.cuh", "bnbq_internal.h")]


def algorithmic_bytes(lay, optim: str, g_bytes: int = 2) -> int:
    """Minimum HBM traffic of one step over the list: p read+write (8 B), g read, each state
    read+write (1+1 B per 8-bit code, 4+4 B per fp32 moment), each 8-bit block scale read+write."""
    two = optim in ("adamw", "adam")
    ns = 2 if two else 1
    total = 0
    B = lay.blocksize
    for s, bits in zip(lay.specs, lay.state_bits):
        if bits == 8:
            total += s.numel * (8 + g_bytes + 2 * ns) + ((s.numel + B - 1) // B) * 8 * ns
        else:
            total += s.numel * (8 + g_bytes + 8 * ns)
    return total


E2E_SLICES = 4  # with the main list's table, within the library's cache of 8 descriptor tables


def e2e_slices(lay, k: int):
    """Contiguous runs of tensors with about 1/k of the elements each: (first tensor, end tensor,
    first element, end element of their gradients in the flat buffer)."""
    n = len(lay.specs)
    total = sum(s.numel for s in lay.specs)
    out, i0, acc = [], 0, 0
    for i, s in enumerate(lay.specs):
        acc += s.numel
        if acc * k >= total * (len(out) + 1) or i == n - 1:
            out.append((i0, i + 1, lay.off[i0], lay.off[i] + s.numel))
            i0 = i + 1
    return out


_CODE_TOKENS = re.compile(r'"(?:\\.|[^"\\])*"|\'(?:\\.|[^\'\\])*\'|//[^\n]*|/\*.*?\*/|\s+|[^"\'/\s]+|/', re.S)


def _code_only(text: str) -> str:
    """The source with comments dropped and whitespace runs folded, so that a change to a
    comment keeps the hash (and the traffic record keyed on it) while any change to code does not."""
    out = []
    for tok in _CODE_TOKENS.findall(text):
        if tok.startswith("//") or tok.startswith("/*") or tok.isspace():
            out.append("\n" if "\n" in tok else " ")  # line breaks end preprocessor lines
        else:
            out.append(tok)
    return re.sub(r" *\n[\s]*", "\n", re.sub(" +", " ", "".join(out))).strip()


QUANT_SOURCES = [os.path.join(ROOT, "block_wise_bit_b200", "csrc", f) for f in
                 ("bnbq_quant.cu", "bnbq_nested.cu", "bnbq_async.cuh", "bnbq_device.cuh", "bnbq_internal.h",
                  "bnbq_search_fma.cuh")]


def quant_source_sha() -> str:
    """Hash of the quantize / dequantize kernels' code (comments and spacing ignored)."""
    h = hashlib.sha256()
    for f in QUANT_SOURCES:
        with open(f, encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
        h.update(b"\0")
    return h.hexdigest()[:16]


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(f, encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
        h.update(b"\0")
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def traffic_per_launch(workload: str, algorithmic: int):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    kernel source: the captured launch's DRAM bytes over its algorithmic bytes, times this
    launch's algorithmic bytes (traffic grows in proportion to the parameters stepped)."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(workload)
    if not e or e.get("kernel_src_sha") != kernel_source_sha():
        return None
    return int(round(e["dram_over_algorithmic"] * algorithmic))


# ------------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid: str | None):
        self.uuid = device_uuid
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [ln.split(",") for ln in self.file.read().strip().splitlines() if ln.count(",") >= 8]
        os.unlink(self.file.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------ CPU oracle leg
def oracle_rate(shape: str, optim: str, hp: dict, elements8: int, threads: int, steps: int = 1):
    """Time the CPU oracle (as it stands) on a bounded sample of the workload: ``elements8``
    elements with 8-bit state plus the list's share of 32-bit-state elements, split over
    ``threads`` threads (ctypes releases the GIL).  Returns (params/s, seconds, sample text)."""
    import oracle
    from block_wise_bit_b200 import workloads as W
    B = 2048
    lay = W.Layout.build(W.SHAPES[shape](), B)
    two = optim in ("adamw", "adam")
    frac32 = lay.n32 / max(1, lay.n_params)
    n8 = (elements8 // B) * B
    n32 = int(n8 * frac32 / max(1e-12, 1 - frac32)) // 4 * 4
    rng = np.random.default_rng(0)

    def arrays(n, bits):
        p = (rng.standard_normal(n) * 0.02).astype(np.float32)
        g = (rng.standard_normal(n) * 1e-3).astype(np.float32).view(np.uint32)
        g = ((g + 0x7FFF + ((g >> 16) & 1)) >> 16).astype(np.uint16)  # bf16 bits (round to nearest even)
        if bits == 8:
            nb = (n + B - 1) // B
            return dict(p=p, g=g, s1=rng.integers(0, 256, n).astype(np.uint8),
                        s2=rng.integers(0, 256, n).astype(np.uint8) if two else None,
                        a1=np.full(nb, 1e-3, np.float32), a2=np.full(nb, 1e-6, np.float32) if two else None)
        return dict(p=p, g=g, s1=np.zeros(n, np.float32), s2=np.zeros(n, np.float32) if two else None,
                    a1=None, a2=None)

    work = [(arrays(n8, 8), n8)] + ([(arrays(n32, 32), n32)] if n32 else [])
    c1 = oracle.code_dynamic_unsigned() if optim == "rmsprop" else oracle.code_dynamic_signed()
    c2 = oracle.code_dynamic_unsigned()
    jobs = []
    for arrs, n in work:
        nb = (n + B - 1) // B
        per = (nb + threads - 1) // threads
        for t0 in range(0, nb, per):
            jobs.append((arrs, (t0, min(nb, t0 + per))))

    def run(job, t):
        arrs, rng_ = job
        oracle.step_tensor(optim, arrs["p"], arrs["g"], arrs["s1"], arrs["s2"], arrs["a1"], arrs["a2"], c1,
                           c2 if two else None, B, step=t, block_range=rng_, **hp)

    oracle.lib()
    t0 = time.perf_counter()
    for t in range(1, steps + 1):
        if threads == 1:  # one thread: the jobs one after another
            for j in jobs:
                run(j, t)
            continue
        ths = [threading.Thread(target=run, args=(j, t)) for j in jobs]
        for th in ths:
            th.start()
        for th in ths:
            th.join()
    dt = time.perf_counter() - t0
    sample = (f"{n8} 8-bit-state + {n32} 32-bit-state elements of the {shape} {optim} step "
              f"(the list's 32-bit share), synthetic inputs, {steps} step(s), {threads} threads")
    return (n8 + n32) * steps / dt, dt, sample


def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- rank aggregation
def max_over_ranks(ms: float, device, world: int) -> float:
    """The slowest rank's time; every rank calls this at the same point (one all-reduce)."""
    if world == 1:
        return ms
    import torch
    import torch.distributed as dist
    tt = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def whole_job_rate(params_per_rank: int, steps: int, world: int, ms: float) -> float:
    """Parameters stepped by all ranks per second, over the slowest rank's time."""
    return params_per_rank * steps * world / (ms / 1e3)


# -------------------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(QUANT_WORKLOADS) + ["quant_sweep", "hbm_mix"],
                    default="llama7b_adamw")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--series", action="store_true",
                    help="add every timed launch's CUDA-event time to the JSON line (power-cap behaviour)")
    ap.add_argument("--zero1", action="store_true",
                    help="ZeRO-1 data-parallel step: reduce-scatter of gradients, each rank steps its share, "
                         "all-gather of parameters (NCCL)")
    ap.add_argument("--cpu-sample", type=int, default=1 << 24, help="8-bit elements in the CPU oracle sample")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="wall time the CPU baseline aims for (consecutive oracle steps over the sample)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload.startswith("quant") or args.workload == "hbm_mix":
        shape, optim, seed, hp, (ofrac, oscale) = WORKLOADS["llama7b_adamw"]
    else:
        shape, optim, seed, hp, (ofrac, oscale) = WORKLOADS[args.workload]

    from block_wise_bit_b200 import workloads as W
    lay = W.Layout.build(W.SHAPES[shape](), 2048)
    config = {"workload": f"{args.workload}8bit", "list": shape, "tensors": len(lay.specs),
              "params": lay.n_params, "params_8bit_state": lay.n8, "params_32bit_state": lay.n32,
              "blocksize": 2048, "grad_dtype": "bf16", "optimizer": optim, **hp,
              "l2": "inputs far larger than the 126 MB L2 (no flush needed)"}
    base = {"metric": METRIC, "unit": "params/s", "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded normal inputs, no weights)",
            "config": config}

    if args.impl == "reference":
        if rank != 0:
            return
        threads = cpu_threads()
        per_step = max(2048, args.cpu_sample // 4)
        oracle_rate(shape, optim, hp, 2048 * threads, threads, 1)  # warm the library / pages
        for _ in range(args.warmup):
            oracle_rate(shape, optim, hp, per_step, threads, 1)
        rates, secs = [], []
        for _ in range(args.steps):
            r, dt, sample = oracle_rate(shape, optim, hp, per_step, threads, 1)
            rates.append(r)
            secs.append(dt)
        total = sum(secs)
        value = float(statistics.median(rates))
        out = dict(base, impl="reference", value=value, n_gpus=args.gpus, steps=args.steps, warmup=args.warmup,
                   ms_per_step=1e3 * total / args.steps,
                   cpu_baseline={"value": value, "unit": "params/s", "cores": threads, "kind": "oracle",
                                 "sample": sample + " per step"},
                   e2e={"value": value, "unit": "params/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0})
        print(json.dumps(out))
        return

    import torch
    import torch.distributed as dist
    import block_wise_bit_b200 as bq
    from block_wise_bit_b200.optim import FlatStateList

    if args.workload.startswith("quant"):
        return bench_quant(args, base)
    if args.workload == "hbm_mix":
        return bench_hbm_mix(args, base)
    if args.zero1:
        return bench_zero1(args, base, shape, optim, seed, hp, (ofrac, oscale))

    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    bq.lib()

    fl = FlatStateList(lay, optim, dev, g_dtype=torch.bfloat16)
    for i, spec in enumerate(lay.specs):
        fl.entries[i].p.copy_(W.normal(spec.numel, 0.02, dev, shape, seed, rank, i, "p"))
        W.grad_fill_(fl.entries[i].g, 1e-3, ofrac, oscale, shape, seed, rank, i, "g")
    torch.cuda.synchronize()
    bq.bnbq_device_flags(clear=True)

    t = 0
    for _ in range(args.warmup):
        t += 1
        fl.step(t, **hp)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    stream = torch.cuda.current_stream(dev)
    k_start = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    k_end = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")
    ev0.record(stream)
    for k in range(args.steps):
        t += 1
        k_start[k].record(stream)
        fl.step(t, **hp)
        k_end[k].record(stream)
    ev1.record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    barrier()
    clk = clocks.stop()

    total_ms = ev0.elapsed_time(ev1)
    launch_ms = [a.elapsed_time(b) for a, b in zip(k_start, k_end)]
    avg_launch_ms = sum(launch_ms) / len(launch_ms)
    total_ms = max_over_ranks(total_ms, dev, world)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(lay.n_params, args.steps, world, total_ms)
    flags = bq.bnbq_device_flags(clear=True)

    alg = algorithmic_bytes(lay, optim, 2)
    peak, peak_kind = measured_peaks()
    achieved = alg / (avg_launch_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic_per_launch(args.workload, alg),
                "peak_source": f"{peak_kind} HBM copy bandwidth", "algorithmic_bytes_per_launch": alg,
                "kernel": f"step_kernel<{optim}, 2048>", "avg_launch_ms": round(avg_launch_ms, 4),
                "median_launch_ms": round(statistics.median(launch_ms), 4),
                "min_launch_ms": round(min(launch_ms), 4), "max_launch_ms": round(max(launch_ms), 4)}
    if roofline["traffic"] is not None:  # the same rate from the ncu DRAM bytes of a captured launch
        roofline["dram_gbs"] = round(roofline["traffic"] / (avg_launch_ms / 1e3) / 1e9, 1)
    if args.series:
        roofline["launch_ms"] = [round(x, 3) for x in launch_ms]
        k = max(1, len(launch_ms) // 3)
        roofline["last_third_mean_ms"] = round(sum(launch_ms[-k:]) / k, 4)

    e2e = None
    if not args.no_e2e and args.e2e_steps > 0:
        # End to end from host gradients, as a user would drive it: the list is stepped in
        # E2E_SLICES contiguous slices of tensors (one public bnbq_step_8bit call each); a slice's
        # gradients are copied host -> device on a side stream and its step starts as soon as they
        # have landed, so the copies of later slices overlap the steps of earlier ones.  The next
        # step's copy of a slice waits for that slice's previous step (which reads the buffer).
        g_host = torch.empty(fl.g.numel(), dtype=fl.g.dtype, pin_memory=True)
        g_host.copy_(fl.g)
        slices = e2e_slices(lay, E2E_SLICES)
        packed = [(bq.pack_tensor_list(fl.entries[i0:i1]), i1 - i0) for (i0, i1, _, _) in slices]
        copy_stream = torch.cuda.Stream(dev)
        landed = [torch.cuda.Event() for _ in slices]
        stepped = [torch.cuda.Event() for _ in slices]
        for ev in stepped:
            ev.record(stream)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            t += 1
            for k, (i0, i1, a, b) in enumerate(slices):
                copy_stream.wait_event(stepped[k])
                with torch.cuda.stream(copy_stream):
                    fl.g[a:b].copy_(g_host[a:b], non_blocking=True)
                landed[k].record(copy_stream)
                stream.wait_event(landed[k])
                bq.bnbq_step_8bit(optim, packed[k][0], ntensors=packed[k][1], step=t, code1=fl.code1, code2=fl.code2,
                                  blocksize=lay.blocksize, stream=stream, **hp)
                stepped[k].record(stream)
            flags |= bq.bnbq_device_flags()  # device -> host read of the step's status word
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = e0.elapsed_time(e1)
        e_ms = max_over_ranks(e_ms, dev, world)
        e2e = {"value": whole_job_rate(lay.n_params, args.e2e_steps, world, e_ms), "unit": "params/s",
               "h2d_bytes_per_step": sum(b - a for (_, _, a, b) in slices) * g_host.element_size(),
               "d2h_bytes_per_step": 4, "steps": args.e2e_steps, "slices": len(slices),
               "scope": "each step uploads that step's bf16 gradients from pinned host memory and reads the "
                        "device status word back; parameters and optimizer state stay resident on the device, "
                        "as in a training loop"}
        del g_host, packed

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = cpu_threads()
        r, dt, sample = oracle_rate(shape, optim, hp, args.cpu_sample, threads, 1)  # also warms up
        if dt < args.cpu_seconds:
            k = max(2, math.ceil(args.cpu_seconds / max(dt, 1e-3)))
            r, dt, sample = oracle_rate(shape, optim, hp, args.cpu_sample, threads, k)
        r1, dt1, sample1 = oracle_rate(shape, optim, hp, 1 << 22, 1, 1)
        cpu = {"value": r, "unit": "params/s", "cores": threads, "kind": "oracle", "sample": sample,
               "seconds": round(dt, 2),
               "single_thread": {"value": r1, "unit": "params/s", "sample": sample1, "seconds": round(dt1, 2)}}

    if rank == 0:
        out = dict(base, value=value, n_gpus=world, steps=args.steps, warmup=args.warmup,
                   ms_per_step=round(ms_per_step, 4), roofline=roofline, cpu_baseline=cpu, e2e=e2e,
                   gpu_launches=args.steps, clocks=clk, device_flags=flags,
                   hbm_gbs_algorithmic=round(alg * args.steps / (total_ms / 1e3) / 1e9 * world, 1))
        print(json.dumps(out))
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
