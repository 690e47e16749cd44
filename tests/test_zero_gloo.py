"""Multi-rank host logic on CPU: a ZeRO-1 split of the tensor list on block boundaries, run as two
gloo ranks.  Each rank steps only its pieces (with the CPU oracle standing in for the kernel);
gathering the pieces must reproduce the single-rank step bit for bit, since blocks are independent
(abstract of "8-bit Optimizers via Block-wise Quantization": blocks are quantized independently)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_wise_bit_b200 import zero

NUMELS = [5000, 3, 4096 * 2 + 17, 70000, 100, 2048]
B = 2048
HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def _inputs():
    import oracle
    rng = np.random.default_rng(42)
    c1, c2 = oracle.code_dynamic_signed(), oracle.code_dynamic_unsigned()
    lst = []
    for n in NUMELS:
        nb = (n + B - 1) // B
        lst.append(dict(p=(rng.standard_normal(n) * 0.02).astype(np.float32),
                        g=(rng.standard_normal(n) * 1e-3).astype(np.float32),
                        s1=rng.integers(0, 256, n).astype(np.uint8), s2=rng.integers(0, 256, n).astype(np.uint8),
                        a1=rng.uniform(1e-4, 1e-3, nb).astype(np.float32),
                        a2=rng.uniform(1e-8, 1e-6, nb).astype(np.float32)))
    return lst, c1, c2


def _step_piece(oracle, d, pc, c1, c2, t):
    s, e = pc.start, pc.start + pc.numel
    b0, b1 = pc.first_block, pc.first_block + pc.n_blocks
    part = {k: np.ascontiguousarray(d[k][s:e]) for k in ("p", "g", "s1", "s2")}
    part["a1"] = np.ascontiguousarray(d["a1"][b0:b1])
    part["a2"] = np.ascontiguousarray(d["a2"][b0:b1])
    oracle.step_tensor("adamw", part["p"], part["g"], part["s1"], part["s2"], part["a1"], part["a2"], c1, c2, B,
                       step=t, **HP)
    return part


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        lst, c1, c2 = _inputs()
        shards = zero.partition(NUMELS, B, world)
        mine = [(pc, _step_piece(oracle, lst[pc.tensor], pc, c1, c2, 3)) for pc in shards[rank]]
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        if rank == 0:
            q.put(gathered)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_partition_covers_every_block_once_and_balances():
    for world in (1, 2, 3, 8):
        shards = zero.partition(NUMELS, B, world)
        seen = {}
        for r, pieces in enumerate(shards):
            for pc in pieces:
                assert pc.start == pc.first_block * B
                for b in range(pc.first_block, pc.first_block + pc.n_blocks):
                    assert (pc.tensor, b) not in seen
                    seen[(pc.tensor, b)] = r
                n = NUMELS[pc.tensor]
                assert pc.numel == min(n, (pc.first_block + pc.n_blocks) * B) - pc.start
        assert len(seen) == sum((n + B - 1) // B for n in NUMELS)
        loads = [sum(pc.numel for pc in pieces) for pieces in shards]
        assert max(loads) - min(loads) <= 2 * B or world > len(seen)


def test_two_gloo_ranks_reproduce_single_rank_step(oracle_mod):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    gathered = q.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    lst, c1, c2 = _inputs()
    for d in lst:  # single-rank reference: the whole list
        oracle_mod.step_tensor("adamw", d["p"], d["g"], d["s1"], d["s2"], d["a1"], d["a2"], c1, c2, B, step=3, **HP)
    covered = 0
    for rank_pieces in gathered:
        for pc, part in rank_pieces:
            d = lst[pc.tensor]
            s, e = pc.start, pc.start + pc.numel
            b0, b1 = pc.first_block, pc.first_block + pc.n_blocks
            np.testing.assert_array_equal(part["p"], d["p"][s:e])
            np.testing.assert_array_equal(part["s1"], d["s1"][s:e])
            np.testing.assert_array_equal(part["s2"], d["s2"][s:e])
            np.testing.assert_array_equal(part["a1"], d["a1"][b0:b1])
            np.testing.assert_array_equal(part["a2"], d["a2"][b0:b1])
            covered += pc.numel
    assert covered == sum(NUMELS)
