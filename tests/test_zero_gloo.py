"""Multi-rank host logic on CPU: a ZeRO-1 split of the tensor list on block boundaries, run as two
gloo ranks.  Each rank steps only its pieces (with the CPU oracle standing in for the kernel);
gathering the pieces must reproduce the single-rank step bit for bit, since blocks are independent
(abstract of "8-bit Optimizers via Block-wise Quantization": blocks are quantized independently)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
from hypothesis import given, settings, strategies as st
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


@settings(max_examples=300, deadline=None)
@given(numels=st.lists(st.integers(0, 20000), max_size=12), bs=st.sampled_from([256, 2048, 4096]),
       world=st.integers(1, 9))
def test_partition_properties_on_random_lists(numels, bs, world):
    """Any list (empty tensors included), blocksize and world size: every block lands on exactly
    one rank, ranks hold consecutive runs of the list's blocks in rank order, pieces are
    block-aligned, and no rank holds more than its equal share plus one block."""
    shards = zero.partition(numels, bs, world)
    assert len(shards) == world
    order = [(t, b) for t, n in enumerate(numels) for b in range((n + bs - 1) // bs)]
    got = []
    for pieces in shards:
        for pc in pieces:
            assert pc.n_blocks >= 1 and pc.start == pc.first_block * bs
            assert pc.numel == min(numels[pc.tensor], (pc.first_block + pc.n_blocks) * bs) - pc.start
            got += [(pc.tensor, b) for b in range(pc.first_block, pc.first_block + pc.n_blocks)]
    assert got == order
    total = sum(numels)
    for pieces in shards:
        assert sum(pc.numel for pc in pieces) < total / world + bs or total == 0


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


# ------------------------------------------------------------------ the ZeRO-1 exchange, 2 gloo ranks
def _exchange_inputs(world):
    rng = np.random.default_rng(7)
    ex = zero.ZeroOneExchange(NUMELS, B, world, 0)
    p = np.zeros(ex.total, np.float32)
    for n, o in zip(NUMELS, ex.offsets):
        p[o:o + n] = (rng.standard_normal(n) * 0.02).astype(np.float32)
    grads = [np.zeros(ex.total, np.float32) for _ in range(world)]
    for r in range(world):
        for n, o in zip(NUMELS, ex.offsets):
            grads[r][o:o + n] = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    states = []
    for n in NUMELS:
        nb = (n + B - 1) // B
        states.append(dict(s1=rng.integers(0, 256, n).astype(np.uint8), s2=rng.integers(0, 256, n).astype(np.uint8),
                           a1=rng.uniform(1e-4, 1e-3, nb).astype(np.float32),
                           a2=rng.uniform(1e-8, 1e-6, nb).astype(np.float32)))
    return ex.offsets, p, grads, states


def _exchange_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        offs, p, grads, states = _exchange_inputs(world)
        c1, c2 = oracle.code_dynamic_signed(), oracle.code_dynamic_unsigned()
        ex = zero.ZeroOneExchange(NUMELS, B, world, rank)
        P, G = torch.from_numpy(p), torch.from_numpy(grads[rank])
        ex.reduce_scatter_grads(G)
        mine = []
        for pc, pv, gv in ex.piece_views(P, G):
            st = states[pc.tensor]
            b0, b1 = pc.first_block, pc.first_block + pc.n_blocks
            s = {k: np.ascontiguousarray(st[k][pc.start:pc.start + pc.numel]) for k in ("s1", "s2")}
            a = {k: np.ascontiguousarray(st[k][b0:b1]) for k in ("a1", "a2")}
            oracle.step_tensor("adamw", pv.numpy(), gv.numpy(), s["s1"], s["s2"], a["a1"], a["a2"], c1, c2, B,
                               step=5, **HP)
            mine.append((pc, s, a))
        ex.all_gather_params(P)
        q.put((rank, P.numpy().copy(), mine))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_zero1_exchange_two_gloo_ranks_equals_single_rank_step(oracle_mod):
    """Reduce-scatter of the gradients, a step of each rank's pieces, all-gather of the
    parameters, both collectives in place on the flat buffers: every rank ends with the
    parameters of one single-rank step on the summed gradient, and the pieces' states equal the
    single-rank states, bit for bit."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_exchange_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    offs, p, grads, states = _exchange_inputs(world)
    g = grads[0] + grads[1]  # two ranks: the sum is the same in either order
    c1, c2 = oracle_mod.code_dynamic_signed(), oracle_mod.code_dynamic_unsigned()
    for n, o, st in zip(NUMELS, offs, states):
        pv = p[o:o + n]
        oracle_mod.step_tensor("adamw", pv, np.ascontiguousarray(g[o:o + n]), st["s1"], st["s2"], st["a1"], st["a2"],
                               c1, c2, B, step=5, **HP)
    covered = 0
    for rank, P, mine in results:
        np.testing.assert_array_equal(P, p)
        for pc, s, a in mine:
            st = states[pc.tensor]
            np.testing.assert_array_equal(s["s1"], st["s1"][pc.start:pc.start + pc.numel])
            np.testing.assert_array_equal(s["s2"], st["s2"][pc.start:pc.start + pc.numel])
            np.testing.assert_array_equal(a["a1"], st["a1"][pc.first_block:pc.first_block + pc.n_blocks])
            np.testing.assert_array_equal(a["a2"], st["a2"][pc.first_block:pc.first_block + pc.n_blocks])
            covered += pc.numel
    assert covered == sum(NUMELS)


def _check_exchange_layout(numels, bs, world):
    ex = zero.ZeroOneExchange(numels, bs, world, 0)
    assert ex.chunk % bs == 0 and ex.total == world * ex.chunk
    for t, (n, o) in enumerate(zip(numels, ex.offsets)):
        assert o % bs == 0 and o + n <= ex.total
        if t + 1 < len(numels):
            assert ex.offsets[t + 1] >= o + n
    owner = {}
    for r, pcs in enumerate(ex.pieces):
        assert pcs == zero.ZeroOneExchange(numels, bs, world, r).pieces[r]
        for pc in pcs:
            a = ex.offsets[pc.tensor] + pc.start
            assert r * ex.chunk <= a and a + pc.numel <= (r + 1) * ex.chunk  # inside the rank's range
            assert pc.start == pc.first_block * bs and pc.n_blocks >= 1
            assert pc.numel == min(numels[pc.tensor], (pc.first_block + pc.n_blocks) * bs) - pc.start
            owner.setdefault(pc.tensor, []).append((pc.start, pc.start + pc.numel))
    for t, n in enumerate(numels):  # every element of every tensor on exactly one rank
        spans = sorted(owner.get(t, []))
        assert sum(e - s for s, e in spans) == n
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:])) and (not spans or spans[0][0] == 0)
    padded = sum((n + bs - 1) // bs * bs for n in numels)
    assert ex.chunk <= max(bs, (padded // bs + world - 1) // world * bs)  # an equal share, to one block


def test_zero1_exchange_layout():
    """Tensor offsets on block boundaries, equal block-aligned chunks per rank, each rank's pieces
    inside its chunk, every element owned once."""
    for world in (1, 2, 3, 8):
        _check_exchange_layout(NUMELS, B, world)


@settings(max_examples=200, deadline=None)
@given(numels=st.lists(st.integers(0, 20000), min_size=1, max_size=10), bs=st.sampled_from([256, 2048]),
       world=st.integers(1, 8))
def test_zero1_exchange_layout_on_random_lists(numels, bs, world):
    _check_exchange_layout(numels, bs, world)
