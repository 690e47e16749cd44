"""The ZeRO-1 exchange on the GPU path (NCCL backend, one rank: the only GPU of these runs).

Reduce-scatter of the gradients, the CUDA step over this rank's pieces (views into the flat
buffers and into the state), all-gather of the parameters: with one rank the pieces are whole
tensors and the result must equal a direct step over the full tensors, bit for bit.  The
multi-rank exchange itself is checked with gloo ranks in test_zero_gloo.py.
"""
import datetime
import socket

import pytest
import torch
import torch.distributed as dist

import block_wise_bit_b200 as bq
from block_wise_bit_b200 import workloads as W
from block_wise_bit_b200 import zero

pytestmark = pytest.mark.gpu
DEV = "cuda"
NUMELS = [5000, 3, 4096 * 2 + 17, 70000, 100, 2048]
B = 2048
HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_zero1_exchange_nccl_one_rank_equals_direct_step():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    c1 = bq.bnbq_codebook("dynamic_signed").to(DEV)
    c2 = bq.bnbq_codebook("dynamic_unsigned").to(DEV)
    offs, o = [], 0
    for n in NUMELS:
        offs.append(o)
        o += (n + 15) // 16 * 16
    P = torch.zeros(o, device=DEV)
    G = torch.zeros(o, device=DEV)
    states = []
    for i, (n, off) in enumerate(zip(NUMELS, offs)):
        P[off:off + n] = W.normal(n, 0.02, DEV, "zero-gpu", i, "p")
        G[off:off + n] = W.normal(n, 1e-3, DEV, "zero-gpu", i, "g")
        nb = (n + B - 1) // B
        if n >= 4096:
            states.append(dict(s1=W.random_codes(n, DEV, "zero-gpu", i, "q1"), s2=W.random_codes(n, DEV, "zero-gpu", i, "q2"),
                               a1=W.log_uniform(nb, 1e-4, 1e-2, DEV, "zero-gpu", i, "a1"),
                               a2=W.log_uniform(nb, 1e-8, 1e-5, DEV, "zero-gpu", i, "a2")))
        else:
            states.append(dict(s1=torch.zeros(n, device=DEV), s2=torch.zeros(n, device=DEV), a1=None, a2=None))
    ref_P = P.clone()
    ref_states = [{k: (None if v is None else v.clone()) for k, v in st.items()} for st in states]
    direct = [bq.TensorState(ref_P[off:off + n], G[off:off + n], st["s1"], st["s2"], st["a1"], st["a2"])
              for n, off, st in zip(NUMELS, offs, ref_states)]
    bq.bnbq_step_8bit("adamw", direct, step=3, code1=c1, code2=c2, blocksize=B, **HP)

    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ex = zero.ZeroOneExchange(NUMELS, offs, B, 1, 0)
        g_chunk = ex.reduce_scatter_grads(G)
        pieces = []
        for pc, pv, gv in ex.piece_views(P, g_chunk):
            st = states[pc.tensor]
            s = slice(pc.start, pc.start + pc.numel)
            a = slice(pc.first_block, pc.first_block + pc.n_blocks)
            pieces.append(bq.TensorState(pv, gv, st["s1"][s], st["s2"][s], None if st["a1"] is None else st["a1"][a],
                                         None if st["a2"] is None else st["a2"][a]))
        bq.bnbq_step_8bit("adamw", pieces, step=3, code1=c1, code2=c2, blocksize=B, **HP)
        ex.all_gather_params(P)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(P, ref_P)
    for st, rs in zip(states, ref_states):
        for k in ("s1", "s2", "a1", "a2"):
            if st[k] is not None:
                assert torch.equal(st[k], rs[k])
