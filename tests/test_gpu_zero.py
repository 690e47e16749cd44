"""The ZeRO-1 exchange on the GPU path (NCCL backend, one rank: the only GPU of these runs).

Reduce-scatter of the gradients (in place on the flat buffer), the CUDA step over this rank's
pieces (views into the flat buffers and into the state), all-gather of the parameters (in place):
the parameters and every piece's state must equal the CPU oracle's step of the same inputs, bit
for bit.  The multi-rank exchange itself is checked with gloo ranks in test_zero_gloo.py.
"""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import block_wise_bit_b200 as bq
from block_wise_bit_b200 import workloads as W
from block_wise_bit_b200 import zero

from . import parity

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


def test_zero1_exchange_nccl_one_rank_matches_oracle(oracle_mod):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    c1 = bq.bnbq_codebook("dynamic_signed")
    c2 = bq.bnbq_codebook("dynamic_unsigned")
    ex = zero.ZeroOneExchange(NUMELS, B, 1, 0)
    P = torch.zeros(ex.total, device=DEV)
    G = torch.zeros(ex.total, device=DEV, dtype=torch.bfloat16)
    states = []
    for i, n in enumerate(NUMELS):
        ex.views(P, i).copy_(W.normal(n, 0.02, DEV, "zero-gpu", i, "p"))
        ex.views(G, i).copy_(W.normal(n, 1e-3, DEV, "zero-gpu", i, "g"))
        nb = (n + B - 1) // B
        if n >= 4096:
            states.append(dict(s1=W.random_codes(n, DEV, "zero-gpu", i, "q1"), s2=W.random_codes(n, DEV, "zero-gpu", i, "q2"),
                               a1=W.log_uniform(nb, 1e-4, 1e-2, DEV, "zero-gpu", i, "a1"),
                               a2=W.log_uniform(nb, 1e-8, 1e-5, DEV, "zero-gpu", i, "a2")))
        else:
            states.append(dict(s1=W.normal(n, 1e-3, DEV, "zero-gpu", i, "m"),
                               s2=W.normal(n, 1e-3, DEV, "zero-gpu", i, "v").square_(), a1=None, a2=None))
    # the oracle's step of the same inputs (one rank: the summed gradient is this rank's gradient)
    host = [dict(p=parity.to_np(ex.views(P, i)), g=parity.to_np(ex.views(G, i)),
                 **{k: (None if v is None else parity.to_np(v)) for k, v in st.items()})
            for i, st in enumerate(states)]
    for h in host:
        oracle_mod.step_tensor("adamw", h["p"], h["g"], h["s1"], h["s2"], h["a1"], h["a2"], c1.numpy(), c2.numpy(), B,
                               step=3, **HP)

    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ex.reduce_scatter_grads(G)
        pieces = []
        for pc, pv, gv in ex.piece_views(P, G):
            st = states[pc.tensor]
            s = slice(pc.start, pc.start + pc.numel)
            a = slice(pc.first_block, pc.first_block + pc.n_blocks)
            pieces.append(bq.TensorState(pv, gv, st["s1"][s], st["s2"][s], None if st["a1"] is None else st["a1"][a],
                                         None if st["a2"] is None else st["a2"][a]))
        bq.bnbq_step_8bit("adamw", pieces, step=3, code1=c1.to(DEV), code2=c2.to(DEV), blocksize=B, **HP)
        ex.all_gather_params(P)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    for i, (st, h) in enumerate(zip(states, host)):
        np.testing.assert_array_equal(parity.to_np(ex.views(P, i)), h["p"])
        for k in ("s1", "s2", "a1", "a2"):
            if st[k] is not None:
                np.testing.assert_array_equal(parity.to_np(st[k]), h[k])
    assert bq.bnbq_device_flags(clear=True) == 0
