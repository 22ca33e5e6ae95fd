"""The graph-transformer block under data parallelism, on CPU: two gloo ranks.

Graphs are independent, so a block's weight gradients over a batch are the
sums of its per-graph gradients (the global update pools within a graph
only).  Each rank computes the block oracle's gradients of its half of the
batch; the sum over ranks through dp.allreduce_weight_grads (the collective
bench.py runs under torchrun) must equal the whole batch's gradients.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from edge_aware_graph_b200 import dp
from edge_aware_graph_b200 import inputs as I

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    p = I.preset("tiny", B=4, n=10)
    d = I.draw_inputs(p, with_grads=True)
    d["M"][1, 6:] = 0
    d["M"][3, :] = 0               # a graph without nodes
    return p, d, I.draw_weights(p), I.draw_block_weights(p), I.draw_block_upstream(p)


def _keys():
    return tuple("d" + k for k in I.WEIGHT_NAMES) + tuple("d" + k for k in I.BLOCK_WEIGHT_NAMES)


def _worker(rank, port, q):
    from oracle import block as OB
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=timedelta(seconds=60))
    try:
        p, d, W, Wb, dyo = _case()
        sl = slice(2 * rank, 2 * rank + 2)
        g = OB.block_backward(dict(H=p.H, dh=p.dh), d["X"][sl], d["E"][sl], d["y"][sl], d["M"][sl], W, Wb,
                              d["dXout"][sl], d["dEout"][sl], dyo[sl])
        flat = torch.from_numpy(np.concatenate([np.ravel(np.asarray(g[k], np.float64)) for k in _keys()]))
        dp.allreduce_weight_grads(flat)
        q.put((rank, flat.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_rank_block_gradients_sum_to_the_whole_batch():
    import oracle
    from oracle import block as OB
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for pr in procs:
        pr.start()
    out = sorted([q.get(timeout=120) for _ in range(WORLD)], key=lambda x: x[0])
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    p, d, W, Wb, dyo = _case()
    g = OB.block_backward(dict(H=p.H, dh=p.dh), d["X"], d["E"], d["y"], d["M"], W, Wb, d["dXout"], d["dEout"], dyo)
    whole = np.concatenate([np.ravel(np.asarray(g[k], np.float64)) for k in _keys()])
    for rank, flat in out:
        np.testing.assert_allclose(flat, whole, rtol=1e-10, atol=1e-12)
