"""The row-sharded path's host logic on CPU: slab bounds, and two gloo ranks
whose parts of the backward sum to the whole layer's gradients.

A rank owns a slab of each graph's rows and computes the gradients of
L_r = <dX', X'> + <dE', E'> restricted to its rows (dX', dE' zero outside the
slab).  The layer is linear in its upstream gradients, so the parts summed
over ranks (edge_aware_graph_b200/rowshard.py's all-reduce) must equal the
whole layer's gradients, and each rank's dE rows must equal the whole dE on
those rows.  The oracle computes each part; the ranks exchange them over gloo.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from edge_aware_graph_b200 import inputs as I
from edge_aware_graph_b200 import rowshard

WORLD = 2
GRAD_KEYS = ("dX", "dy") + tuple("d" + k for k in I.WEIGHT_NAMES)


@pytest.mark.parametrize("n,world", [(12, 2), (16, 2), (192, 3), (1024, 2), (1024, 8), (30, 4), (2, 2), (100, 16)])
def test_row_slabs_cover_the_rows(n, world):
    slabs = rowshard.row_slabs(n, world)
    assert len(slabs) == world
    covered = []
    for row0, rows in slabs:
        assert rows >= 0
        if rows:          # an empty slab (a rank past the last row block) computes nothing
            assert row0 % 8 == 0 and (rows % 8 == 0 or row0 + rows == n)
        covered += list(range(row0, row0 + rows))
    assert covered == list(range(n))


def test_mask_rows():
    t = torch.arange(2 * 12 * 3, dtype=torch.float64).reshape(2, 12, 3)
    m = rowshard.mask_rows(t, 8, 4)
    assert torch.equal(m[:, 8:], t[:, 8:]) and torch.all(m[:, :8] == 0)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    p = I.preset("tiny", n=16)
    d = I.draw_inputs(p, with_grads=True)
    d["M"][0, 13:] = 0          # graph 0: 13 nodes (a slab with padding rows)
    return p, d, I.draw_weights(p)


def _worker(rank, port, q):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=timedelta(seconds=60))
    try:
        p, d, W = _case()
        row0, rows = rowshard.row_slabs(p.n, WORLD)[rank]
        dXo = rowshard.mask_rows(torch.from_numpy(np.asarray(d["dXout"], np.float64)), row0, rows).numpy()
        dEo = rowshard.mask_rows(torch.from_numpy(np.asarray(d["dEout"], np.float64)), row0, rows).numpy()
        g = oracle.backward(dict(H=p.H, dh=p.dh), d["X"], d["E"], d["y"], d["M"], W, dXo, dEo)
        parts = [torch.from_numpy(np.ascontiguousarray(g[k], np.float64)) for k in GRAD_KEYS]
        rowshard.allreduce_parts(parts)
        dE_rows = np.asarray(g["dE"], np.float64)[:, row0:row0 + rows]
        q.put((rank, row0, rows, [t.numpy() for t in parts], dE_rows))
    finally:
        dist.destroy_process_group()


def test_two_rank_row_parts_sum_to_the_whole_layer():
    import oracle
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
    p, d, W = _case()
    whole = oracle.backward(dict(H=p.H, dh=p.dh), d["X"], d["E"], d["y"], d["M"], W, d["dXout"], d["dEout"])
    for rank, row0, rows, parts, dE_rows in out:
        assert rows > 0
        for k, v in zip(GRAD_KEYS, parts):
            np.testing.assert_allclose(v, np.asarray(whole[k], np.float64), rtol=1e-9, atol=1e-11, err_msg=k)
        np.testing.assert_allclose(dE_rows, np.asarray(whole["dE"], np.float64)[:, row0:row0 + rows],
                                   rtol=1e-12, atol=1e-14)
