"""The multi-rank (N > 1) path on CPU: two gloo ranks, no GPU.

The layer shards over graphs with no exchange on the data path; a training
step adds one collective, the sum of the weight gradients over ranks.  These
tests run the plumbing that bench.py uses under torchrun
(edge_aware_graph_b200/dp.py) in two spawned processes, and check with the
oracle that the summed per-rank weight gradients equal those of the whole
batch (the gradient of a sum over graphs is the sum of the per-graph
gradients), and that the per-rank batches differ while the weights agree.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from edge_aware_graph_b200 import dp
from edge_aware_graph_b200 import inputs as I

WORLD = 2
GRAD_KEYS = ("Wq", "bq", "Wk", "bk", "Wv", "bv", "Wfe", "Wfy", "bf", "We", "Wo", "bo")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=timedelta(seconds=60))


def _plumbing_worker(rank, port, q):
    _init(rank, port)
    try:
        flat = torch.full((1000,), float(rank + 1), dtype=torch.float32)
        dp.allreduce_weight_grads(flat)
        ms = dp.max_over_ranks(1.5 + rank)
        p = I.preset("tiny", seed=dp.rank_seed(I.preset("tiny").seed, rank))
        d = I.draw_inputs(p, with_grads=True)
        W = I.draw_weights(I.preset("tiny"))
        q.put((rank, float(flat.min()), float(flat.max()), ms, float(np.abs(d["E"]).sum()),
               float(np.abs(W["Wq"]).sum())))
    finally:
        dist.destroy_process_group()


def _grad_worker(rank, port, q):
    import oracle
    _init(rank, port)
    try:
        p = I.preset("tiny")
        d = I.draw_inputs(p, with_grads=True)
        W = I.draw_weights(p)
        sl = {k: d[k][rank:rank + 1] for k in ("X", "E", "y", "M", "dXout", "dEout")}
        g = oracle.backward(dict(H=p.H, dh=p.dh), sl["X"], sl["E"], sl["y"], sl["M"], W, sl["dXout"], sl["dEout"])
        flat = torch.from_numpy(np.concatenate([np.asarray(g["d" + k], np.float64).ravel() for k in GRAD_KEYS]))
        dp.allreduce_weight_grads(flat)
        q.put((rank, flat.numpy()))
    finally:
        dist.destroy_process_group()


def _run(worker):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=worker, args=(r, port, q)) for r in range(WORLD)]
    for pr in procs:
        pr.start()
    out = [q.get(timeout=120) for _ in range(WORLD)]
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    return sorted(out, key=lambda x: x[0])


def test_two_rank_plumbing():
    out = _run(_plumbing_worker)
    for rank, lo, hi, ms, esum, wsum in out:
        assert lo == hi == 3.0            # 1 + 2 summed over the two ranks
        assert ms == 2.5                  # max over ranks, seen by both
    assert out[0][4] != out[1][4]         # distinct graphs per rank
    assert out[0][5] == out[1][5]         # one model: identical weights


def test_two_rank_weight_grads_match_whole_batch():
    import oracle
    oracle.build()
    out = _run(_grad_worker)
    p = I.preset("tiny")
    d = I.draw_inputs(p, with_grads=True)
    W = I.draw_weights(p)
    g = oracle.backward(dict(H=p.H, dh=p.dh), d["X"], d["E"], d["y"], d["M"], W, d["dXout"], d["dEout"])
    whole = np.concatenate([np.asarray(g["d" + k], np.float64).ravel() for k in GRAD_KEYS])
    for _, flat in out:
        np.testing.assert_allclose(flat, whole, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("workload", ["sbm-train", "planar-sample"])
def test_reference_arm_under_torchrun(workload):
    """bench.py --impl reference launched as the multi-GPU runs are: rank 0
    alone runs the oracle arm and prints one JSON line; the other rank exits 0."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(WORLD),
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", str(WORLD), "--steps", "1", "--warmup", "3", "--ref-graphs", "1", "--workload", workload]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, OMP_NUM_THREADS="2"))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["n_gpus"] == WORLD and out["value"] > 0
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["cpu_baseline"]["kind"] == "oracle"
