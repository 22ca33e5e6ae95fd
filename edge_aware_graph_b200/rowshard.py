"""Row-sharded layer: the rows of each graph split over the ranks of a process
group (one large graph's pairs over several GPUs; the AI-summary page's method
paragraph notes the edge update stays quadratic, so large graphs need their
pairs split).

Each rank owns a slab of rows [row0, row0 + rows) of every graph and holds the
[B, rows, n, de] slabs of E, E' and of their gradients; node tensors (X, y,
M, the weights) are whole on every rank.

  forward   eaga_forward_rows: every rank computes Q, K, V of all nodes (a node
            GEMM, cheaper than exchanging them) and the pairs of its rows.  No
            exchange.  The slab's rows of X' are the rank's.
  backward  eaga_backward_rows with dX' zero outside the slab gives the rank's
            part of dX, dy and the weight gradients (the layer is linear in its
            upstream gradients); one all-reduce sums the parts.  dE of the
            slab is final.

Only host logic lives here (slab bounds, the masking of dX', the sum); the
arithmetic runs in the library's kernels.
"""
from __future__ import annotations

from . import eaga


def row_slabs(n: int, world: int) -> list:
    """(row0, rows) of each rank: whole row blocks of 8, the last slab ending
    at n; ranks past the last row block get (n, 0) and compute nothing."""
    blocks = (n + 7) // 8
    per = (blocks + world - 1) // world
    out = []
    for r in range(world):
        b0, b1 = min(blocks, r * per), min(blocks, (r + 1) * per)
        row0, row1 = min(n, 8 * b0), min(n, 8 * b1)
        out.append((row0, row1 - row0))
    return out


def mask_rows(t, row0: int, rows: int):
    """A copy of a [B, n, ...] node tensor that is zero outside rows row0 .. row0+rows-1."""
    out = t.new_zeros(t.shape)
    if rows > 0:
        out[:, row0:row0 + rows] = t[:, row0:row0 + rows]
    return out


def allreduce_parts(tensors, group=None):
    """Sum each rank's part of the gradients (in place, fp32) over the group."""
    import torch.distributed as dist
    for t in tensors:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


def forward_rows(dims, row0, rows, X, E_rows, y, M, W, Xout, Eout_rows, saved, workspace, stream=None,
                 variant="layer"):
    """This rank's slab of the forward (no exchange)."""
    if rows > 0:
        eaga.forward_rows(dims, row0, rows, X, E_rows, y, M, W, Xout, Eout_rows, saved, workspace, stream, variant)


def backward_rows(dims, row0, rows, X, E_rows, y, M, W, saved, dXout, dEout_rows, dX, dE_rows, dy, dW, workspace,
                  stream=None, variant="layer"):
    """This rank's part of the backward: dXout is masked to the slab here;
    dX, dy and dW then hold the rank's part (zero on a rank without rows)."""
    if rows > 0:
        eaga.backward_rows(dims, row0, rows, X, E_rows, y, M, W, saved, mask_rows(dXout, row0, rows), dEout_rows,
                           dX, dE_rows, dy, dW, workspace, stream, variant)
    else:
        dX.zero_()
        dy.zero_()
        for t in dW.values():
            t.zero_()
