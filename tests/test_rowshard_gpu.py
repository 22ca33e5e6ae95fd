"""GPU check of the row-sharded layer (eaga_forward_rows, eaga_backward_rows):
the ranks of a row-sharded run are emulated one after another on one GPU (they
do not wait on one another: the forward has no exchange and the backward's
only exchange, the sum of the parts, is done here on the host).

Against the whole-layer calls on the same inputs:
  - each slab's E' rows, X' rows and saved O, LSE rows are bitwise the whole
    layer's (the same kernels on the same row blocks);
  - each slab's dE rows are bitwise the whole layer's dE rows (dE depends on
    the row's own statistics, not on the dk, dv sums over row blocks);
  - the parts of dX, dy and the weight gradients, summed over the slabs, match
    the oracle's gradients of the whole layer within the bf16 parity tolerance
    (each part carries its own bf16 roundings of dX, dy and of the dk, dv
    sums, so the sum is not bitwise the whole layer's; it is within 1e-2 of
    each one's scale of it as well).
"""
import numpy as np
import pytest
import torch

from edge_aware_graph_b200 import eaga, rowshard
from edge_aware_graph_b200 import inputs as I
from edge_aware_graph_b200.buffers import LayerBuffers

from harness import TOL, custom_case, oracle_backward, rel_err

pytestmark = pytest.mark.gpu


def _slab(t, row0, rows):
    return t[:, row0:row0 + rows].contiguous()


@pytest.mark.parametrize("case", [
    (4, 192, "prefix", 2),      # SBM-sized slabs of 96 rows
    (4, 192, "blocks", 3),      # three slabs of 64, with rows and chunks without valid pairs
    (2, 544, "random", 2),      # slabs of 272 rows, columns over clusters of 4 CTAs
    (1, 1024, "prefix", 4),     # a Large-sized graph over four slabs of 256 rows
    (3, 100, "random", 2),      # the last slab ends at n (52 rows, a partial row block)
], ids=lambda c: f"B{c[0]}-n{c[1]}-{c[2]}-x{c[3]}")
def test_row_slabs_match_the_whole_layer(oracle_lib, case):
    B, n, mask, world = case
    p, d, W = custom_case(B, n, 256, 64, 64, 8, 32, "bf16", seed=70 + n, mask=mask)
    full = LayerBuffers(B, n, 256, 64, 64, 8, 32, dtype="bf16", backward=True)
    full.load_inputs(d, W)
    full.forward()
    full.backward()
    torch.cuda.synchronize()
    ref_saved = full.saved_parts()

    rk = LayerBuffers(B, n, 256, 64, 64, 8, 32, dtype="bf16", backward=True)   # node tensors, saved, workspaces
    rk.load_inputs(d, W)
    dX_sum = torch.zeros(B, n, 256, dtype=torch.float32, device="cuda")
    dy_sum = torch.zeros(B, 64, dtype=torch.float32, device="cuda")
    dW_sum = torch.zeros_like(rk.dW_flat)
    for row0, rows in rowshard.row_slabs(n, world):
        if rows == 0:
            continue
        E_r, dEo_r = _slab(full.E, row0, rows), _slab(full.dEout, row0, rows)
        Eout_r, dE_r = torch.empty_like(E_r), torch.empty_like(E_r)
        rowshard.forward_rows(rk.dims, row0, rows, rk.X, E_r, rk.y, rk.M, rk.W, rk.Xout, Eout_r, rk.saved,
                              rk.ws_fwd)
        torch.cuda.synchronize()
        sv = rk.saved_parts()
        assert torch.equal(Eout_r, _slab(full.Eout, row0, rows))
        assert torch.equal(_slab(rk.Xout, row0, rows), _slab(full.Xout, row0, rows))
        assert torch.equal(_slab(sv["O"], row0, rows), _slab(ref_saved["O"], row0, rows))
        assert torch.equal(sv["LSE"][:, :, row0:row0 + rows], ref_saved["LSE"][:, :, row0:row0 + rows])
        rk.dW_flat.fill_(float("nan"))
        rowshard.backward_rows(rk.dims, row0, rows, rk.X, E_r, rk.y, rk.M, rk.W, rk.saved, full.dXout, dEo_r,
                               rk.dX, dE_r, rk.dy, rk.dW, rk.ws_bwd)
        torch.cuda.synchronize()
        assert torch.equal(dE_r, _slab(full.dE, row0, rows))
        dX_sum += rk.dX.float()
        dy_sum += rk.dy.float()
        dW_sum += torch.nan_to_num(rk.dW_flat, nan=0.0)   # (padding between the flat views)

    sums = {"dX": dX_sum, "dy": dy_sum}
    for k in I.WEIGHT_NAMES:
        a = dW_sum[(full.dW[k].data_ptr() - full.dW_flat.data_ptr()) // 4:][:full.dW[k].numel()]
        sums["d" + k] = a.view(full.dW[k].shape)
    whole = {"dX": full.dX, "dy": full.dy}
    whole.update({"d" + k: full.dW[k] for k in I.WEIGHT_NAMES})
    ref = oracle_backward(oracle_lib, p, d, W)
    errs = {k: rel_err(v, ref[k]) for k, v in sums.items()}
    bad = {k: v for k, v in errs.items() if not v <= TOL["bf16"]}
    assert not bad, f"summed parts vs the oracle: {bad} (all: {errs})"
    errs = {k: rel_err(v, whole[k].float().cpu().numpy()) for k, v in sums.items()}
    bad = {k: v for k, v in errs.items() if not v <= 1e-2}
    assert not bad, f"summed parts vs the whole layer: {bad} (all: {errs})"


def test_slab_arguments_are_checked():
    p, d, W = custom_case(2, 64, 256, 64, 64, 8, 32, "bf16", seed=3, mask="random")
    rk = LayerBuffers(2, 64, 256, 64, 64, 8, 32, dtype="bf16", backward=False)
    rk.load_inputs(d, W)
    E_r = _slab(rk.E, 8, 16)
    for row0, rows in [(4, 16), (8, 12), (56, 16), (8, 0), (-8, 16)]:
        with pytest.raises(eaga.EagaError) as ei:
            eaga.forward_rows(rk.dims, row0, rows, rk.X, E_r, rk.y, rk.M, rk.W, rk.Xout, torch.empty_like(E_r),
                              rk.saved, rk.ws_fwd)
        assert ei.value.code == 1, (row0, rows)          # EAGA_ERR_INVALID_ARG
    # the CUDA-core path (fp32) has no row slabs
    p32, d32, W32 = custom_case(2, 16, 16, 8, 8, 2, 8, "fp32", seed=1, mask="full", with_grads=False)
    b32 = LayerBuffers(2, 16, 16, 8, 8, 2, 8, dtype="fp32", backward=False)
    b32.load_inputs(d32, W32)
    E32 = _slab(b32.E, 0, 8)
    with pytest.raises(eaga.EagaError) as ei:
        eaga.forward_rows(b32.dims, 0, 8, b32.X, E32, b32.y, b32.M, b32.W, b32.Xout, torch.empty_like(E32),
                          b32.saved, b32.ws_fwd)
    assert ei.value.code == 2                           # EAGA_ERR_UNSUPPORTED
