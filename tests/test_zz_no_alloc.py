"""eaga_forward_noalloc against eaga_forward.

eaga_forward_noalloc is the forward for callers that cannot allocate device
memory for scratch (a plain C client that links the library but no device
allocator, or code under a framework whose memory pool only hands out the
tensors it owns).  It keeps the forward's small scratch in a fixed array
inside the library instead of a caller workspace.  These tests call it
through the C ABI twice in a row, each time on fresh inputs, and compare its
outputs with those of eaga_forward on the same inputs, within the parity
tolerance of the other GPU tests.

The file is named to be collected last, so that a run stopping at the first
failure has already run every other test; it passes on its own in a fresh
process as well as after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

from edge_aware_graph_b200 import eaga
from edge_aware_graph_b200 import inputs as I
from edge_aware_graph_b200.buffers import LayerBuffers

from harness import TOL, custom_case, rel_err

pytestmark = pytest.mark.gpu


def _case(name, seed):
    if name == "sbm2":
        p = I.preset("sbm", B=2, seed=seed)
        return p, I.draw_inputs(p, with_grads=False), I.draw_weights(p)
    if name == "tiny":
        p = I.preset("tiny", seed=seed)
        return p, I.draw_inputs(p, with_grads=False), I.draw_weights(p)
    return custom_case(3, 40, 64, 16, 8, 2, 16, "bf16", seed=seed, mask="random", with_grads=False)


def _compare(buf, p):
    """Run eaga_forward, then eaga_forward_noalloc into outputs poisoned with NaN."""
    buf.forward()
    torch.cuda.synchronize()
    ref = {"Xout": buf.Xout.clone(), "Eout": buf.Eout.clone()}
    ref_sv = {k: v.clone() for k, v in buf.saved_parts().items()}
    buf.Xout.fill_(float("nan"))
    buf.Eout.fill_(float("nan"))
    buf.saved.zero_()
    eaga.forward_noalloc(buf.dims, buf.X, buf.E, buf.y, buf.M, buf.W, buf.Xout, buf.Eout, buf.saved)
    torch.cuda.synchronize()
    tol = TOL[p.dtype]
    for k in ("Xout", "Eout"):
        got = getattr(buf, k)
        assert torch.isfinite(got.float()).all(), k
        assert rel_err(got, ref[k].float().cpu().numpy()) <= tol, k
    sv = buf.saved_parts()
    for k in ("Q", "K", "V", "O"):
        assert rel_err(sv[k], ref_sv[k].float().cpu().numpy()) <= tol, k
    lse, lse_ref = sv["LSE"].cpu().numpy(), ref_sv["LSE"].cpu().numpy()
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin)
    if fin.any():
        assert np.abs(lse[fin] - lse_ref[fin]).max() <= tol * np.abs(lse_ref[fin]).max()


@pytest.mark.parametrize("name", ["sbm2", "tiny", "ragged"])
def test_noalloc_forward_matches_forward_twice(name):
    p, d, W = _case(name, 21)
    buf = LayerBuffers(p.B, p.n, p.dx, p.de, p.dy, p.H, p.dh, dtype=p.dtype, backward=False)
    buf.load_inputs(d, W)
    _compare(buf, p)
    # second call in a row, on other inputs: the fixed scratch keeps the first
    # call's contents and must not leak into the result
    _, d2, W2 = _case(name, 22)
    buf.load_inputs(d2, W2)
    _compare(buf, p)


def test_noalloc_rejects_too_many_graphs():
    L = eaga.lib()
    d = eaga.dims(100000, 8, 64, 64, 64, 8, 32, "bf16")   # g alone needs 6.4 MB > 64 KiB
    fake = ctypes.c_void_p(0x100000)
    w = eaga.Weights(*([0x100000] * 12))
    rc = L.eaga_forward_noalloc(ctypes.byref(d), fake, fake, fake, fake, ctypes.byref(w), fake, fake, fake, None)
    assert rc == 2   # EAGA_ERR_UNSUPPORTED, nothing launched
