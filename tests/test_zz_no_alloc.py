"""eaga_forward_noalloc against eaga_forward.

eaga_forward_noalloc is the forward for callers that cannot allocate device
memory for scratch (a plain C client that links the library but no device
allocator, or code under a framework whose memory pool only hands out the
tensors it owns).  It keeps the forward's small scratch in a fixed array
inside the library instead of a caller workspace.  These tests call it
through the C ABI twice in a row, each time on fresh inputs, and compare its
outputs with those of eaga_forward on the same inputs.  Both entry points run
the same kernels on the same inputs, so the outputs must be bit-identical,
which also shows that nothing left in the shared scratch by an earlier call
reaches a later result.  Further tests check that repeated calls allocate
no device memory and that the call's status word can be read (and that a
bounded wait that runs out is reported through it).

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

from harness import custom_case

pytestmark = pytest.mark.gpu


def _case(name, seed):
    if name == "sbm2":
        p = I.preset("sbm", B=2, seed=seed)
        return p, I.draw_inputs(p, with_grads=False), I.draw_weights(p)
    if name == "tiny":
        p = I.preset("tiny", seed=seed)
        return p, I.draw_inputs(p, with_grads=False), I.draw_weights(p)
    if name == "manygraphs":
        # specialised path, B = 800 graphs of n = 16: the status word, g and
        # the operand images fit the 64 KiB array (256 + 51200 + 8192 bytes)
        # but the pair kernel's row-block order (6400 bytes more) does not, so
        # the no-allocation call takes the row blocks in index order while
        # eaga_forward takes them longest first: the results must not differ
        return custom_case(800, 16, 64, 64, 16, 8, 32, "bf16", seed=seed, mask="random", with_grads=False)
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
    for k in ("Xout", "Eout"):
        assert torch.equal(getattr(buf, k), ref[k]), k
    sv = buf.saved_parts()
    for k in ("Q", "K", "V", "O", "LSE"):
        assert torch.equal(sv[k], ref_sv[k]), k
    assert eaga.get_device_status(None) == 0


@pytest.mark.parametrize("name", ["sbm2", "tiny", "ragged", "manygraphs"])
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


def test_noalloc_allocates_no_device_memory():
    """After a first call (library load, the scratch address lookup), repeated
    no-allocation calls leave the device's free memory and torch's
    allocations unchanged."""
    p, d, W = _case("sbm2", 31)
    buf = LayerBuffers(p.B, p.n, p.dx, p.de, p.dy, p.H, p.dh, dtype=p.dtype, backward=False)
    buf.load_inputs(d, W)
    eaga.forward_noalloc(buf.dims, buf.X, buf.E, buf.y, buf.M, buf.W, buf.Xout, buf.Eout, buf.saved)
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(4):
        eaga.forward_noalloc(buf.dims, buf.X, buf.E, buf.y, buf.M, buf.W, buf.Xout, buf.Eout, buf.saved)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0


def test_noalloc_status_word_reports_a_timeout():
    """The status word of the no-allocation forward lives in the fixed array;
    eaga_get_device_status(NULL) reads (and clears) it.  The bounded-wait
    probe pointed at it (workspace NULL) makes a wait run out; the timeout is
    reported there, the next read is clean, and a following call runs
    normally and reports no timeout."""
    p, d, W = _case("ragged", 41)
    buf = LayerBuffers(p.B, p.n, p.dx, p.de, p.dy, p.H, p.dh, dtype=p.dtype, backward=False)
    buf.load_inputs(d, W)
    eaga.forward_noalloc(buf.dims, buf.X, buf.E, buf.y, buf.M, buf.W, buf.Xout, buf.Eout, buf.saved)
    assert eaga.get_device_status(None) == 0
    eaga.debug_wait_probe(None, 2000)
    torch.cuda.synchronize()
    assert eaga.get_device_status(None) == 6            # EAGA_ERR_TIMEOUT
    assert eaga.get_device_status(None) == 0            # reading it cleared it
    eaga.forward_noalloc(buf.dims, buf.X, buf.E, buf.y, buf.M, buf.W, buf.Xout, buf.Eout, buf.saved)
    assert eaga.get_device_status(None) == 0


def test_noalloc_argument_errors_match_forward():
    """Invalid dims give EAGA_ERR_INVALID_ARG, as eaga_forward does; checked on
    the host before anything is launched."""
    L = eaga.lib()
    fake = ctypes.c_void_p(0x100000)
    w = eaga.Weights(*([0x100000] * 12))
    for bad in (eaga.dims(0, 8, 64, 64, 64, 8, 32, "bf16"), eaga.dims(2, 0, 64, 64, 64, 8, 32, "bf16"),
                eaga.Dims(2, 8, 64, 64, 64, 8, 32, 7)):
        rc = L.eaga_forward_noalloc(ctypes.byref(bad), fake, fake, fake, fake, ctypes.byref(w), fake, fake, fake,
                                    None)
        rf = L.eaga_forward(ctypes.byref(bad), fake, fake, fake, fake, ctypes.byref(w), fake, fake, fake, fake,
                            1 << 20, None)
        assert rc == rf == 1
