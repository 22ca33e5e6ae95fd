"""CPU checks of the C ABI: the library loads, exports every declared entry
point, and its host-side validation returns the documented codes without
touching a GPU (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from edge_aware_graph_b200 import build as B
from edge_aware_graph_b200 import eaga

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    B.build()
    return eaga.lib()


def declared_symbols():
    out = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            out += re.findall(r"EAGA_API\s+[\w\s\*]+?\b(eaga_\w+)\s*\(", txt)
    return sorted(set(out))


def test_exports_every_declared_symbol(L):
    syms = declared_symbols()
    assert len(syms) >= 7
    for s in syms:
        assert hasattr(L, s), s
    assert set(eaga.EXPORTED) <= set(syms)


def good_dims():
    return eaga.dims(32, 192, 256, 64, 64, 8, 32, "bf16")


def test_sizes(L):
    d = good_dims()
    ws_f, ws_b, sv = eaga.workspace_size(d, False), eaga.workspace_size(d, True), eaga.saved_size(d)
    assert ws_f > 0 and ws_b > 0 and sv > 0
    # saved: LSE [B,H,n] fp32 + Q,K,V,O [B,n,256] bf16
    assert sv >= 32 * 8 * 192 * 4 + 4 * 32 * 192 * 256 * 2
    # forward: no B*H*n^2 term, doubling n at fixed B*n leaves it about the same
    d2 = eaga.dims(16, 384, 256, 64, 64, 8, 32, "bf16")
    assert eaga.workspace_size(d2, False) < 1.2 * ws_f
    # backward: node terms plus a and ds in bf16, 32 bytes per pair (a quarter of E)
    pairs = 32 * 192 * 192
    assert 32 * pairs <= ws_b < 32 * pairs + 64 * 32 * 192 * 256
    big = eaga.dims(4, 1024, 256, 64, 64, 8, 32, "bf16")
    assert eaga.workspace_size(big, True) < 32 * 4 * 1024 * 1024 + 64 * 4 * 1024 * 256


@pytest.mark.parametrize("field,value,code", [
    ("n", 0, 1), ("B", -1, 1), ("dtype", 7, 1),
    ("n", 1025, 2), ("de", 12, 2), ("dh", 12, 2), ("H", 17, 2), ("dx", 1032, 2),
])
def test_bad_dims(L, field, value, code):
    d = good_dims()
    setattr(d, field, value)
    assert eaga.workspace_size(d, True) == 0
    fake = ctypes.c_void_p(0x100000)
    w = eaga.Weights(*([0x100000] * 12))
    rc = L.eaga_forward(ctypes.byref(d), fake, fake, fake, fake, ctypes.byref(w), fake, fake, None, fake, 1 << 40,
                        None)
    assert rc == code


def test_null_and_misaligned_and_workspace(L):
    d = good_dims()
    ok = ctypes.c_void_p(0x100000)
    w = eaga.Weights(*([0x100000] * 12))
    big = eaga.workspace_size(d, False)
    f = L.eaga_forward
    assert f(None, ok, ok, ok, ok, ctypes.byref(w), ok, ok, None, ok, big, None) == 1
    assert f(ctypes.byref(d), None, ok, ok, ok, ctypes.byref(w), ok, ok, None, ok, big, None) == 1
    assert f(ctypes.byref(d), ctypes.c_void_p(0x100008), ok, ok, ok, ctypes.byref(w), ok, ok, None, ok, big,
             None) == 3
    w_bad = eaga.Weights(*([0x100000] * 11 + [0x100004]))
    assert f(ctypes.byref(d), ok, ok, ok, ok, ctypes.byref(w_bad), ok, ok, None, ok, big, None) == 3
    assert f(ctypes.byref(d), ok, ok, ok, ok, ctypes.byref(w), ok, ok, None, ok, big - 1, None) == 4
    g = L.eaga_backward
    bigb = eaga.workspace_size(d, True)
    assert g(ctypes.byref(d), ok, ok, ok, ok, ctypes.byref(w), ok, ok, ok, ok, ok, ok, None, ok, bigb, None) == 1
    assert g(ctypes.byref(d), ok, ok, ok, ok, ctypes.byref(w), ok, ok, ok, ok, ok, ok, ctypes.byref(w), ok,
             bigb - 1, None) == 4


def test_strerror(L):
    for code in range(7):
        assert eaga.strerror(code)
    assert eaga.strerror(99) == "unknown status"


def test_wait_probe_arguments(L):
    # argument checks happen on the host, before any launch
    assert L.eaga_debug_wait_probe(None, 100, None) == 1           # EAGA_ERR_INVALID_ARG
    fake = ctypes.c_void_p(0x100000)
    assert L.eaga_debug_wait_probe(fake, 0, None) == 1
    assert L.eaga_debug_wait_probe(fake, (1 << 24) + 1, None) == 1
    assert L.eaga_debug_wait_probe(ctypes.c_void_p(0x100008), 100, None) == 3   # misaligned


def test_binding_refuses_host_tensors(L):
    # the binding checks every tensor before a pointer reaches the library: a
    # host tensor would otherwise be read as device memory
    import torch
    d = eaga.dims(2, 12, 16, 8, 8, 2, 8, "fp32")
    t = lambda *s: torch.zeros(*s, dtype=torch.float32)
    W = {k: t(4) for k in eaga.WEIGHT_NAMES}
    M = torch.zeros(2, 12, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        eaga.forward(d, t(2, 12, 16), t(2, 12, 12, 8), t(2, 8), M, W, t(2, 12, 16), t(2, 12, 12, 8),
                     None, torch.zeros(64, dtype=torch.uint8))
    with pytest.raises(ValueError, match="CUDA tensor"):
        eaga.get_device_status(torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(ValueError, match="CUDA tensor"):
        eaga.debug_wait_probe(torch.zeros(16, dtype=torch.uint8), 100)


@pytest.mark.parametrize("dims,fast", [
    ((32, 192, 256, 64, 64, 8, 32, "bf16"), True),      # the SBM-shaped workload
    ((64, 64, 256, 64, 64, 8, 32, "bf16"), True),       # Planar / Tree shaped
    ((4, 1024, 256, 64, 64, 8, 32, "bf16"), True),      # Large shaped
    ((2, 2, 64, 64, 8, 8, 32, "bf16"), True),           # smallest n, narrowest dx
    ((2, 96, 576, 64, 64, 8, 32, "bf16"), True),        # dx a multiple of 64 only
    ((32, 192, 256, 64, 64, 8, 32, "fp32"), False),     # fp32 storage
    ((2, 191, 256, 64, 64, 8, 32, "bf16"), False),      # odd n
    ((2, 96, 72, 64, 64, 8, 32, "bf16"), False),        # dx not a multiple of 64
    ((2, 96, 256, 32, 64, 8, 32, "bf16"), False),       # de != 64
    ((2, 96, 256, 64, 64, 4, 32, "bf16"), False),       # H != 8
    ((2, 96, 256, 64, 64, 8, 16, "bf16"), False),       # dh != 32
])
def test_dispatch_rule(L, dims, fast):
    # the tcgen05 path (4 forward, 11 backward launches) takes bf16, de = 64,
    # H = 8, dh = 32, n even, dx a multiple of 64; every other supported shape
    # runs the CUDA-core kernels (4 and 10)
    d = eaga.dims(*dims)
    assert (eaga.kernel_launches(d, False), eaga.kernel_launches(d, True)) == ((4, 11) if fast else (4, 10))


def test_dispatch_rejects_unsupported(L):
    assert eaga.kernel_launches(eaga.dims(2, 1025, 256, 64, 64, 8, 32, "bf16"), False) == -1
    assert eaga.kernel_launches(eaga.dims(0, 64, 256, 64, 64, 8, 32, "bf16"), False) == -1
