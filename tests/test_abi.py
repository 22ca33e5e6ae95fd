"""CPU checks of the C ABI: the library loads, exports every declared entry
point, and its host-side validation returns the documented codes without
touching a GPU (no compute call is made here)."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

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
    # backward: no per-pair term either.  With the node count B*n fixed, going
    # from n = 192 to n = 1024 multiplies the pairs by 5.3 and leaves the
    # workspace about the same; it stays a few dozen bytes per node feature
    for dd in ((32, 192), (6, 1024), (192, 32), (64, 96)):
        db = eaga.dims(dd[0], dd[1], 256, 64, 64, 8, 32, "bf16")
        nodes = dd[0] * dd[1]
        assert eaga.workspace_size(db, True) < 24 * nodes * 256 + (8 << 20), dd
    d3 = eaga.dims(6, 1024, 256, 64, 64, 8, 32, "bf16")      # 6144 nodes, as the SBM batch
    assert eaga.workspace_size(d3, True) < 1.2 * ws_b
    # at fixed B, doubling n (four times the pairs) at most doubles it
    for n in (64, 256, 512):
        w1 = eaga.workspace_size(eaga.dims(4, n, 256, 64, 64, 8, 32, "bf16"), True)
        w2 = eaga.workspace_size(eaga.dims(4, 2 * n, 256, 64, 64, 8, 32, "bf16"), True)
        assert w2 <= 2.05 * w1, n


def test_block_sizes(L):
    """The graph-transformer block's saved state and workspaces grow with the
    node count only: the second difference over n = 256, 512, 768 at fixed B
    (a per-pair term c B n^2 would leave 2 c B 256^2 there) is alignment only."""
    f = lambda n, fb: eaga.block_workspace_size(eaga.dims(4, n, 256, 64, 64, 8, 32, "bf16"), fb)
    s = lambda n: eaga.block_saved_size(eaga.dims(4, n, 256, 64, 64, 8, 32, "bf16"))
    for g in (lambda n: f(n, False), lambda n: f(n, True), s):
        a, b, c = g(256), g(512), g(768)
        assert a > 0 and b > a and c > b
        assert abs(c - 2 * b + a) < 64 * 1024
    d = good_dims()
    assert eaga.block_saved_size(d) > eaga.saved_size(d)
    assert eaga.block_workspace_size(d, True) > eaga.workspace_size(d, True)
    # unsupported: fp32, de != 64, dx not 256 or 512, dy not a multiple of 32
    for bad in (eaga.dims(2, 16, 16, 8, 8, 2, 8, "fp32"), eaga.dims(4, 64, 128, 64, 64, 8, 32, "bf16"),
                eaga.dims(4, 64, 256, 64, 48, 8, 32, "bf16")):
        assert eaga.block_workspace_size(bad, False) == 0 and eaga.block_saved_size(bad) == 0
        assert eaga.block_kernel_launches(bad, True) == -1
    assert eaga.block_kernel_launches(d, False) > eaga.kernel_launches(d, False)


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
    g = L.eaga_backward
    bigb = eaga.workspace_size(d, True)
    assert g(ctypes.byref(d), ok, ok, ok, ok, ctypes.byref(w), ok, ok, ok, ok, ok, ok, None, ok, bigb, None) == 1
    # a workspace one byte short (distinct, non-overlapping fake buffers: the
    # size check comes after the overlap check; both return before any launch)
    fw = forward_layout(d, far=True)
    assert f(ctypes.byref(d), *fw.args(ws_bytes=big - 1)) == 4
    bw = backward_layout(d, far=True)
    assert g(ctypes.byref(d), *bw.args(ws_bytes=bigb - 1)) == 4


def test_strerror(L):
    for code in range(7):
        assert eaga.strerror(code)
    assert eaga.strerror(99) == "unknown status"


def test_wait_probe_arguments(L):
    # argument checks happen on the host, before any launch
    assert L.eaga_debug_wait_probe(None, 0, None) == 1             # EAGA_ERR_INVALID_ARG
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
    assert (eaga.kernel_launches(d, False), eaga.kernel_launches(d, True)) == ((5, 12) if fast else (4, 10))


def test_dispatch_rejects_unsupported(L):
    assert eaga.kernel_launches(eaga.dims(2, 1025, 256, 64, 64, 8, 32, "bf16"), False) == -1
    assert eaga.kernel_launches(eaga.dims(0, 64, 256, 64, 64, 8, 32, "bf16"), False) == -1

# ------------------------------------------------------------ buffer layouts

WSHAPES = lambda d: {"Wq": (d.dx, d.H * d.dh), "bq": (d.H * d.dh,), "Wk": (d.dx, d.H * d.dh),
                     "bk": (d.H * d.dh,), "Wv": (d.dx, d.H * d.dh), "bv": (d.H * d.dh,),
                     "Wfe": (d.de, 2 * d.H), "Wfy": (d.dy, 2 * d.H), "bf": (2 * d.H,), "We": (d.H, d.de),
                     "Wo": (d.H * d.dh, d.dx), "bo": (d.dx,)}


def tensor_bytes(d):
    """Bytes of each buffer as a caller allocates it (the shapes of the C ABI)."""
    s = 2 if d.dtype == eaga.EAGA_BF16 else 4
    out = {"X": d.B * d.n * d.dx * s, "E": d.B * d.n * d.n * d.de * s, "y": d.B * d.dy * s, "M": d.B * d.n}
    for k, sh in WSHAPES(d).items():
        out["W" + k] = int(np.prod(sh)) * s
        out["G" + k] = int(np.prod(sh)) * 4
    return out


class Layout:
    """Named fake device pointers: either tightly packed (each buffer starts at
    the next 16-byte boundary after the previous one, so that any range the
    library over-estimates runs into its neighbour) or spread 1 GiB apart.
    Nothing is ever dereferenced on the host."""

    def __init__(self, sizes: dict, far=False):
        self.ptr, off = {}, 0x100000000
        for k, n in sizes.items():
            self.ptr[k] = off
            off = off + (1 << 30) if far else (off + n + 15) // 16 * 16
        self.sizes = sizes

    def p(self, k):
        return ctypes.c_void_p(self.ptr[k])

    def weights(self, prefix):
        return eaga.Weights(*(self.ptr[prefix + k] for k in eaga.WEIGHT_NAMES))


class FwdLayout(Layout):
    def args(self, ws_bytes=None, **over):
        q = lambda k: ctypes.c_void_p(over[k]) if k in over else self.p(k)
        self._w = self.weights("W")
        return (q("X"), q("E"), q("y"), q("M"), ctypes.byref(self._w), q("Xout"), q("Eout"), q("saved"),
                q("ws"), self.sizes["ws"] if ws_bytes is None else ws_bytes, None)


class BwdLayout(Layout):
    def args(self, ws_bytes=None, **over):
        q = lambda k: ctypes.c_void_p(over[k]) if k in over else self.p(k)
        self._w = self.weights("W")
        gp = {k: over.get("G" + k, self.ptr["G" + k]) for k in eaga.WEIGHT_NAMES}
        self._g = eaga.Weights(*(gp[k] for k in eaga.WEIGHT_NAMES))
        return (q("X"), q("E"), q("y"), q("M"), ctypes.byref(self._w), q("saved"), q("dXout"), q("dEout"),
                q("dX"), q("dE"), q("dy"), ctypes.byref(self._g), q("ws"),
                self.sizes["ws"] if ws_bytes is None else ws_bytes, None)


def forward_layout(d, far=False):
    t = tensor_bytes(d)
    sizes = {"X": t["X"], "E": t["E"], "y": t["y"], "M": t["M"]}
    sizes.update({"W" + k: t["W" + k] for k in eaga.WEIGHT_NAMES})
    sizes.update({"Xout": t["X"], "Eout": t["E"], "saved": eaga.saved_size(d), "ws": eaga.workspace_size(d, False)})
    return FwdLayout(sizes, far)


def backward_layout(d, far=False):
    t = tensor_bytes(d)
    sizes = {"X": t["X"], "E": t["E"], "y": t["y"], "M": t["M"]}
    sizes.update({"W" + k: t["W" + k] for k in eaga.WEIGHT_NAMES})
    sizes.update({"saved": eaga.saved_size(d), "dXout": t["X"], "dEout": t["E"], "dX": t["X"], "dE": t["E"],
                  "dy": t["y"]})
    sizes.update({"G" + k: t["G" + k] for k in eaga.WEIGHT_NAMES})
    sizes["ws"] = eaga.workspace_size(d, True)
    return BwdLayout(sizes, far)


ALIAS_DIMS = [eaga.dims(2, 64, 256, 64, 64, 8, 32, "bf16"),      # the tcgen05 path
              eaga.dims(3, 37, 24, 24, 16, 3, 16, "fp32")]       # the CUDA-core path
no_cuda = pytest.mark.skipif(torch.cuda.is_available(),
                             reason="a clean call goes on to its first CUDA call, with fake pointers")


@no_cuda
@pytest.mark.parametrize("d", ALIAS_DIMS, ids=["bf16-fast", "fp32-generic"])
def test_overlap_check_forward(L, d):
    f = lambda **kw: L.eaga_forward(ctypes.byref(d), *lay.args(**kw))
    lay = forward_layout(d)
    # tightly packed, nothing shared: the check passes, and the first CUDA
    # call fails on this host without a GPU (EAGA_ERR_CUDA)
    assert f() == 5
    assert f(Eout=lay.ptr["E"]) == 1                                    # E' in place over E
    assert f(Xout=lay.ptr["X"] + lay.sizes["X"] - 16) == 1              # last 16 bytes of X
    assert f(saved=lay.ptr["ws"]) == 1                                  # two outputs
    assert f(ws=lay.ptr["WWo"]) == 1                                    # workspace over a weight
    assert f(E=lay.ptr["X"], y=lay.ptr["X"]) == 5                       # inputs may share memory


@no_cuda
@pytest.mark.parametrize("d", ALIAS_DIMS, ids=["bf16-fast", "fp32-generic"])
def test_overlap_check_backward(L, d):
    g = lambda **kw: L.eaga_backward(ctypes.byref(d), *lay.args(**kw))
    lay = backward_layout(d)
    assert g() == 5
    assert g(dE=lay.ptr["dEout"]) == 1                                  # dE in place over dE'
    assert g(dX=lay.ptr["saved"] + 16) == 1                             # inside the saved state
    assert g(Gbo=lay.ptr["dy"]) == 1                                    # two outputs
    assert g(ws=lay.ptr["E"] + lay.sizes["E"] - 16) == 1                # workspace over E's tail


@no_cuda
def test_overlap_check_attention_map_and_noalloc(L):
    d = ALIAS_DIMS[0]
    t = tensor_bytes(d)
    sizes = {"E": t["E"], "M": t["M"], "y": t["y"], "saved": eaga.saved_size(d)}
    sizes.update({"W" + k: t["W" + k] for k in eaga.WEIGHT_NAMES})
    sizes["A"] = (d.B * d.H * d.n * d.n + 2 * d.B * d.H) * 4
    lay = Layout(sizes)
    w = lay.weights("W")
    m = lambda A: L.eaga_debug_attention_map(ctypes.byref(d), lay.p("E"), lay.p("M"), ctypes.byref(w), lay.p("y"),
                                             lay.p("saved"), ctypes.c_void_p(A), None)
    assert m(lay.ptr["A"]) == 5
    assert m(lay.ptr["saved"]) == 1
    fw = forward_layout(d)
    n = lambda **kw: L.eaga_forward_noalloc(ctypes.byref(d), *(fw.args(**kw)[:8]), None)
    assert n(Eout=fw.ptr["E"]) == 1
    assert n(saved=fw.ptr["Xout"]) == 1


def _before(sizes: dict, k: str, o: str) -> dict:
    """The same buffers with k placed directly before o, at the end."""
    out = {key: v for key, v in sizes.items() if key not in (k, o)}
    out[k] = sizes[k]
    out[o] = sizes[o]
    return out


@no_cuda
@pytest.mark.parametrize("d", ALIAS_DIMS, ids=["bf16-fast", "fp32-generic"])
def test_overlap_check_extents_never_exceed_the_buffers(L, d):
    # every buffer, followed directly by an output: a range the library
    # over-estimates by a 16-byte step would reach that output and be refused
    fw = forward_layout(d)
    for k in fw.sizes:
        o = "ws" if k != "ws" else "Xout"
        lay = FwdLayout(_before(fw.sizes, k, o))
        assert L.eaga_forward(ctypes.byref(d), *lay.args()) == 5, k
    bw = backward_layout(d)
    for k in bw.sizes:
        o = "ws" if k != "ws" else "dX"
        lay = BwdLayout(_before(bw.sizes, k, o))
        assert L.eaga_backward(ctypes.byref(d), *lay.args()) == 5, k


def test_unknown_variant_is_refused(L):
    # host-side check, before anything is launched
    d = good_dims()
    fake = ctypes.c_void_p(0x100000)
    w = eaga.Weights(*([0x100000] * 12))
    for v in (-1, 3, 7):
        rc = L.eaga_forward_variant(ctypes.byref(d), v, fake, fake, fake, fake, ctypes.byref(w), fake, fake, fake,
                                    fake, 1 << 40, None)
        assert rc == 1
        rc = L.eaga_backward_variant(ctypes.byref(d), v, fake, fake, fake, fake, ctypes.byref(w), fake, fake, fake,
                                     fake, fake, fake, ctypes.byref(w), fake, 1 << 40, None)
        assert rc == 1


@no_cuda
@pytest.mark.parametrize("dims_of", [lambda B: eaga.dims(B, 16, 64, 64, 16, 8, 32, "bf16"),
                                     lambda B: eaga.dims(B, 8, 24, 24, 16, 2, 16, "fp32")],
                         ids=["bf16-fast-892", "fp32-generic-H2-4080"])
def test_noalloc_graph_limit_boundaries(L, dims_of):
    """The no-allocation forward keeps its scratch in a fixed 64 KiB array:
    256 + roundup256(8*H*B) bytes, plus 8 KiB of operand images on the
    specialised path, must fit, so the largest batch is B = 892 there and
    B = 4080 at H = 2 on the CUDA-core path.  One graph more is refused as
    unsupported before any device work; the largest batch passes the size
    check (and goes on to the device, which this CPU-only test does not have)."""
    limit = 892 if dims_of(1).dtype == eaga.EAGA_BF16 else 4080
    for B, refused in ((limit, False), (limit + 1, True)):
        d = dims_of(B)
        fw = forward_layout(d, far=True)
        rc = L.eaga_forward_noalloc(ctypes.byref(d), *(fw.args()[:8]), None)
        assert (rc == 2) == refused, (B, rc)   # 2: EAGA_ERR_UNSUPPORTED
