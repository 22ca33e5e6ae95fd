"""Thin ctypes binding of libeaga.so (include/eaga.h).

Argument marshalling only: every function takes torch tensors that already
live on the GPU (or plain ints), passes their data pointers and the current
CUDA stream to the C entry point of the same name, and raises on a non-OK
status.  All arithmetic runs in the library's CUDA kernels; there is no
fallback of any kind.  The library must have been built in-tree
(edge_aware_graph_b200/build.py); loading fails loudly otherwise.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libeaga.so")

WEIGHT_NAMES = ("Wq", "bq", "Wk", "bk", "Wv", "bv", "Wfe", "Wfy", "bf", "We", "Wo", "bo")
EAGA_FP32, EAGA_BF16 = 0, 1
STATUS = {0: "EAGA_OK", 1: "EAGA_ERR_INVALID_ARG", 2: "EAGA_ERR_UNSUPPORTED", 3: "EAGA_ERR_MISALIGNED",
          4: "EAGA_ERR_WORKSPACE", 5: "EAGA_ERR_CUDA", 6: "EAGA_ERR_TIMEOUT"}
EXPORTED = ("eaga_workspace_size", "eaga_saved_size", "eaga_forward", "eaga_backward",
            "eaga_debug_attention_map", "eaga_get_device_status", "eaga_strerror",
            "eaga_set_profile_events", "eaga_kernel_launches", "eaga_forward_noalloc", "eaga_debug_wait_probe",
            "eaga_forward_variant", "eaga_backward_variant", "eaga_forward_rows", "eaga_backward_rows",
            "eaga_block_saved_size", "eaga_block_workspace_size", "eaga_block_kernel_launches",
            "eaga_block_forward", "eaga_block_backward")
# parameters of the graph-transformer block (eaga_block_weights field order)
BLOCK_SUB_PARAMS = ("ln1_g", "ln1_s", "W1", "b1", "W2", "b2", "ln2_g", "ln2_s")
BLOCK_WEIGHT_NAMES = tuple(f"{s}_{k}" for s in ("x", "e", "y") for k in BLOCK_SUB_PARAMS) + ("Wyx", "Wye", "by")
# layer variants (eaga_variant): the layer, Light Edge, the unnormalised edge update
VARIANTS = {"layer": 0, "light_edge": 1, "unnormalised": 2}


class Dims(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int) for k in ("B", "n", "dx", "de", "dy", "H", "dh", "dtype")]


class Weights(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in WEIGHT_NAMES]


class BlockWeights(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in BLOCK_WEIGHT_NAMES]


class EagaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


_lib = None


def lib():
    """Load libeaga.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libeaga.so not built ({LIB_PATH}); run edge_aware_graph_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        L.eaga_workspace_size.argtypes = [ctypes.POINTER(Dims), i32]
        L.eaga_workspace_size.restype = sz
        L.eaga_saved_size.argtypes = [ctypes.POINTER(Dims)]
        L.eaga_saved_size.restype = sz
        L.eaga_forward.argtypes = [ctypes.POINTER(Dims), vp, vp, vp, vp, ctypes.POINTER(Weights),
                                   vp, vp, vp, vp, sz, vp]
        L.eaga_forward.restype = i32
        L.eaga_backward.argtypes = [ctypes.POINTER(Dims), vp, vp, vp, vp, ctypes.POINTER(Weights), vp,
                                    vp, vp, vp, vp, vp, ctypes.POINTER(Weights), vp, sz, vp]
        L.eaga_backward.restype = i32
        L.eaga_forward_variant.argtypes = [ctypes.POINTER(Dims), i32, vp, vp, vp, vp, ctypes.POINTER(Weights),
                                           vp, vp, vp, vp, sz, vp]
        L.eaga_forward_variant.restype = i32
        L.eaga_backward_variant.argtypes = [ctypes.POINTER(Dims), i32, vp, vp, vp, vp, ctypes.POINTER(Weights), vp,
                                            vp, vp, vp, vp, vp, ctypes.POINTER(Weights), vp, sz, vp]
        L.eaga_backward_variant.restype = i32
        L.eaga_forward_rows.argtypes = [ctypes.POINTER(Dims), i32, i32, i32, vp, vp, vp, vp, ctypes.POINTER(Weights),
                                        vp, vp, vp, vp, sz, vp]
        L.eaga_forward_rows.restype = i32
        L.eaga_backward_rows.argtypes = [ctypes.POINTER(Dims), i32, i32, i32, vp, vp, vp, vp, ctypes.POINTER(Weights),
                                         vp, vp, vp, vp, vp, vp, ctypes.POINTER(Weights), vp, sz, vp]
        L.eaga_backward_rows.restype = i32
        L.eaga_forward_noalloc.argtypes = [ctypes.POINTER(Dims), vp, vp, vp, vp, ctypes.POINTER(Weights),
                                           vp, vp, vp, vp]
        L.eaga_forward_noalloc.restype = i32
        L.eaga_debug_attention_map.argtypes = [ctypes.POINTER(Dims), vp, vp, ctypes.POINTER(Weights), vp, vp,
                                               vp, vp]
        L.eaga_debug_attention_map.restype = i32
        L.eaga_get_device_status.argtypes = [vp, vp]
        L.eaga_get_device_status.restype = i32
        L.eaga_debug_wait_probe.argtypes = [vp, ctypes.c_uint, vp]
        L.eaga_debug_wait_probe.restype = i32
        L.eaga_set_profile_events.argtypes = [i32, vp, vp]
        L.eaga_set_profile_events.restype = i32
        L.eaga_kernel_launches.argtypes = [ctypes.POINTER(Dims), i32]
        L.eaga_kernel_launches.restype = i32
        L.eaga_block_saved_size.argtypes = [ctypes.POINTER(Dims)]
        L.eaga_block_saved_size.restype = sz
        L.eaga_block_workspace_size.argtypes = [ctypes.POINTER(Dims), i32]
        L.eaga_block_workspace_size.restype = sz
        L.eaga_block_kernel_launches.argtypes = [ctypes.POINTER(Dims), i32]
        L.eaga_block_kernel_launches.restype = i32
        W_, BW_ = ctypes.POINTER(Weights), ctypes.POINTER(BlockWeights)
        L.eaga_block_forward.argtypes = [ctypes.POINTER(Dims), vp, vp, vp, vp, W_, BW_, vp, vp, vp, vp, vp, vp,
                                         vp, sz, vp]
        L.eaga_block_forward.restype = i32
        L.eaga_block_backward.argtypes = [ctypes.POINTER(Dims), vp, vp, vp, vp, W_, BW_, vp, vp, vp, vp, vp, vp,
                                          vp, vp, vp, vp, W_, BW_, vp, sz, vp]
        L.eaga_block_backward.restype = i32
        L.eaga_strerror.argtypes = [i32]
        L.eaga_strerror.restype = ctypes.c_char_p
        _lib = L
    return _lib


def dims(B, n, dx, de, dy, H, dh, dtype) -> Dims:
    if isinstance(dtype, str):
        dtype = EAGA_BF16 if dtype == "bf16" else EAGA_FP32
    return Dims(B, n, dx, de, dy, H, dh, dtype)


def _p(t, name="tensor", dtype=None):
    """Data pointer of a tensor handed to the library: a contiguous CUDA tensor
    on the current device (and of `dtype`, when given); None passes NULL.  A
    host tensor or one on another GPU would reach the kernels as a bad device
    pointer, so it is refused here."""
    if t is None:
        return None
    import torch
    if not t.is_cuda:
        raise ValueError(f"{name}: a CUDA tensor is required (got {t.device})")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name}: on {t.device}, but the current device is cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _storage(d: Dims):
    import torch
    return torch.bfloat16 if d.dtype == EAGA_BF16 else torch.float32


def _u8():
    import torch
    return torch.uint8


def _f32():
    import torch
    return torch.float32


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _weights(W: dict, dtype=None, what="W") -> Weights:
    return Weights(*(_p(W[k], f"{what}[{k}]", dtype).value for k in WEIGHT_NAMES))


def _check(rc: int, where: str):
    if rc != 0:
        raise EagaError(rc, where)


def workspace_size(d: Dims, for_backward: bool) -> int:
    return int(lib().eaga_workspace_size(ctypes.byref(d), int(bool(for_backward))))


def saved_size(d: Dims) -> int:
    return int(lib().eaga_saved_size(ctypes.byref(d)))


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def forward(d: Dims, X, E, y, M, W: dict, Xout, Eout, saved, workspace, stream=None, variant: str = "layer"):
    """eaga_forward (variant "layer"), else eaga_forward_variant."""
    sd = _storage(d)
    args = (_p(X, "X", sd), _p(E, "E", sd), _p(y, "y", sd), _p(M, "M", _u8()),
            ctypes.byref(_weights(W, sd)), _p(Xout, "Xout", sd), _p(Eout, "Eout", sd),
            _p(saved, "saved"), _p(workspace, "workspace"), _nbytes(workspace), _stream(stream))
    if variant == "layer":
        _check(lib().eaga_forward(ctypes.byref(d), *args), "eaga_forward")
    else:
        _check(lib().eaga_forward_variant(ctypes.byref(d), VARIANTS[variant], *args), "eaga_forward_variant")


def forward_noalloc(d: Dims, X, E, y, M, W: dict, Xout, Eout, saved, stream=None):
    """eaga_forward without a workspace argument (the library's own fixed scratch is used)."""
    sd = _storage(d)
    rc = lib().eaga_forward_noalloc(ctypes.byref(d), _p(X, "X", sd), _p(E, "E", sd), _p(y, "y", sd),
                                    _p(M, "M", _u8()), ctypes.byref(_weights(W, sd)), _p(Xout, "Xout", sd),
                                    _p(Eout, "Eout", sd), _p(saved, "saved"), _stream(stream))
    _check(rc, "eaga_forward_noalloc")


def backward(d: Dims, X, E, y, M, W: dict, saved, dXout, dEout, dX, dE, dy, dW: dict, workspace, stream=None,
             variant: str = "layer"):
    """eaga_backward (variant "layer"), else eaga_backward_variant."""
    sd = _storage(d)
    args = (_p(X, "X", sd), _p(E, "E", sd), _p(y, "y", sd), _p(M, "M", _u8()),
            ctypes.byref(_weights(W, sd)), _p(saved, "saved"), _p(dXout, "dXout", sd),
            _p(dEout, "dEout", sd), _p(dX, "dX", sd), _p(dE, "dE", sd), _p(dy, "dy", sd),
            ctypes.byref(_weights(dW, _f32(), "dW")), _p(workspace, "workspace"),
            _nbytes(workspace), _stream(stream))
    if variant == "layer":
        _check(lib().eaga_backward(ctypes.byref(d), *args), "eaga_backward")
    else:
        _check(lib().eaga_backward_variant(ctypes.byref(d), VARIANTS[variant], *args), "eaga_backward_variant")


def forward_rows(d: Dims, row0: int, rows: int, X, E_rows, y, M, W: dict, Xout, Eout_rows, saved, workspace,
                 stream=None, variant: str = "layer"):
    """eaga_forward_rows: the rows row0 .. row0+rows-1 of every graph, E_rows and
    Eout_rows [B, rows, n, de] slabs."""
    sd = _storage(d)
    rc = lib().eaga_forward_rows(ctypes.byref(d), VARIANTS[variant], int(row0), int(rows), _p(X, "X", sd),
                                 _p(E_rows, "E_rows", sd), _p(y, "y", sd), _p(M, "M", _u8()),
                                 ctypes.byref(_weights(W, sd)), _p(Xout, "Xout", sd), _p(Eout_rows, "Eout_rows", sd),
                                 _p(saved, "saved"), _p(workspace, "workspace"), _nbytes(workspace), _stream(stream))
    _check(rc, "eaga_forward_rows")


def backward_rows(d: Dims, row0: int, rows: int, X, E_rows, y, M, W: dict, saved, dXout, dEout_rows, dX, dE_rows,
                  dy, dW: dict, workspace, stream=None, variant: str = "layer"):
    """eaga_backward_rows: this slab's part of dX, dy and the weight gradients
    (dXout zero outside the slab's rows), and the slab's dE."""
    sd = _storage(d)
    rc = lib().eaga_backward_rows(ctypes.byref(d), VARIANTS[variant], int(row0), int(rows), _p(X, "X", sd),
                                  _p(E_rows, "E_rows", sd), _p(y, "y", sd), _p(M, "M", _u8()),
                                  ctypes.byref(_weights(W, sd)), _p(saved, "saved"), _p(dXout, "dXout", sd),
                                  _p(dEout_rows, "dEout_rows", sd), _p(dX, "dX", sd), _p(dE_rows, "dE_rows", sd),
                                  _p(dy, "dy", sd), ctypes.byref(_weights(dW, _f32(), "dW")),
                                  _p(workspace, "workspace"), _nbytes(workspace), _stream(stream))
    _check(rc, "eaga_backward_rows")


def debug_attention_map(d: Dims, E, M, W: dict, y, saved, A, stream=None):
    sd = _storage(d)
    rc = lib().eaga_debug_attention_map(ctypes.byref(d), _p(E, "E", sd), _p(M, "M", _u8()),
                                        ctypes.byref(_weights(W, sd)), _p(y, "y", sd), _p(saved, "saved"),
                                        _p(A, "A", _f32()), _stream(stream))
    _check(rc, "eaga_debug_attention_map")


def get_device_status(workspace, stream=None) -> int:
    return int(lib().eaga_get_device_status(_p(workspace, "workspace"), _stream(stream)))


def debug_wait_probe(workspace, limit: int, stream=None):
    """Run the bounded-wait failure path once (test aid): a wait that never
    completes gives up after `limit` polls and records a timeout."""
    _check(lib().eaga_debug_wait_probe(_p(workspace, "workspace"), int(limit), _stream(stream)),
           "eaga_debug_wait_probe")


def set_profile_events(point: int, before=None, after=None):
    """point 0: forward pair kernels, 1: backward pair kernels, 2: the backward's
    row pair kernel alone, 3 / 4: the edge kernel of the block's forward /
    backward; torch.cuda.Event or None."""
    b = ctypes.c_void_p(before.cuda_event) if before is not None else None
    a = ctypes.c_void_p(after.cuda_event) if after is not None else None
    _check(lib().eaga_set_profile_events(int(point), b, a), "eaga_set_profile_events")


def kernel_launches(d: Dims, for_backward: bool) -> int:
    return int(lib().eaga_kernel_launches(ctypes.byref(d), int(bool(for_backward))))


def strerror(code: int) -> str:
    return lib().eaga_strerror(int(code)).decode()


# ---------------------------------------------------------------- the block around the layer

def _block_weights(Wb: dict, dtype=None, what="Wb") -> BlockWeights:
    return BlockWeights(*(_p(Wb[k], f"{what}[{k}]", dtype).value for k in BLOCK_WEIGHT_NAMES))


def block_saved_size(d: Dims) -> int:
    return int(lib().eaga_block_saved_size(ctypes.byref(d)))


def block_workspace_size(d: Dims, for_backward: bool) -> int:
    return int(lib().eaga_block_workspace_size(ctypes.byref(d), int(bool(for_backward))))


def block_kernel_launches(d: Dims, for_backward: bool) -> int:
    return int(lib().eaga_block_kernel_launches(ctypes.byref(d), int(bool(for_backward))))


def block_forward(d: Dims, X, E, y, M, W: dict, Wb: dict, Xmid, Emid, Xout, Eout, yout, saved, workspace,
                  stream=None):
    """eaga_block_forward."""
    sd = _storage(d)
    rc = lib().eaga_block_forward(
        ctypes.byref(d), _p(X, "X", sd), _p(E, "E", sd), _p(y, "y", sd), _p(M, "M", _u8()),
        ctypes.byref(_weights(W, sd)), ctypes.byref(_block_weights(Wb, sd)), _p(Xmid, "Xmid", sd),
        _p(Emid, "Emid", sd), _p(Xout, "Xout", sd), _p(Eout, "Eout", sd), _p(yout, "yout", sd),
        _p(saved, "saved"), _p(workspace, "workspace"), _nbytes(workspace), _stream(stream))
    _check(rc, "eaga_block_forward")


def block_backward(d: Dims, X, E, y, M, W: dict, Wb: dict, Xmid, Emid, saved, dXout, dEout, dyout, dEmid,
                   dX, dE, dy, dW: dict, dWb: dict, workspace, stream=None):
    """eaga_block_backward."""
    sd = _storage(d)
    rc = lib().eaga_block_backward(
        ctypes.byref(d), _p(X, "X", sd), _p(E, "E", sd), _p(y, "y", sd), _p(M, "M", _u8()),
        ctypes.byref(_weights(W, sd)), ctypes.byref(_block_weights(Wb, sd)), _p(Xmid, "Xmid", sd),
        _p(Emid, "Emid", sd), _p(saved, "saved"), _p(dXout, "dXout", sd), _p(dEout, "dEout", sd),
        _p(dyout, "dyout", sd), _p(dEmid, "dEmid", sd), _p(dX, "dX", sd), _p(dE, "dE", sd), _p(dy, "dy", sd),
        ctypes.byref(_weights(dW, _f32(), "dW")), ctypes.byref(_block_weights(dWb, _f32(), "dWb")),
        _p(workspace, "workspace"), _nbytes(workspace), _stream(stream))
    _check(rc, "eaga_block_backward")
