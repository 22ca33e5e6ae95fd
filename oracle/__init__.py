"""Test infrastructure: ctypes binding of the fp64 CPU oracle (eaga_oracle.c).

Only tests, the smoke check and the benchmark's CPU-baseline leg import this
package.  It shares no code with the CUDA library: it builds its own shared
object from eaga_oracle.c with gcc and takes plain numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "eaga_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

WEIGHT_NAMES = ("Wq", "bq", "Wk", "bk", "Wv", "bv", "Wfe", "Wfy", "bf", "We", "Wo", "bo")
# layer variants (eaga_oracle.c): the layer, and the two ablations of the
# AI-summary page (Light Edge: no per-edge modulation; unnormalised: the edge
# update from the modulated scores instead of the normalised coefficients)
VARIANTS = {"layer": 0, "light_edge": 1, "unnormalised": 2}


class _Dims(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int) for k in ("B", "n", "dx", "de", "dy", "H", "dh")]


class _Weights(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in WEIGHT_NAMES]


def build(force: bool = False) -> str:
    """Compile eaga_oracle.c into liboracle.so (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        for fn in (_lib.orc_forward, _lib.orc_backward, _lib.orc_forward_variant, _lib.orc_backward_variant):
            fn.restype = ctypes.c_int
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _dims(d: dict) -> _Dims:
    if d["H"] > 32:
        raise ValueError("oracle supports H <= 32")
    return _Dims(*(int(d[k]) for k in ("B", "n", "dx", "de", "dy", "H", "dh")))


def _shapes_of(X, E, y):
    B, n, dx = X.shape
    return B, n, dx, E.shape[-1], y.shape[-1]


def forward(dims: dict, X, E, y, M, W: dict, want_attention: bool = False, variant: str = "layer"):
    """fp64 forward.  dims needs H and dh; B, n, dx, de, dy come from shapes.

    Returns dict with Xout, Eout, O [B,n,H*dh], LSE [B,H,n] and, if asked,
    A [B,H,n,n].  `variant` is one of VARIANTS.
    """
    lib = _load()
    B, n, dx, de, dyd = _shapes_of(X, E, y)
    d = dict(B=B, n=n, dx=dx, de=de, dy=dyd, H=dims["H"], dh=dims["dh"])
    X, E, y = _f64(X), _f64(E), _f64(y)
    M = np.ascontiguousarray(M, dtype=np.uint8)
    Wd = {k: _f64(W[k]) for k in WEIGHT_NAMES}
    wst = _Weights(*(_ptr(Wd[k]) for k in WEIGHT_NAMES))
    hd = d["H"] * d["dh"]
    out = {
        "Xout": np.empty_like(X), "Eout": np.empty_like(E),
        "O": np.empty((B, n, hd)), "LSE": np.empty((B, d["H"], n)),
    }
    if want_attention:
        out["A"] = np.empty((B, d["H"], n, n))
    rc = lib.orc_forward_variant(ctypes.byref(_dims(d)), VARIANTS[variant], _ptr(X), _ptr(E), _ptr(y), _ptr(M),
                                 ctypes.byref(wst), _ptr(out["Xout"]), _ptr(out["Eout"]),
                                 _ptr(out.get("A")), _ptr(out["O"]), _ptr(out["LSE"]))
    if rc != 0:
        raise RuntimeError(f"orc_forward failed: {rc}")
    return out


def backward(dims: dict, X, E, y, M, W: dict, dXout, dEout, variant: str = "layer"):
    """fp64 backward.  Returns dict with dX, dE, dy and d<weight> for each weight."""
    lib = _load()
    B, n, dx, de, dyd = _shapes_of(X, E, y)
    d = dict(B=B, n=n, dx=dx, de=de, dy=dyd, H=dims["H"], dh=dims["dh"])
    X, E, y, dXout, dEout = _f64(X), _f64(E), _f64(y), _f64(dXout), _f64(dEout)
    M = np.ascontiguousarray(M, dtype=np.uint8)
    Wd = {k: _f64(W[k]) for k in WEIGHT_NAMES}
    wst = _Weights(*(_ptr(Wd[k]) for k in WEIGHT_NAMES))
    grads = {k: np.zeros_like(Wd[k]) for k in WEIGHT_NAMES}
    gst = _Weights(*(_ptr(grads[k]) for k in WEIGHT_NAMES))
    out = {"dX": np.empty_like(X), "dE": np.empty_like(E), "dy": np.empty_like(y)}
    rc = lib.orc_backward_variant(ctypes.byref(_dims(d)), VARIANTS[variant], _ptr(X), _ptr(E), _ptr(y), _ptr(M),
                                  ctypes.byref(wst), _ptr(dXout), _ptr(dEout),
                          _ptr(out["dX"]), _ptr(out["dE"]), _ptr(out["dy"]), ctypes.byref(gst))
    if rc != 0:
        raise RuntimeError(f"orc_backward failed: {rc}")
    for k in WEIGHT_NAMES:
        out["d" + k] = grads[k]
    return out


_threads = None


def set_threads(n: int | None) -> None:
    """Run the oracle's OpenMP loops on n threads (None: back to all usable
    cores).  Only the thread count changes, never the arithmetic."""
    global _threads
    _load()
    gomp = ctypes.CDLL("libgomp.so.1")
    gomp.omp_set_num_threads(int(n) if n else len(os.sched_getaffinity(0)))
    _threads = int(n) if n else None


def threads_used() -> int:
    """OpenMP threads the oracle runs with (set_threads, OMP_NUM_THREADS, else all usable cores)."""
    if _threads:
        return _threads
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        return int(env)
    return len(os.sched_getaffinity(0))
