"""Test infrastructure, not product code: a plain fp64 numpy restatement of
the graph-transformer block around the edge-aware attention layer.

Only the tests, the smoke check and the benchmark's CPU-baseline leg use this
module; the CUDA library shares no code with it.  The layer itself comes from
the C oracle (oracle.forward / oracle.backward); this file adds what the
pages say surrounds it: the layer sits in DeFoG's graph-transformer backbone,
which updates node, edge and global features jointly (AI-summary page,
method paragraph; paper index page, abstract).  The pages print none of the
block's equations, so the steps below are the plain post-norm reading, in
this order:

  b0  (X', E') = the layer on (X, E, y, M)
  b1  pX_b = sum_i M_bi X'_bi / max(cnt_b, 1)
      pE_b = sum_ij valid_bij E'_bij / max(cnt_b^2, 1)       cnt_b = sum_i M_bi
  b2  y1_b = y_b + pX_b Wyx + pE_b Wye + by
  b3  for Z in (X', E', y1):  Za = LN(Z; g1, s1)
                              Zz = Za + relu(Za W1 + b1) W2 + b2
                              Zo = LN(Zz; g2, s2)
  b4  Xout = M * Xo,  Eout = valid * Eo,  yout = yo

LN: LayerNorm over the last axis, biased variance, eps = 1e-5.  FFN widths
2*dx, 2*de, 2*dy.  Weights are [in, out] (Y = X W).  The backward is the
chain rule of b0..b4 written out step by step.

Storage: with storage="bf16" the block's inputs X', E' are the layer's
outputs rounded to bfloat16 (round to nearest even), as a bf16 layer stores
them; everything after that is fp64.  The pooled means are sensitive to that
rounding: E' of many pairs shares a few values (the edge features of a graph
come from few classes), so their rounding errors do not average out, while
the mean over pairs of unit-size channels can be near zero.

Pins (tests/test_block_oracle.py): the LayerNorm closed form, torch's
float64 LayerNorm/Linear/ReLU modules and autograd for each sub-block,
masked outputs, the pooling's independence of padding, and central finite
differences of the whole block (layer included) on a tiny case.
"""
from __future__ import annotations

import numpy as np

from . import backward as layer_backward
from . import forward as layer_forward

LN_EPS = 1e-5

# parameter names of one block, per sub-block: LayerNorm 1 (gain, shift),
# FFN (W1, b1, W2, b2), LayerNorm 2
SUB_PARAMS = ("ln1_g", "ln1_s", "W1", "b1", "W2", "b2", "ln2_g", "ln2_s")
SUBS = ("x", "e", "y")                     # node, edge, global sub-blocks
BLOCK_WEIGHT_NAMES = tuple(f"{s}_{k}" for s in SUBS for k in SUB_PARAMS) + ("Wyx", "Wye", "by")


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def round_bf16(a):
    """a rounded to the nearest bfloat16 (ties to even), via its float32 bits."""
    bits = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


def _storage(a, storage):
    return round_bf16(a) if storage == "bf16" else _f64(a)


def layer_norm(z, g, s):
    """LN(z; g, s) over the last axis; returns the output, x_hat and 1/sqrt(var + eps)."""
    mu = z.mean(axis=-1, keepdims=True)
    var = ((z - mu) ** 2).mean(axis=-1, keepdims=True)
    r = 1.0 / np.sqrt(var + LN_EPS)
    xh = (z - mu) * r
    return xh * g + s, xh, r


def layer_norm_input_grad(d, xh, r, g):
    """Gradient of LN's input: r (d g - mean(d g) - x_hat mean(d g x_hat))."""
    dg = d * g
    return r * (dg - dg.mean(axis=-1, keepdims=True) - xh * (dg * xh).mean(axis=-1, keepdims=True))


def sub_forward(Z, P):
    """b3 for one sub-block: LN, FFN with residual, LN.  P holds SUB_PARAMS."""
    Za, xh1, r1 = layer_norm(Z, P["ln1_g"], P["ln1_s"])
    hpre = Za @ P["W1"] + P["b1"]
    h = np.maximum(hpre, 0.0)
    Zz = Za + h @ P["W2"] + P["b2"]
    Zo, xh2, r2 = layer_norm(Zz, P["ln2_g"], P["ln2_s"])
    return Zo, dict(Za=Za, xh1=xh1, r1=r1, hpre=hpre, h=h, xh2=xh2, r2=r2)


def sub_backward(dZo, P, c):
    """Chain rule of sub_forward given its cache c; rows are summed over every
    leading axis for the parameter gradients.  Returns dZ and the gradients."""
    flat = lambda a: a.reshape(-1, a.shape[-1])
    dZz = layer_norm_input_grad(dZo, c["xh2"], c["r2"], P["ln2_g"])
    g = {"ln2_g": flat(dZo * c["xh2"]).sum(0), "ln2_s": flat(dZo).sum(0)}
    g["W2"] = flat(c["h"]).T @ flat(dZz)
    g["b2"] = flat(dZz).sum(0)
    dh = (dZz @ P["W2"].T) * (c["hpre"] > 0)
    g["W1"] = flat(c["Za"]).T @ flat(dh)
    g["b1"] = flat(dh).sum(0)
    dZa = dZz + dh @ P["W1"].T
    dZ = layer_norm_input_grad(dZa, c["xh1"], c["r1"], P["ln1_g"])
    g["ln1_g"] = flat(dZa * c["xh1"]).sum(0)
    g["ln1_s"] = flat(dZa).sum(0)
    return dZ, g


def _sub(Wb, s):
    return {k: _f64(Wb[f"{s}_{k}"]) for k in SUB_PARAMS}


def _masks(M):
    Mf = _f64(M)
    cnt = Mf.sum(axis=1)
    valid = Mf[:, :, None] * Mf[:, None, :]
    return Mf, valid, np.maximum(cnt, 1.0), np.maximum(cnt * cnt, 1.0)


def pooled(Xm, Em, M):
    """b1: masked means of the layer's node and edge outputs per graph."""
    Mf, valid, cx, ce = _masks(M)
    pX = (Mf[:, :, None] * Xm).sum(axis=1) / cx[:, None]
    pE = (valid[..., None] * Em).sum(axis=(1, 2)) / ce[:, None]
    return pX, pE


def block_tail_forward(Xm, Em, y, M, Wb):
    """b1-b4 given the layer's outputs X', E'."""
    Xm, Em, y = _f64(Xm), _f64(Em), _f64(y)
    Mf, valid, _, _ = _masks(M)
    pX, pE = pooled(Xm, Em, M)
    y1 = y + pX @ _f64(Wb["Wyx"]) + pE @ _f64(Wb["Wye"]) + _f64(Wb["by"])
    Xo, cx = sub_forward(Xm, _sub(Wb, "x"))
    Eo, ce = sub_forward(Em, _sub(Wb, "e"))
    yo, cy = sub_forward(y1, _sub(Wb, "y"))
    out = {"Xout": Mf[:, :, None] * Xo, "Eout": valid[..., None] * Eo, "yout": yo,
           "Xmid": Xm, "Emid": Em, "y1": y1, "pX": pX, "pE": pE}
    return out, dict(x=cx, e=ce, y=cy)


def block_forward(dims: dict, X, E, y, M, W: dict, Wb: dict, storage: str = "fp64"):
    """b0-b4: the layer (C oracle) then the block.  Returns Xout, Eout, yout
    and the intermediates Xmid (X'), Emid (E'), y1, pX, pE."""
    lay = layer_forward(dims, X, E, y, M, W)
    out, _ = block_tail_forward(_storage(lay["Xout"], storage), _storage(lay["Eout"], storage), y, M, Wb)
    return out


def block_tail_backward(Xm, Em, y, M, Wb, dXout, dEout, dyout):
    """Chain rule of b1-b4: returns dX', dE', dy1 (the residual part of dy)
    and the block's parameter gradients."""
    fwd, cache = block_tail_forward(Xm, Em, y, M, Wb)
    Mf, valid, cx, ce = _masks(M)
    grads = {}
    dy1, gy = sub_backward(_f64(dyout), _sub(Wb, "y"), cache["y"])
    dXm, gx = sub_backward(Mf[:, :, None] * _f64(dXout), _sub(Wb, "x"), cache["x"])
    dEm, ge = sub_backward(valid[..., None] * _f64(dEout), _sub(Wb, "e"), cache["e"])
    for s, g in (("x", gx), ("e", ge), ("y", gy)):
        for k, v in g.items():
            grads[f"{s}_{k}"] = v
    grads["Wyx"] = fwd["pX"].T @ dy1
    grads["Wye"] = fwd["pE"].T @ dy1
    grads["by"] = dy1.sum(axis=0)
    dpX = dy1 @ _f64(Wb["Wyx"]).T / cx[:, None]
    dpE = dy1 @ _f64(Wb["Wye"]).T / ce[:, None]
    dXm = dXm + Mf[:, :, None] * dpX[:, None, :]
    dEm = dEm + valid[..., None] * dpE[:, None, None, :]
    return dXm, dEm, dy1, grads


def block_backward(dims: dict, X, E, y, M, W: dict, Wb: dict, dXout, dEout, dyout, storage: str = "fp64"):
    """Gradients of the whole block (layer included): dX, dE, dy, the layer's
    d<weight> and the block's d<name> for every name of BLOCK_WEIGHT_NAMES."""
    lay = layer_forward(dims, X, E, y, M, W)
    dXm, dEm, dy1, gb = block_tail_backward(_storage(lay["Xout"], storage), _storage(lay["Eout"], storage), y, M,
                                            Wb, dXout, dEout, dyout)
    g = layer_backward(dims, X, E, y, M, W, dXm, dEm)
    out = {"dX": g["dX"], "dE": g["dE"], "dy": g["dy"] + dy1, "dXmid": dXm, "dEmid": dEm, "dy1": dy1}
    for k, v in g.items():
        if k not in ("dX", "dE", "dy"):
            out[k] = v
    for k, v in gb.items():
        out["d" + k] = v
    return out
