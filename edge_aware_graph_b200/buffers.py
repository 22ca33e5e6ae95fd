"""Device buffers for one layer call, allocated with torch (memory only).

`LayerBuffers` owns the inputs, weights, outputs, saved state and workspaces
of one problem size on one device, so that repeated calls reuse memory.
Inputs may be copied in from host arrays (`load_inputs`) or from pinned host
tensors (`copy_in_async`).
"""
from __future__ import annotations

import numpy as np
import torch

from . import eaga
from .eaga import WEIGHT_NAMES


def torch_dtype(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def host_to_storage_tensor(a: np.ndarray, dtype: str) -> torch.Tensor:
    """float32 numpy array holding storage-dtype values -> CPU tensor of that dtype (exact)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch_dtype(dtype))


class LayerBuffers:
    def __init__(self, B, n, dx, de, dy, H, dh, dtype="bf16", device="cuda", backward=True):
        self.shape = dict(B=B, n=n, dx=dx, de=de, dy=dy, H=H, dh=dh)
        self.dtype = dtype
        self.device = torch.device(device)
        self.dims = eaga.dims(B, n, dx, de, dy, H, dh, dtype)
        td = torch_dtype(dtype)
        dev = self.device
        hd = H * dh
        e = lambda *s: torch.empty(*s, dtype=td, device=dev)
        self.X, self.E, self.y = e(B, n, dx), e(B, n, n, de), e(B, dy)
        self.M = torch.empty(B, n, dtype=torch.uint8, device=dev)
        shapes = {"Wq": (dx, hd), "bq": (hd,), "Wk": (dx, hd), "bk": (hd,), "Wv": (dx, hd), "bv": (hd,),
                  "Wfe": (de, 2 * H), "Wfy": (dy, 2 * H), "bf": (2 * H,), "We": (H, de), "Wo": (hd, dx),
                  "bo": (dx,)}
        self.W = {k: e(*shapes[k]) for k in WEIGHT_NAMES}
        self.Xout, self.Eout = e(B, n, dx), e(B, n, n, de)
        self.saved = torch.empty(eaga.saved_size(self.dims), dtype=torch.uint8, device=dev)
        self.ws_fwd = torch.empty(eaga.workspace_size(self.dims, False), dtype=torch.uint8, device=dev)
        self.has_backward = backward
        if backward:
            self.dXout, self.dEout = e(B, n, dx), e(B, n, n, de)
            self.dX, self.dE, self.dy = e(B, n, dx), e(B, n, n, de), e(B, dy)
            # weight gradients: views into one flat fp32 buffer (one all-reduce in data parallel use)
            offs, off = {}, 0
            for k in WEIGHT_NAMES:
                offs[k] = off
                off += (int(np.prod(shapes[k])) + 63) // 64 * 64
            self.dW_flat = torch.zeros(off, dtype=torch.float32, device=dev)
            self.dW = {k: self.dW_flat[offs[k]:offs[k] + int(np.prod(shapes[k]))].view(shapes[k])
                       for k in WEIGHT_NAMES}
            self.ws_bwd = torch.empty(eaga.workspace_size(self.dims, True), dtype=torch.uint8, device=dev)

    # ------------------------------------------------------------ inputs

    def load_inputs(self, inputs: dict, weights: dict):
        dt = self.dtype
        for k in ("X", "E", "y"):
            getattr(self, k).copy_(host_to_storage_tensor(inputs[k], dt))
        self.M.copy_(torch.from_numpy(np.ascontiguousarray(inputs["M"], dtype=np.uint8)))
        for k in WEIGHT_NAMES:
            self.W[k].copy_(host_to_storage_tensor(weights[k], dt))
        if self.has_backward and "dXout" in inputs:
            self.dXout.copy_(host_to_storage_tensor(inputs["dXout"], dt))
            self.dEout.copy_(host_to_storage_tensor(inputs["dEout"], dt))

    # ------------------------------------------------------------ calls

    def forward(self, stream=None, saved=True, variant="layer"):
        eaga.forward(self.dims, self.X, self.E, self.y, self.M, self.W, self.Xout, self.Eout,
                     self.saved if saved else None, self.ws_fwd, stream, variant=variant)

    def backward(self, stream=None, variant="layer"):
        eaga.backward(self.dims, self.X, self.E, self.y, self.M, self.W, self.saved, self.dXout, self.dEout,
                      self.dX, self.dE, self.dy, self.dW, self.ws_bwd, stream, variant=variant)

    def attention_map(self, stream=None):
        B, n, H = self.shape["B"], self.shape["n"], self.shape["H"]
        A = torch.empty(B * H * n * n + 2 * B * H, dtype=torch.float32, device=self.device)
        eaga.debug_attention_map(self.dims, self.E, self.M, self.W, self.y, self.saved, A, stream)
        return A[: B * H * n * n].view(B, H, n, n)

    def saved_parts(self):
        """Views of the saved state: LSE [B,H,n] fp32 and Q, K, V, O [B,n,H*dh]."""
        B, n, H, dh = (self.shape[k] for k in ("B", "n", "H", "dh"))
        hd = H * dh
        es = 2 if self.dtype == "bf16" else 4
        al = lambda x: (x + 255) // 256 * 256
        off = 0
        out = {}
        sz = B * H * n * 4
        out["LSE"] = self.saved[off:off + sz].view(torch.float32).view(B, H, n)
        off = al(off + sz)
        for k in ("Q", "K", "V", "O"):
            sz = B * n * hd * es
            out[k] = self.saved[off:off + sz].view(torch_dtype(self.dtype)).view(B, n, hd)
            off = al(off + sz)
        return out


class BlockBuffers(LayerBuffers):
    """LayerBuffers plus the graph-transformer block around the layer: the
    block's parameters, the layer's outputs X', E' (Xmid, Emid), the block's
    outputs, saved state, workspaces and gradients."""

    def __init__(self, B, n, dx, de, dy, H, dh, dtype="bf16", device="cuda", backward=True):
        super().__init__(B, n, dx, de, dy, H, dh, dtype, device, backward)
        td = torch_dtype(dtype)
        dev = self.device
        e = lambda *s: torch.empty(*s, dtype=td, device=dev)
        self.bshapes = {}
        for s, w in (("x", dx), ("e", de), ("y", dy)):
            self.bshapes.update({f"{s}_ln1_g": (w,), f"{s}_ln1_s": (w,), f"{s}_W1": (w, 2 * w), f"{s}_b1": (2 * w,),
                                 f"{s}_W2": (2 * w, w), f"{s}_b2": (w,), f"{s}_ln2_g": (w,), f"{s}_ln2_s": (w,)})
        self.bshapes.update({"Wyx": (dx, dy), "Wye": (de, dy), "by": (dy,)})
        self.Wb = {k: e(*self.bshapes[k]) for k in eaga.BLOCK_WEIGHT_NAMES}
        self.Xmid, self.Emid = e(B, n, dx), e(B, n, n, de)
        self.yout = e(B, dy)
        self.bsaved = torch.empty(eaga.block_saved_size(self.dims), dtype=torch.uint8, device=dev)
        self.bws_fwd = torch.empty(eaga.block_workspace_size(self.dims, False), dtype=torch.uint8, device=dev)
        if backward:
            self.dyout = e(B, dy)
            self.dEmid = e(B, n, n, de)
            offs, off = {}, 0
            for k in eaga.BLOCK_WEIGHT_NAMES:
                offs[k] = off
                off += (int(np.prod(self.bshapes[k])) + 63) // 64 * 64
            self.dWb_flat = torch.zeros(off, dtype=torch.float32, device=dev)
            self.dWb = {k: self.dWb_flat[offs[k]:offs[k] + int(np.prod(self.bshapes[k]))].view(self.bshapes[k])
                        for k in eaga.BLOCK_WEIGHT_NAMES}
            self.bws_bwd = torch.empty(eaga.block_workspace_size(self.dims, True), dtype=torch.uint8, device=dev)

    def load_block(self, block_weights: dict, dyout=None):
        for k in eaga.BLOCK_WEIGHT_NAMES:
            self.Wb[k].copy_(host_to_storage_tensor(block_weights[k], self.dtype))
        if dyout is not None and self.has_backward:
            self.dyout.copy_(host_to_storage_tensor(dyout, self.dtype))

    def block_forward(self, stream=None):
        eaga.block_forward(self.dims, self.X, self.E, self.y, self.M, self.W, self.Wb, self.Xmid, self.Emid,
                           self.Xout, self.Eout, self.yout, self.bsaved, self.bws_fwd, stream)

    def block_backward(self, stream=None):
        eaga.block_backward(self.dims, self.X, self.E, self.y, self.M, self.W, self.Wb, self.Xmid, self.Emid,
                            self.bsaved, self.dXout, self.dEout, self.dyout, self.dEmid, self.dX, self.dE,
                            self.dy, self.dW, self.dWb, self.bws_bwd, stream)
