"""Seeded synthetic inputs for the edge-aware attention layer.

This module holds random draws only: the five workload presets (their dims,
seeds and graph families), the graph-structure samplers (Bernoulli "planar"
adjacency, uniform labelled trees, stochastic block models), the edge-feature
recipe built on them, and rounding of every drawn value to the storage dtype.
It contains none of the layer's arithmetic, so both the CUDA path and the
CPU oracle tests can take their inputs from here.

The paper ("Efficient Edge-aware Attention Network for Graph Generation",
section 4) trains on the Planar, Tree and SBM graph datasets; those are not
available here, so each preset draws graphs with the same structure
(size, density, block pattern) and builds edge features from the sampled
adjacency: E_ij = c[A_ij] + eps_ij, two class embeddings plus small noise.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# ---------------------------------------------------------------- presets


@dataclasses.dataclass(frozen=True)
class Preset:
    name: str
    seed: int
    dtype: str          # "fp32" or "bf16": storage dtype of every tensor
    B: int
    n: int              # padded node count
    dx: int
    de: int
    dy: int
    H: int
    dh: int
    family: str         # "dense", "planar", "tree", "sbm"
    training: bool      # True: forward + backward is the workload
    # family parameters
    n_real: tuple = ()          # fixed real node counts (dense family)
    n_real_range: tuple = ()    # (lo, hi) inclusive, uniform
    p_edge: float = 0.0         # planar-shaped Bernoulli density
    p_in: float = 0.0
    p_out: float = 0.0
    blocks: tuple = ()          # sbm: (k_min, k_max, size_min, size_max) or ("even", k)

    @property
    def pairs(self) -> int:
        return self.B * self.n * self.n


PRESETS = {
    "tiny": Preset("tiny", 0, "fp32", B=2, n=12, dx=16, de=8, dy=8, H=2, dh=8,
                   family="dense", training=False, n_real=(9, 12)),
    "planar": Preset("planar", 1, "bf16", B=64, n=64, dx=256, de=64, dy=64, H=8, dh=32,
                     family="planar", training=False, p_edge=0.09),
    "tree": Preset("tree", 2, "bf16", B=64, n=64, dx=256, de=64, dy=64, H=8, dh=32,
                   family="tree", training=False),
    "sbm": Preset("sbm", 3, "bf16", B=32, n=192, dx=256, de=64, dy=64, H=8, dh=32,
                  family="sbm", training=True, n_real_range=(44, 187),
                  p_in=0.3, p_out=0.05, blocks=(2, 5, 20, 40)),
    "large": Preset("large", 4, "bf16", B=4, n=1024, dx=256, de=64, dy=64, H=8, dh=32,
                    family="sbm", training=True, n_real_range=(768, 1024),
                    p_in=0.05, p_out=0.005, blocks=("even", 8)),
}


def preset(name: str, **overrides) -> Preset:
    """Return a named preset, optionally with fields replaced (e.g. a smaller B)."""
    p = PRESETS[name]
    return dataclasses.replace(p, **overrides) if overrides else p


# ---------------------------------------------------------------- rounding


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even.

    Finite inputs only (the sum below cannot carry out of 32 bits for them).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    out = np.empty(x.shape, np.uint16)
    flat_u, flat_o = u.reshape(-1), out.reshape(-1)
    step = 1 << 24
    for s in range(0, flat_u.size, step):
        c = flat_u[s:s + step]
        flat_o[s:s + step] = ((c + np.uint32(0x7FFF) + ((c >> np.uint32(16)) & np.uint32(1)))
                              >> np.uint32(16)).astype(np.uint16)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Values of x as the storage dtype represents them, held in float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "fp32":
        return x
    u = x.view(np.uint32).reshape(-1)
    step = 1 << 24
    for s in range(0, u.size, step):
        c = u[s:s + step]
        c[:] = ((c + np.uint32(0x7FFF) + ((c >> np.uint32(16)) & np.uint32(1)))
                >> np.uint32(16)) << np.uint32(16)
    return x


# ---------------------------------------------------------------- graph samplers


def planar_adjacency(rng: np.random.Generator, n: int, p: float) -> np.ndarray:
    """Symmetric Bernoulli(p) adjacency, empty diagonal."""
    up = rng.random((n, n)) < p
    a = np.triu(up, 1)
    return (a | a.T).astype(np.uint8)


def prufer_tree_adjacency(rng: np.random.Generator, n: int) -> np.ndarray:
    """Uniform labelled tree on n nodes: decode a uniform Pruefer sequence."""
    a = np.zeros((n, n), np.uint8)
    if n < 2:
        return a
    if n == 2:
        a[0, 1] = a[1, 0] = 1
        return a
    seq = rng.integers(0, n, size=n - 2)
    degree = np.ones(n, np.int64)
    for v in seq:
        degree[v] += 1
    for v in seq:
        leaf = int(np.flatnonzero(degree == 1)[0])
        a[leaf, v] = a[v, leaf] = 1
        degree[leaf] -= 1
        degree[v] -= 1
    u, w = np.flatnonzero(degree == 1)
    a[u, w] = a[w, u] = 1
    return a


def sbm_block_sizes(rng: np.random.Generator, n_real: int, spec: tuple) -> list:
    """Block sizes summing to n_real.

    spec = (k_min, k_max, size_min, size_max): k uniform over the feasible
    counts, sizes a uniform bounded composition (rejection sampling).
    spec = ("even", k): k blocks whose sizes differ by at most one, the
    larger ones placed at random.
    """
    if spec[0] == "even":
        k = spec[1]
        base, extra = divmod(n_real, k)
        sizes = [base] * k
        for idx in rng.permutation(k)[:extra]:
            sizes[idx] += 1
        return sizes
    k_min, k_max, s_min, s_max = spec
    lo = max(k_min, math.ceil(n_real / s_max))
    hi = min(k_max, n_real // s_min)
    if lo > hi:
        raise ValueError(f"no feasible block count for n_real={n_real}")
    k = int(rng.integers(lo, hi + 1))
    while True:
        sizes = rng.integers(s_min, s_max + 1, size=k - 1)
        last = n_real - int(sizes.sum())
        if s_min <= last <= s_max:
            return [int(s) for s in sizes] + [last]


def sbm_adjacency(rng: np.random.Generator, n: int, n_real: int, sizes: list,
                  p_in: float, p_out: float) -> np.ndarray:
    """SBM adjacency on the first n_real nodes, zero elsewhere."""
    labels = np.repeat(np.arange(len(sizes)), sizes)
    same = labels[:, None] == labels[None, :]
    prob = np.where(same, p_in, p_out)
    up = rng.random((n_real, n_real)) < prob
    a_real = np.triu(up, 1)
    a = np.zeros((n, n), np.uint8)
    a[:n_real, :n_real] = a_real | a_real.T
    return a


# ---------------------------------------------------------------- full draw


WEIGHT_NAMES = ("Wq", "bq", "Wk", "bk", "Wv", "bv", "Wfe", "Wfy", "bf", "We", "Wo", "bo")


def weight_shapes(p: Preset) -> dict:
    """[in, out] shapes (row-major, Y = X @ W) and the fan-in of each draw."""
    hd = p.H * p.dh
    return {
        "Wq": ((p.dx, hd), p.dx), "bq": ((hd,), p.dx),
        "Wk": ((p.dx, hd), p.dx), "bk": ((hd,), p.dx),
        "Wv": ((p.dx, hd), p.dx), "bv": ((hd,), p.dx),
        "Wfe": ((p.de, 2 * p.H), p.de), "Wfy": ((p.dy, 2 * p.H), p.dy),
        "bf": ((2 * p.H,), p.de),
        "We": ((p.H, p.de), p.H),
        "Wo": ((hd, p.dx), hd), "bo": ((p.dx,), hd),
    }


def draw_weights(p: Preset, seed_offset: int = 1000) -> dict:
    """Weights and biases ~ N(0,1)/sqrt(fan_in), rounded to the storage dtype."""
    rng = np.random.default_rng(p.seed + seed_offset)
    out = {}
    for name in WEIGHT_NAMES:
        shape, fan_in = weight_shapes(p)[name]
        w = rng.standard_normal(shape) / math.sqrt(fan_in)
        out[name] = to_storage(w, p.dtype)
    return out


# parameters of the graph-transformer block around the layer: per sub-block
# (x node, e edge, y global) LayerNorm 1, the FFN (hidden width twice the
# feature width) and LayerNorm 2; then the pooling maps of the global update
BLOCK_SUB_PARAMS = ("ln1_g", "ln1_s", "W1", "b1", "W2", "b2", "ln2_g", "ln2_s")
BLOCK_WEIGHT_NAMES = tuple(f"{s}_{k}" for s in ("x", "e", "y") for k in BLOCK_SUB_PARAMS) + ("Wyx", "Wye", "by")


def block_weight_shapes(p: Preset) -> dict:
    """[in, out] shapes of the block's parameters and the fan-in of each draw
    (None for LayerNorm parameters)."""
    out = {}
    for s, w in (("x", p.dx), ("e", p.de), ("y", p.dy)):
        f = 2 * w
        out.update({f"{s}_ln1_g": ((w,), None), f"{s}_ln1_s": ((w,), None),
                    f"{s}_W1": ((w, f), w), f"{s}_b1": ((f,), w),
                    f"{s}_W2": ((f, w), f), f"{s}_b2": ((w,), f),
                    f"{s}_ln2_g": ((w,), None), f"{s}_ln2_s": ((w,), None)})
    out.update({"Wyx": ((p.dx, p.dy), p.dx), "Wye": ((p.de, p.dy), p.de), "by": ((p.dy,), p.dx)})
    return out


def draw_block_weights(p: Preset, seed_offset: int = 2000) -> dict:
    """Block parameters: matrices and biases ~ N(0,1)/sqrt(fan_in); LayerNorm
    gains 1 + 0.1 N(0,1), shifts 0.1 N(0,1); rounded to the storage dtype."""
    rng = np.random.default_rng(p.seed + seed_offset)
    out = {}
    for name in BLOCK_WEIGHT_NAMES:
        shape, fan_in = block_weight_shapes(p)[name]
        r = rng.standard_normal(shape)
        if fan_in is not None:
            w = r / math.sqrt(fan_in)
        elif name.endswith("_g"):
            w = 1.0 + 0.1 * r
        else:
            w = 0.1 * r
        out[name] = to_storage(w, p.dtype)
    return out


def draw_block_upstream(p: Preset, seed_offset: int = 3000) -> np.ndarray:
    """Upstream gradient of the block's global output, dyout [B, dy] ~ N(0,1)."""
    rng = np.random.default_rng(p.seed + seed_offset)
    return to_storage(rng.standard_normal((p.B, p.dy)), p.dtype)


def _symmetric_noise(rng, n, de, std, dtype=np.float32):
    r = rng.standard_normal((n, n, de), dtype=np.float32) * np.float32(std)
    iu = np.triu(np.ones((n, n), bool))
    return np.where(iu[:, :, None], r, r.transpose(1, 0, 2)).astype(dtype, copy=False)


def draw_inputs(p: Preset, with_grads: bool | None = None) -> dict:
    """Seeded inputs of one preset.

    Returns float32 arrays holding storage-dtype values: X [B,n,dx],
    E [B,n,n,de], y [B,dy], M [B,n] (uint8), adjacency A [B,n,n] (uint8),
    n_real [B], and, when with_grads (default: p.training), the upstream
    gradients dXout [B,n,dx] and dEout [B,n,n,de] ~ N(0,1).
    """
    if with_grads is None:
        with_grads = p.training
    rng = np.random.default_rng(p.seed)
    B, n, de = p.B, p.n, p.de
    if p.family == "dense":
        n_real = np.array([p.n_real[b % len(p.n_real)] for b in range(B)], np.int64)
    elif p.n_real_range:
        lo, hi = p.n_real_range
        n_real = rng.integers(lo, hi + 1, size=B)
    else:
        n_real = np.full(B, n, np.int64)
    M = (np.arange(n)[None, :] < n_real[:, None]).astype(np.uint8)

    A = np.zeros((B, n, n), np.uint8)
    E = np.empty((B, n, n, de), np.float32)
    if p.family == "dense":
        for b in range(B):
            E[b] = _symmetric_noise(rng, n, de, 1.0)
    else:
        cls = rng.standard_normal((2, de), dtype=np.float32)
        for b in range(B):
            nr = int(n_real[b])
            if p.family == "planar":
                A[b] = planar_adjacency(rng, n, p.p_edge)
            elif p.family == "tree":
                A[b] = prufer_tree_adjacency(rng, n)
            elif p.family == "sbm":
                sizes = sbm_block_sizes(rng, nr, p.blocks)
                A[b] = sbm_adjacency(rng, n, nr, sizes, p.p_in, p.p_out)
            else:
                raise ValueError(p.family)
            eb = _symmetric_noise(rng, n, de, 0.1)
            eb += cls[A[b].astype(np.int64)]
            E[b] = eb
    X = rng.standard_normal((B, n, p.dx), dtype=np.float32)
    y = rng.standard_normal((B, p.dy), dtype=np.float32)
    out = {
        "X": to_storage(X, p.dtype),
        "E": to_storage(E, p.dtype),
        "y": to_storage(y, p.dtype),
        "M": M,
        "A": A,
        "n_real": n_real,
    }
    del E
    if with_grads:
        grng = np.random.default_rng(p.seed + 2000)
        out["dXout"] = to_storage(grng.standard_normal((B, n, p.dx), dtype=np.float32), p.dtype)
        out["dEout"] = to_storage(grng.standard_normal((B, n, n, de), dtype=np.float32), p.dtype)
    return out
