"""CPU checks of the seeded input generators against the structure they claim:
the graph families the synthetic workloads stand in for (Planar-, Tree- and
SBM-shaped graphs of the pages' experiments), and the rounding of every drawn
value to the storage dtype."""
import collections
import math

import numpy as np
import pytest
import torch

from edge_aware_graph_b200 import inputs as I


def is_connected(a):
    n = a.shape[0]
    seen, stack = {0}, [0]
    while stack:
        u = stack.pop()
        for v in np.flatnonzero(a[u]):
            if int(v) not in seen:
                seen.add(int(v))
                stack.append(int(v))
    return len(seen) == n


def test_planar_adjacency_is_symmetric_bernoulli():
    rng = np.random.default_rng(5)
    n, p = 64, 0.09
    dens = []
    for _ in range(50):
        a = I.planar_adjacency(rng, n, p)
        assert a.dtype == np.uint8 and (a == a.T).all() and not a.diagonal().any()
        dens.append(a[np.triu_indices(n, 1)].mean())
    # 50 x 2016 Bernoulli(0.09) draws: standard error ~ 0.0014
    assert abs(np.mean(dens) - p) < 0.006


@pytest.mark.parametrize("n", [2, 3, 7, 64])
def test_prufer_trees_are_trees(n):
    rng = np.random.default_rng(n)
    for _ in range(20):
        a = I.prufer_tree_adjacency(rng, n)
        assert (a == a.T).all() and not a.diagonal().any()
        assert int(a.sum()) // 2 == n - 1                 # n - 1 edges
        assert is_connected(a)                            # + connected = a tree


def test_prufer_trees_are_uniform_over_labelled_trees():
    # Cayley: n^(n-2) labelled trees on n nodes (16 for n = 4); Pruefer
    # decoding of a uniform sequence hits each with probability 1/16
    rng = np.random.default_rng(11)
    n, draws = 4, 16000
    counts = collections.Counter()
    for _ in range(draws):
        a = I.prufer_tree_adjacency(rng, n)
        counts[tuple(np.flatnonzero(np.triu(a, 1)))] += 1
    assert len(counts) == n ** (n - 2)
    expected = draws / len(counts)
    chi2 = sum((c - expected) ** 2 / expected for c in counts.values())
    assert chi2 < 40.0          # 15 degrees of freedom: P(chi2 > 40) < 1e-3


@pytest.mark.parametrize("n_real", [44, 60, 99, 140, 187])
def test_sbm_block_sizes_bounded_composition(n_real):
    rng = np.random.default_rng(n_real)
    spec = I.preset("sbm").blocks
    k_min, k_max, s_min, s_max = spec
    ks = set()
    for _ in range(40):
        sizes = I.sbm_block_sizes(rng, n_real, spec)
        assert sum(sizes) == n_real
        assert all(s_min <= s <= s_max for s in sizes)
        assert k_min <= len(sizes) <= k_max
        ks.add(len(sizes))
    feasible = set(range(max(k_min, math.ceil(n_real / s_max)), min(k_max, n_real // s_min) + 1))
    assert ks <= feasible
    if len(feasible) > 1:
        assert len(ks) > 1          # the count is drawn, not fixed


def test_sbm_even_blocks():
    rng = np.random.default_rng(3)
    for n_real in (768, 800, 1023, 1024):
        sizes = I.sbm_block_sizes(rng, n_real, ("even", 8))
        assert len(sizes) == 8 and sum(sizes) == n_real and max(sizes) - min(sizes) <= 1


def test_sbm_adjacency_densities_and_padding():
    rng = np.random.default_rng(9)
    n, n_real, sizes, p_in, p_out = 192, 180, [40, 40, 40, 30, 30], 0.3, 0.05
    labels = np.repeat(np.arange(len(sizes)), sizes)
    same = labels[:, None] == labels[None, :]
    iu = np.triu_indices(n_real, 1)
    ins, outs = [], []
    for _ in range(20):
        a = I.sbm_adjacency(rng, n, n_real, sizes, p_in, p_out)
        assert (a == a.T).all() and not a.diagonal().any()
        assert not a[n_real:].any() and not a[:, n_real:].any()
        up = a[:n_real, :n_real][iu].astype(bool)
        ins.append(up[same[iu]].mean())
        outs.append(up[~same[iu]].mean())
    assert abs(np.mean(ins) - p_in) < 0.02
    assert abs(np.mean(outs) - p_out) < 0.01


@pytest.mark.parametrize("name", ["planar", "tree"])
def test_edge_features_are_symmetric_and_follow_the_graph(name):
    p = I.preset(name, B=3)
    d = I.draw_inputs(p)
    E, A = d["E"], d["A"]
    assert (E == E.transpose(0, 2, 1, 3)).all()
    assert d["M"].all()                                   # all nodes real
    # E_ij = c[A_ij] + noise of standard deviation 0.1: the two classes separate
    b = 0
    m1 = E[b][A[b] == 1].mean(axis=0)
    m0 = E[b][(A[b] == 0) & ~np.eye(p.n, dtype=bool)].mean(axis=0)
    assert np.abs(m1 - m0).max() > 0.5


def test_sbm_masks_are_prefixes_in_range():
    p = I.preset("sbm", B=8)
    d = I.draw_inputs(p, with_grads=False)
    lo, hi = p.n_real_range
    for b in range(p.B):
        nr = int(d["n_real"][b])
        assert lo <= nr <= hi
        assert d["M"][b, :nr].all() and not d["M"][b, nr:].any()


def test_bf16_rounding_matches_torch():
    # torch's float32 -> bfloat16 conversion rounds to nearest, ties to even
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * np.float32(10.0),
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 0.0, -0.0, 65504.0,
                  1e-30, 3.0e38], np.float32),                       # ties, signed zero, tiny, huge
    ])
    ours = I.round_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (ours == ref).all()
    st = I.to_storage(x, "bf16")
    assert (st == I.bf16_bits_to_f32(ours)).all()
    assert (I.to_storage(st, "bf16") == st).all()          # idempotent
