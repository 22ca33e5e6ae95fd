"""Pins of the block oracle (oracle/block.py): the graph-transformer block
around the layer (LayerNorm, FFNs, global update from pooled features).

Each pin checks the oracle against something other than itself:
  - the LayerNorm closed form (zero mean, second moment var / (var + eps));
  - torch's float64 LayerNorm / Linear / ReLU modules for every sub-block's
    forward, and torch autograd for its backward;
  - the pooling's closed forms (constant features pool to the constant; one
    valid edge entry moves y1 by delta * Wye[c] / cnt^2) and its independence
    of padding;
  - the masked outputs (padding rows and invalid pairs are zero);
  - central finite differences of the whole block, layer included, for every
    input and parameter on a tiny case.
A planted mistake in the oracle (a wrong eps, a dropped pooling term, a
scaled gradient, an unmasked upstream gradient) fails at least one of them (the mutant tests below).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import block as OB
from edge_aware_graph_b200 import inputs as I


def _rng(seed):
    return np.random.default_rng(seed)


def _sub_params(rng, w):
    f = 2 * w
    return {"ln1_g": 1 + 0.1 * rng.standard_normal(w), "ln1_s": 0.1 * rng.standard_normal(w),
            "W1": rng.standard_normal((w, f)) / np.sqrt(w), "b1": rng.standard_normal(f) / np.sqrt(w),
            "W2": rng.standard_normal((f, w)) / np.sqrt(f), "b2": rng.standard_normal(w) / np.sqrt(f),
            "ln2_g": 1 + 0.1 * rng.standard_normal(w), "ln2_s": 0.1 * rng.standard_normal(w)}


def test_block_weight_names_agree_with_the_input_generator():
    assert OB.BLOCK_WEIGHT_NAMES == I.BLOCK_WEIGHT_NAMES


def test_round_bf16_against_torch():
    rng = _rng(2)
    x = np.concatenate([rng.standard_normal(5000) * 10.0 ** rng.integers(-6, 6, 5000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.01171875, -3.0078125]])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(OB.round_bf16(x), ref)


def test_layer_norm_closed_form():
    rng = _rng(1)
    z = rng.standard_normal((50, 64)) * rng.uniform(0.01, 5, (50, 1)) + rng.standard_normal((50, 1))
    out, xh, r = OB.layer_norm(z, np.ones(64), np.zeros(64))
    var = z.var(axis=-1)
    np.testing.assert_allclose(out.mean(-1), 0, atol=1e-12)
    np.testing.assert_allclose((out ** 2).mean(-1), var / (var + 1e-5), rtol=1e-12)
    # a constant row normalises to zero (no division by zero)
    out0, _, _ = OB.layer_norm(np.full((1, 8), 3.0), np.ones(8), np.full(8, 0.5))
    np.testing.assert_allclose(out0, 0.5)


class _TorchSub(torch.nn.Module):
    def __init__(self, P, w):
        super().__init__()
        f = 2 * w
        self.ln1 = torch.nn.LayerNorm(w, eps=1e-5, dtype=torch.float64)
        self.l1 = torch.nn.Linear(w, f, dtype=torch.float64)
        self.l2 = torch.nn.Linear(f, w, dtype=torch.float64)
        self.ln2 = torch.nn.LayerNorm(w, eps=1e-5, dtype=torch.float64)
        with torch.no_grad():
            self.ln1.weight.copy_(torch.from_numpy(P["ln1_g"]))
            self.ln1.bias.copy_(torch.from_numpy(P["ln1_s"]))
            self.l1.weight.copy_(torch.from_numpy(P["W1"].T.copy()))
            self.l1.bias.copy_(torch.from_numpy(P["b1"]))
            self.l2.weight.copy_(torch.from_numpy(P["W2"].T.copy()))
            self.l2.bias.copy_(torch.from_numpy(P["b2"]))
            self.ln2.weight.copy_(torch.from_numpy(P["ln2_g"]))
            self.ln2.bias.copy_(torch.from_numpy(P["ln2_s"]))

    def forward(self, z):
        a = self.ln1(z)
        return self.ln2(a + self.l2(torch.relu(self.l1(a))))

    def grads(self):
        return {"ln1_g": self.ln1.weight.grad, "ln1_s": self.ln1.bias.grad,
                "W1": self.l1.weight.grad.T, "b1": self.l1.bias.grad,
                "W2": self.l2.weight.grad.T, "b2": self.l2.bias.grad,
                "ln2_g": self.ln2.weight.grad, "ln2_s": self.ln2.bias.grad}


@pytest.mark.parametrize("shape", [(3, 5, 16), (2, 4, 4, 8), (6, 8)])
def test_sub_block_matches_torch_modules_and_autograd(shape):
    rng = _rng(sum(shape))
    w = shape[-1]
    P = _sub_params(rng, w)
    Z = rng.standard_normal(shape) * 2 + 0.5
    dZo = rng.standard_normal(shape)
    Zo, cache = OB.sub_forward(Z, P)
    dZ, g = OB.sub_backward(dZo, P, cache)

    mod = _TorchSub(P, w)
    zt = torch.from_numpy(Z).requires_grad_(True)
    out = mod(zt)
    np.testing.assert_allclose(Zo, out.detach().numpy(), rtol=1e-12, atol=1e-12)
    out.backward(torch.from_numpy(dZo))
    np.testing.assert_allclose(dZ, zt.grad.numpy(), rtol=1e-10, atol=1e-11)
    for k, v in mod.grads().items():
        np.testing.assert_allclose(g[k], v.numpy(), rtol=1e-10, atol=1e-11, err_msg=k)


def _tiny(n=12, seed=0):
    p = I.preset("tiny", n=n)
    d = I.draw_inputs(p, with_grads=True)
    d["M"][1, 7:] = 0                      # graph 1: 7 real nodes
    W = I.draw_weights(p)
    Wb = I.draw_block_weights(p)
    dyo = I.draw_block_upstream(p)
    return p, d, W, Wb, dyo


def test_outputs_are_zero_on_padding():
    p, d, W, Wb, _ = _tiny()
    out = OB.block_forward(dict(H=p.H, dh=p.dh), d["X"], d["E"], d["y"], d["M"], W, Wb)
    M = d["M"].astype(bool)
    assert np.all(out["Xout"][~M] == 0)
    inval = ~(M[:, :, None] & M[:, None, :])
    assert np.all(out["Eout"][inval] == 0)
    assert np.all(np.abs(out["Xout"][M]).sum(-1) > 0)


def test_pooling_closed_forms_and_padding_independence():
    rng = _rng(5)
    B, n, dx, de, dy = 3, 6, 8, 4, 4
    M = np.ones((B, n), np.uint8)
    M[1, 4:] = 0
    M[2, :] = 0                              # a graph without nodes pools to zero
    p = I.preset("tiny", n=n, dx=dx, de=de, dy=dy)
    Wb = {k: np.asarray(v, np.float64) for k, v in I.draw_block_weights(p).items()}
    cx = rng.standard_normal((B, dx))
    ce = rng.standard_normal((B, de))
    Xm = np.broadcast_to(cx[:, None, :], (B, n, dx)).copy()
    Em = np.broadcast_to(ce[:, None, None, :], (B, n, n, de)).copy()
    # padding holds garbage: it must not enter the means
    Xm[1, 4:] += 100.0
    Em[1, 4:, :] -= 50.0
    Em[1, :, 4:] += 70.0
    Xm[2] += 9.0
    Em[2] += 9.0
    pX, pE = OB.pooled(Xm, Em, M)
    np.testing.assert_allclose(pX[:2], cx[:2], rtol=1e-13)
    np.testing.assert_allclose(pE[:2], ce[:2], rtol=1e-13)
    assert np.all(pX[2] == 0) and np.all(pE[2] == 0)
    y = rng.standard_normal((B, dy))
    base, _ = OB.block_tail_forward(Xm, Em, y, M, Wb)
    # one valid edge entry moves y1 by delta * Wye[c] / cnt^2 (cnt = 4 in graph 1)
    Em2 = Em.copy()
    Em2[1, 2, 3, 1] += 0.25
    moved, _ = OB.block_tail_forward(Xm, Em2, y, M, Wb)
    np.testing.assert_allclose(moved["y1"][1] - base["y1"][1], 0.25 * Wb["Wye"][1] / 16.0, rtol=1e-9, atol=1e-14)
    np.testing.assert_allclose(moved["y1"][0], base["y1"][0], rtol=0, atol=0)
    # one real node's features move y1 by delta * Wyx[c] / cnt
    Xm2 = Xm.copy()
    Xm2[0, 5, 3] -= 0.5
    moved, _ = OB.block_tail_forward(Xm2, Em, y, M, Wb)
    np.testing.assert_allclose(moved["y1"][0] - base["y1"][0], -0.5 * Wb["Wyx"][3] / 6.0, rtol=1e-9, atol=1e-14)


def _loss(p, d, W, Wb, dyo, X, E, y):
    out = OB.block_forward(dict(H=p.H, dh=p.dh), X, E, y, d["M"], W, Wb)
    return (float(np.sum(out["Xout"] * d["dXout"])) + float(np.sum(out["Eout"] * d["dEout"]))
            + float(np.sum(out["yout"] * dyo)))


def test_block_gradients_match_finite_differences():
    p, d, W, Wb, dyo = _tiny()
    W = {k: np.asarray(v, np.float64) for k, v in W.items()}
    Wb = {k: np.asarray(v, np.float64) for k, v in Wb.items()}
    X, E, y = (np.asarray(d[k], np.float64) for k in ("X", "E", "y"))
    g = OB.block_backward(dict(H=p.H, dh=p.dh), X, E, y, d["M"], W, Wb, d["dXout"], d["dEout"], dyo)
    rng = _rng(11)
    h = 1e-6

    def check(arr, grad, name, count):
        for _ in range(count):
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            old = arr[idx]
            arr[idx] = old + h
            lp = _loss(p, d, W, Wb, dyo, X, E, y)
            arr[idx] = old - h
            lm = _loss(p, d, W, Wb, dyo, X, E, y)
            arr[idx] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-5 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])

    check(X, g["dX"], "X", 4)
    # E: a real pair, and a pair touching a padding node of graph 1
    check(E, g["dE"], "E", 4)
    check(y, g["dy"], "y", 3)
    for k in ("Wq", "Wfe", "Wfy", "We", "Wo", "bo"):
        check(W[k], g["d" + k], k, 1)
    for k in OB.BLOCK_WEIGHT_NAMES:
        check(Wb[k], g["d" + k], k, 2)


# ---------------------------------------------------------------- mutants


def test_mutant_wrong_eps_is_caught(monkeypatch):
    monkeypatch.setattr(OB, "LN_EPS", 1e-3)
    with pytest.raises(AssertionError):
        test_sub_block_matches_torch_modules_and_autograd((2, 4, 4, 8))


def test_mutant_dropped_edge_pooling_is_caught(monkeypatch):
    real = OB.pooled
    monkeypatch.setattr(OB, "pooled", lambda Xm, Em, M: (real(Xm, Em, M)[0], 0 * real(Xm, Em, M)[1]))
    with pytest.raises(AssertionError):
        test_pooling_closed_forms_and_padding_independence()


def test_mutant_scaled_ffn_gradient_is_caught(monkeypatch):
    real = OB.sub_backward

    def bad(dZo, P, c):
        dZ, g = real(dZo, P, c)
        if g["W1"].shape[0] == g["W1"].shape[1] // 2:
            g["W1"] = g["W1"] * 1.01
        return dZ, g
    monkeypatch.setattr(OB, "sub_backward", bad)
    with pytest.raises(AssertionError):
        test_block_gradients_match_finite_differences()


def test_mutant_unmasked_edge_gradient_is_caught(monkeypatch):
    real = OB.block_tail_backward

    def bad(Xm, Em, y, M, Wb, dXout, dEout, dyout):
        # the upstream edge gradient no longer masked: padding pairs leak in
        return real(Xm, Em, y, np.ones_like(M), Wb, dXout, dEout, dyout)
    monkeypatch.setattr(OB, "block_tail_backward", bad)
    with pytest.raises(AssertionError):
        test_block_gradients_match_finite_differences()
