"""Pins of the fp64 CPU oracle against facts that do not come from the oracle.

The paper's pages print no worked example for the layer, so the oracle is
pinned by:
  - special cases that reduce to library routines (torch float64 scaled dot
    product attention and softmax, scipy softmax over the [V | I] trick),
  - closed forms (gamma = -1 gives uniform attention over real nodes),
  - invariants (row sums, masked-entry invariance, permutation equivariance,
    beta-shift invariance and its zero gradient),
  - brute force on the tiny preset (a per-pair pure-Python evaluation without
    max subtraction; fp64 central finite differences of the forward for every
    gradient the backward returns, and torch autograd in the zero-FiLM case).
Each is chosen so that a dropped term, a wrong sign or index, or a transposed
operand in the oracle fails at least one of them.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

from edge_aware_graph_b200 import inputs as I

WN = I.WEIGHT_NAMES


def tiny(seed=None, **over):
    p = I.preset("tiny", **over)
    if seed is not None:
        p = I.preset("tiny", seed=seed, **over)
    d = I.draw_inputs(p, with_grads=True)
    W = I.draw_weights(p)
    dims = dict(H=p.H, dh=p.dh)
    return p, dims, d, W


def valid_mask(M):
    return (M[:, :, None] & M[:, None, :]).astype(bool)


def qkv(p, X, W):
    Q = X.astype(np.float64) @ W["Wq"].astype(np.float64) + W["bq"]
    K = X.astype(np.float64) @ W["Wk"].astype(np.float64) + W["bk"]
    V = X.astype(np.float64) @ W["Wv"].astype(np.float64) + W["bv"]
    B, n, _ = X.shape
    sh = lambda t: t.reshape(B, n, p.H, p.dh).transpose(0, 2, 1, 3)  # [B,H,n,dh]
    return sh(Q), sh(K), sh(V)


def zero_film(W, H, gamma=0.0, beta=0.0):
    W = dict(W)
    W["Wfe"] = np.zeros_like(W["Wfe"])
    W["Wfy"] = np.zeros_like(W["Wfy"])
    W["bf"] = np.concatenate([np.full(H, gamma), np.full(H, beta)]).astype(np.float32)
    return W


# --------------------------------------------------------------- special case → library


def test_zero_film_is_masked_sdpa(oracle_lib):
    p, dims, d, W = tiny()
    W = zero_film(W, p.H)
    out = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, want_attention=True)
    Q, K, V = qkv(p, d["X"], W)
    valid = torch.from_numpy(valid_mask(d["M"]))[:, None]          # [B,1,n,n]
    rows = d["M"].astype(bool)
    Qt, Kt, Vt = (torch.from_numpy(np.ascontiguousarray(t)) for t in (Q, K, V))
    # rows of masked nodes have no valid key; give them a dummy key so SDPA stays finite
    mask = valid | torch.from_numpy(~rows)[:, None, :, None]
    ref = torch.nn.functional.scaled_dot_product_attention(Qt, Kt, Vt, attn_mask=mask)
    ref = ref.permute(0, 2, 1, 3).reshape(p.B, p.n, p.H * p.dh).numpy()
    np.testing.assert_allclose(out["O"][rows], ref[rows], rtol=0, atol=1e-12)
    assert np.all(out["O"][~rows] == 0.0)
    # attention map against torch softmax, then the two residuals
    s = torch.einsum("bhid,bhjd->bhij", Qt, Kt) / math.sqrt(p.dh)
    a = torch.softmax(s.masked_fill(~mask, float("-inf")), dim=-1)
    a = torch.where(valid, a, torch.zeros_like(a)).numpy()
    np.testing.assert_allclose(out["A"], a, rtol=0, atol=1e-12)
    Eref = d["E"] + np.einsum("bhij,hc->bijc", a, W["We"].astype(np.float64))
    np.testing.assert_allclose(out["Eout"], Eref, rtol=0, atol=1e-12)
    Xref = d["X"] + rows[:, :, None] * (ref @ W["Wo"].astype(np.float64) + W["bo"])
    np.testing.assert_allclose(out["Xout"], Xref, rtol=0, atol=1e-12)


def test_light_edge_is_sdpa_with_a_global_temperature(oracle_lib):
    """Light Edge (no per-edge modulation) is the layer with Wfe = 0: gamma and
    beta are then constant per graph and head, beta cancels in the softmax, and
    the map is scaled dot-product attention at scale (1 + gamma_bh) / sqrt(dh)."""
    p, dims, d, W = tiny(seed=7)
    W = dict(W)
    W["Wfe"] = np.zeros_like(W["Wfe"])
    out = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, want_attention=True)
    g = d["y"].astype(np.float64) @ W["Wfy"].astype(np.float64) + W["bf"]       # [B, 2H]
    assert np.abs(g[:, p.H:]).max() > 0.1 and np.abs(g[:, :p.H]).max() > 0.1   # beta and gamma both present
    Q, K, V = qkv(p, d["X"], W)
    valid = torch.from_numpy(valid_mask(d["M"]))                                # [B,n,n]
    rows = d["M"].astype(bool)
    mask = valid | torch.from_numpy(~rows)[:, :, None]      # dummy keys for masked rows, as above
    O = np.zeros((p.B, p.n, p.H, p.dh))
    for b in range(p.B):
        for h in range(p.H):
            q, k, v = (torch.from_numpy(np.ascontiguousarray(t[b, h])) for t in (Q, K, V))
            O[b, :, h] = torch.nn.functional.scaled_dot_product_attention(
                q, k, v, attn_mask=mask[b], scale=(1.0 + g[b, h]) / math.sqrt(p.dh)).numpy()
    O = O.reshape(p.B, p.n, p.H * p.dh)
    np.testing.assert_allclose(out["O"][rows], O[rows], rtol=0, atol=1e-11)
    # the map no longer depends on E: a different E changes only the residual
    d2 = dict(d)
    d2["E"] = d["E"] + np.float32(3.0)
    out2 = oracle_lib.forward(dims, d2["X"], d2["E"], d2["y"], d2["M"], W, want_attention=True)
    np.testing.assert_array_equal(out2["A"], out["A"])
    dE_in = d2["E"].astype(np.float64) - d["E"].astype(np.float64)
    np.testing.assert_allclose(out2["Eout"] - out["Eout"], dE_in, rtol=0, atol=1e-12)
    # a key bias adds q_i . bk to every score of row i, times the same (1 + gamma):
    # the softmax cancels it, so its gradient vanishes (it does not with Wfe != 0)
    g = oracle_lib.backward(dims, d["X"], d["E"], d["y"], d["M"], W, d["dXout"], d["dEout"])
    assert np.abs(g["dbk"]).max() <= 1e-12 * np.abs(g["dbq"]).max()
    p3, dims3, d3, W3 = tiny(seed=7)
    g3 = oracle_lib.backward(dims3, d3["X"], d3["E"], d3["y"], d3["M"], W3, d3["dXout"], d3["dEout"])
    assert np.abs(g3["dbk"]).max() > 1e-3 * np.abs(g3["dbq"]).max()


def test_v_concat_identity_formulation(oracle_lib):
    """The pages' trick: attention applied to [V | I] returns O and the map."""
    p, dims, d, W = tiny()
    out = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, want_attention=True)
    Q, K, V = qkv(p, d["X"], W)
    g = d["y"].astype(np.float64) @ W["Wfy"].astype(np.float64) + W["bf"]   # [B,2H]
    f = np.einsum("bijc,ck->bijk", d["E"].astype(np.float64), W["Wfe"].astype(np.float64))
    f = f + g[:, None, None, :]
    gam = f[..., :p.H].transpose(0, 3, 1, 2)
    bet = f[..., p.H:].transpose(0, 3, 1, 2)
    s = np.einsum("bhid,bhjd->bhij", Q, K) / math.sqrt(p.dh)
    sp = s * (1 + gam) + bet
    valid = valid_mask(d["M"])[:, None]
    with np.errstate(invalid="ignore"):      # a fully masked row gives NaN, zeroed below
        P = scipy.special.softmax(np.where(valid, sp, -np.inf), axis=-1)
    P = np.where(valid, np.nan_to_num(P), 0.0)
    VI = np.concatenate([V, np.broadcast_to(np.eye(p.n), (p.B, p.H, p.n, p.n))], axis=-1)
    res = P @ VI
    O = res[..., :p.dh].transpose(0, 2, 1, 3).reshape(p.B, p.n, -1)
    np.testing.assert_allclose(out["O"], O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["A"], res[..., p.dh:], rtol=0, atol=1e-12)


# --------------------------------------------------------------- closed form


def test_gamma_minus_one_is_uniform(oracle_lib):
    p, dims, d, W = tiny()
    W = zero_film(W, p.H, gamma=-1.0, beta=0.0)
    out = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, want_attention=True)
    V = (d["X"].astype(np.float64) @ W["Wv"] + W["bv"])
    for b in range(p.B):
        nr = int(d["n_real"][b])
        assert np.allclose(out["A"][b, :, :nr, :nr], 1.0 / nr, rtol=0, atol=1e-15)
        assert np.all(out["A"][b, :, nr:, :] == 0) and np.all(out["A"][b, :, :, nr:] == 0)
        np.testing.assert_allclose(out["O"][b, :nr], np.broadcast_to(V[b, :nr].mean(0), (nr, V.shape[-1])),
                                   rtol=0, atol=1e-13)
        shift = W["We"].astype(np.float64).sum(0) / nr
        np.testing.assert_allclose(out["Eout"][b, :nr, :nr], d["E"][b, :nr, :nr] + shift, rtol=0, atol=1e-13)
        np.testing.assert_array_equal(out["Eout"][b, nr:], d["E"][b, nr:])
        np.testing.assert_array_equal(out["Eout"][b, :, nr:], d["E"][b, :, nr:])


def test_gamma_minus_one_backward_closed_forms(oracle_lib):
    """gamma = -1, beta = 0: every score is zero and a is uniform over real
    nodes.  Then ds = dS' (1 + gamma) vanishes, so Q and K receive no
    gradient; dV_j is the mean of M dX' Wo^T over the real rows; dWe[h] is the
    per-graph mean of the sum of dE' over valid pairs, the same for every
    head; and dE = dE'."""
    p, dims, d, W = tiny()
    W = zero_film(W, p.H, gamma=-1.0, beta=0.0)
    g = oracle_lib.backward(dims, d["X"], d["E"], d["y"], d["M"], W, d["dXout"], d["dEout"])
    for k in ("dWq", "dbq", "dWk", "dbk"):
        assert np.abs(g[k]).max() <= 1e-13, k
    np.testing.assert_array_equal(g["dE"], d["dEout"].astype(np.float64))
    X, dXo = d["X"].astype(np.float64), d["dXout"].astype(np.float64)
    Wo, Wv = W["Wo"].astype(np.float64), W["Wv"].astype(np.float64)
    dWv = np.zeros_like(Wv)
    dbv = np.zeros(Wv.shape[1])
    dWe = np.zeros((p.H, p.de))
    dX = dXo.copy()
    for b in range(p.B):
        nr = int(d["n_real"][b])
        dO = dXo[b, :nr] @ Wo.T                               # [nr, H*dh], masked rows contribute nothing
        dv = dO.mean(0)                                       # the same for every real j
        dWv += np.outer(X[b, :nr].sum(0), dv)
        dbv += nr * dv
        dWe += d["dEout"][b, :nr, :nr].astype(np.float64).sum((0, 1))[None, :] / nr
        dX[b, :nr] += (dv @ Wv.T)[None, :]
    np.testing.assert_allclose(g["dWv"], dWv, rtol=0, atol=1e-11)
    np.testing.assert_allclose(g["dbv"], dbv, rtol=0, atol=1e-11)
    np.testing.assert_allclose(g["dWe"], dWe, rtol=0, atol=1e-11)
    np.testing.assert_allclose(g["dX"], dX, rtol=0, atol=1e-11)


# --------------------------------------------------------------- invariants


def test_row_sums(oracle_lib):
    p, dims, d, W = tiny()
    out = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, want_attention=True)
    sums = out["A"].sum(-1)                                  # [B,H,n]
    rows = d["M"].astype(bool)[:, None, :].repeat(p.H, 1)
    np.testing.assert_allclose(sums[rows], 1.0, rtol=0, atol=1e-14)
    assert np.all(sums[~rows] == 0)
    cols = ~d["M"].astype(bool)
    for b in range(p.B):
        assert np.all(out["A"][b][:, :, cols[b]] == 0)
    assert np.all(out["A"] >= 0)


def test_masked_entries_do_not_matter(oracle_lib):
    p, dims, d, W = tiny()
    base = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, want_attention=True)
    rng = np.random.default_rng(7)
    X2, E2 = d["X"].copy(), d["E"].copy()
    rows = d["M"].astype(bool)
    valid = valid_mask(d["M"])
    X2[~rows] = rng.standard_normal(X2[~rows].shape) * 100
    E2[~valid] = rng.standard_normal(E2[~valid].shape) * 100
    out = oracle_lib.forward(dims, X2, E2, d["y"], d["M"], W, want_attention=True)
    np.testing.assert_array_equal(out["A"], base["A"])
    np.testing.assert_array_equal(out["Xout"][rows], base["Xout"][rows])
    np.testing.assert_array_equal(out["Eout"][valid], base["Eout"][valid])
    # masked nodes and pairs keep their inputs (residual only)
    np.testing.assert_array_equal(out["Xout"][~rows], X2[~rows])
    np.testing.assert_array_equal(out["Eout"][~valid], E2[~valid])


def test_permutation_equivariance(oracle_lib):
    p, dims, d, W = tiny()
    base = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, want_attention=True)
    perm = np.random.default_rng(3).permutation(p.n)
    Xp = d["X"][:, perm]
    Ep = d["E"][:, perm][:, :, perm]
    Mp = d["M"][:, perm]
    out = oracle_lib.forward(dims, Xp, Ep, d["y"], Mp, W, want_attention=True)
    np.testing.assert_allclose(out["Xout"], base["Xout"][:, perm], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["Eout"], base["Eout"][:, perm][:, :, perm], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["A"], base["A"][:, :, perm][:, :, :, perm], rtol=0, atol=1e-14)


def test_beta_shift_invariance(oracle_lib):
    p, dims, d, W = tiny()
    base = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, want_attention=True)
    W2 = dict(W)
    W2["bf"] = W["bf"].astype(np.float64) + np.concatenate([np.zeros(p.H), np.arange(1, p.H + 1) * 3.0])
    out = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W2, want_attention=True)
    np.testing.assert_allclose(out["A"], base["A"], rtol=0, atol=1e-13)
    g = oracle_lib.backward(dims, d["X"], d["E"], d["y"], d["M"], W, d["dXout"], d["dEout"])
    scale = np.abs(g["dbf"]).max()
    assert np.abs(g["dbf"][p.H:]).max() <= 1e-12 * scale
    assert np.abs(g["dWfy"][:, p.H:]).max() <= 1e-12 * np.abs(g["dWfy"]).max()


# --------------------------------------------------------------- brute force


def brute_forward(p, d, W):
    """Per-pair pure-Python evaluation: no max subtraction, no shared loops."""
    B, n, H, dh, de = p.B, p.n, p.H, p.dh, p.de
    X = d["X"].tolist(); E = d["E"]; y = d["y"].tolist(); M = d["M"].tolist()
    Wd = {k: W[k].astype(float).tolist() for k in WN}
    hd = H * dh

    def lin(x, Wm, bm):
        return [sum(x[k] * Wm[k][o] for k in range(len(x))) + bm[o] for o in range(len(bm))]

    A = np.zeros((B, H, n, n)); O = np.zeros((B, n, hd))
    Eout = E.astype(np.float64).copy(); Xout = d["X"].astype(np.float64).copy()
    for b in range(B):
        q = [lin(X[b][i], Wd["Wq"], Wd["bq"]) for i in range(n)]
        k = [lin(X[b][i], Wd["Wk"], Wd["bk"]) for i in range(n)]
        v = [lin(X[b][i], Wd["Wv"], Wd["bv"]) for i in range(n)]
        gy = lin(y[b], Wd["Wfy"], Wd["bf"])
        for i in range(n):
            if not M[b][i]:
                continue
            for h in range(H):
                w = {}
                for j in range(n):
                    if not M[b][j]:
                        continue
                    e = E[b, i, j].tolist()
                    gam = sum(e[c] * Wd["Wfe"][c][h] for c in range(de)) + gy[h]
                    bet = sum(e[c] * Wd["Wfe"][c][H + h] for c in range(de)) + gy[H + h]
                    s = sum(q[i][h * dh + t] * k[j][h * dh + t] for t in range(dh)) / math.sqrt(dh)
                    w[j] = math.exp(s * (1 + gam) + bet)
                tot = sum(w.values())
                for j, wj in w.items():
                    A[b, h, i, j] = wj / tot
                for t in range(dh):
                    O[b, i, h * dh + t] = sum(A[b, h, i, j] * v[j][h * dh + t] for j in w)
            for j in range(n):
                for c in range(de):
                    Eout[b, i, j, c] += sum(A[b, h, i, j] * Wd["We"][h][c] for h in range(H))
            for o in range(p.dx):
                Xout[b, i, o] += sum(O[b, i, kk] * Wd["Wo"][kk][o] for kk in range(hd)) + Wd["bo"][o]
    return dict(A=A, O=O, Eout=Eout, Xout=Xout)


def test_brute_force_tiny(oracle_lib):
    p, dims, d, W = tiny()
    out = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, want_attention=True)
    ref = brute_forward(p, d, W)
    for k in ("A", "O", "Eout", "Xout"):
        np.testing.assert_allclose(out[k], ref[k], rtol=1e-11, atol=1e-12, err_msg=k)


def _loss(oracle_lib, dims, X, E, y, M, W, dXo, dEo):
    o = oracle_lib.forward(dims, X, E, y, M, W)
    return float((o["Xout"] * dXo).sum() + (o["Eout"] * dEo).sum())


def test_backward_finite_differences(oracle_lib):
    """Every gradient of orc_backward against fp64 central differences of orc_forward."""
    p, dims, d, W = tiny()
    X, E, y = (d[k].astype(np.float64) for k in ("X", "E", "y"))
    Wd = {k: W[k].astype(np.float64) for k in WN}
    dXo, dEo = d["dXout"].astype(np.float64), d["dEout"].astype(np.float64)
    g = oracle_lib.backward(dims, X, E, y, d["M"], Wd, dXo, dEo)
    h = 1e-6
    rng = np.random.default_rng(11)

    def check(name, arr, setter, grad, max_entries=None):
        idx = np.arange(arr.size)
        if max_entries and arr.size > max_entries:
            idx = rng.choice(arr.size, max_entries, replace=False)
        fd = np.empty(len(idx))
        for t, flat in enumerate(idx):
            plus = arr.copy().reshape(-1); plus[flat] += h
            minus = arr.copy().reshape(-1); minus[flat] -= h
            fd[t] = (setter(plus.reshape(arr.shape)) - setter(minus.reshape(arr.shape))) / (2 * h)
        an = grad.reshape(-1)[idx]
        err = np.abs(fd - an).max() / max(np.abs(an).max(), 1e-30)
        assert err < 1e-6, f"{name}: rel err {err:.3e}"

    L = lambda **kw: _loss(oracle_lib, dims, kw.get("X", X), kw.get("E", E), kw.get("y", y), d["M"],
                           kw.get("W", Wd), dXo, dEo)
    check("X", X, lambda a: L(X=a), g["dX"])
    check("E", E, lambda a: L(E=a), g["dE"], max_entries=600)
    check("y", y, lambda a: L(y=a), g["dy"])
    for k in WN:
        def setk(a, k=k):
            W2 = dict(Wd); W2[k] = a
            return L(W=W2)
        check(k, Wd[k], setk, g["d" + k], max_entries=200)


def test_backward_zero_film_autograd(oracle_lib):
    """Zero FiLM: the layer is library attention + linears; torch autograd gives the grads."""
    p, dims, d, W = tiny(seed=5)
    W = zero_film(W, p.H)
    Wd = {k: torch.tensor(W[k], dtype=torch.float64, requires_grad=True) for k in WN}
    X = torch.tensor(d["X"], dtype=torch.float64, requires_grad=True)
    E = torch.tensor(d["E"], dtype=torch.float64, requires_grad=True)
    M = torch.from_numpy(d["M"].astype(bool))
    B, n, H, dh = p.B, p.n, p.H, p.dh
    sh = lambda t: t.reshape(B, n, H, dh).permute(0, 2, 1, 3)
    Q, K, V = (sh(X @ Wd[w] + Wd[b]) for w, b in (("Wq", "bq"), ("Wk", "bk"), ("Wv", "bv")))
    valid = (M[:, :, None] & M[:, None, :])[:, None]
    mask = valid | (~M)[:, None, :, None]
    s = Q @ K.transpose(-1, -2) / math.sqrt(dh)
    a = torch.softmax(s.masked_fill(~mask, float("-inf")), -1)
    a = torch.where(valid, a, torch.zeros_like(a))
    O = (a @ V).permute(0, 2, 1, 3).reshape(B, n, H * dh)
    Xout = X + M[:, :, None] * (O @ Wd["Wo"] + Wd["bo"])
    Eout = E + torch.einsum("bhij,hc->bijc", a, Wd["We"])
    loss = (Xout * torch.from_numpy(d["dXout"]).double()).sum() + (Eout * torch.from_numpy(d["dEout"]).double()).sum()
    loss.backward()
    g = oracle_lib.backward(dims, d["X"], d["E"], d["y"], d["M"], W, d["dXout"], d["dEout"])
    np.testing.assert_allclose(g["dX"], X.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(g["dE"], E.grad.numpy(), rtol=0, atol=1e-11)
    for k in ("Wq", "bq", "Wk", "bk", "Wv", "bv", "We", "Wo", "bo"):
        np.testing.assert_allclose(g["d" + k], Wd[k].grad.numpy(), rtol=0, atol=1e-10, err_msg=k)


def test_masked_gradients_are_residual_only(oracle_lib):
    p, dims, d, W = tiny()
    g = oracle_lib.backward(dims, d["X"], d["E"], d["y"], d["M"], W, d["dXout"], d["dEout"])
    rows = d["M"].astype(bool)
    valid = valid_mask(d["M"])
    np.testing.assert_array_equal(g["dX"][~rows], d["dXout"][~rows])
    np.testing.assert_array_equal(g["dE"][~valid], d["dEout"][~valid])


# --------------------------------------------------------------- ablation variants
# AI-summary page, method paragraph (the ablation of unnormalised coefficients)
# and its "Light Edge" bullet (no per-edge modulation).  Readings:
#   unnormalised: E' = E + sum_h s'^h We[h,:] on valid pairs, s' the modulated
#                 score (the coefficients before the softmax); nodes as the layer;
#   light edge:   gamma, beta from y alone (Wfe absent, its gradient zero).


def test_unnormalised_closed_form(oracle_lib):
    """gamma = -1 and beta = c_h: every modulated score equals c_h, so the
    unnormalised edge update adds sum_h c_h We[h] to each valid pair; node
    outputs stay those of uniform attention."""
    p, dims, d, W = tiny(seed=3)
    c = np.array([0.7, -1.3], dtype=np.float32)[: p.H]
    W = zero_film(W, p.H, gamma=-1.0)
    W["bf"] = np.concatenate([np.full(p.H, -1.0), c]).astype(np.float32)
    out = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, variant="unnormalised")
    lay = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W)
    valid = valid_mask(d["M"])
    shift = (c.astype(np.float64)[:, None] * W["We"].astype(np.float64)).sum(0)      # [de]
    E = d["E"].astype(np.float64)
    np.testing.assert_allclose(out["Eout"][valid], (E + shift)[valid], rtol=0, atol=1e-13)
    np.testing.assert_array_equal(out["Eout"][~valid], E[~valid])
    for k in ("Xout", "O"):
        np.testing.assert_array_equal(out[k], lay[k])


def test_unnormalised_brute_force(oracle_lib):
    """Per-pair pure-Python modulated scores and the edge update they give."""
    p, dims, d, W = tiny()
    out = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, variant="unnormalised")
    H, dh, de = p.H, p.dh, p.de
    Wd = {k: W[k].astype(float).tolist() for k in WN}
    Eref = d["E"].astype(np.float64).copy()
    for b in range(p.B):
        X = d["X"][b].tolist()
        y = d["y"][b].tolist()
        lin = lambda x, Wm, bm: [sum(x[k] * Wm[k][o] for k in range(len(x))) + bm[o] for o in range(len(bm))]
        q = [lin(X[i], Wd["Wq"], Wd["bq"]) for i in range(p.n)]
        k_ = [lin(X[i], Wd["Wk"], Wd["bk"]) for i in range(p.n)]
        gy = lin(y, Wd["Wfy"], Wd["bf"])
        for i in range(p.n):
            for j in range(p.n):
                if not (d["M"][b, i] and d["M"][b, j]):
                    continue
                e = d["E"][b, i, j].tolist()
                for h in range(H):
                    gam = sum(e[c] * Wd["Wfe"][c][h] for c in range(de)) + gy[h]
                    bet = sum(e[c] * Wd["Wfe"][c][H + h] for c in range(de)) + gy[H + h]
                    s = sum(q[i][h * dh + t] * k_[j][h * dh + t] for t in range(dh)) / math.sqrt(dh)
                    sp = s * (1 + gam) + bet
                    for c in range(de):
                        Eref[b, i, j, c] += sp * Wd["We"][h][c]
    np.testing.assert_allclose(out["Eout"], Eref, rtol=1e-12, atol=1e-12)


def test_unnormalised_backward_closed_forms(oracle_lib):
    """gamma = -1, beta = c_h: ds vanishes (no Q, K gradient); the edge path
    reaches beta directly, so dbf[H+h] = sum over valid pairs of We[h] . dE'
    (the softmax alone would give zero) and dWe[h] = c_h times the sum of dE'
    over valid pairs; dE = dE'."""
    p, dims, d, W = tiny(seed=4)
    c = np.array([0.5, -2.0], dtype=np.float32)[: p.H]
    W = zero_film(W, p.H, gamma=-1.0)
    W["bf"] = np.concatenate([np.full(p.H, -1.0), c]).astype(np.float32)
    g = oracle_lib.backward(dims, d["X"], d["E"], d["y"], d["M"], W, d["dXout"], d["dEout"], variant="unnormalised")
    for k in ("dWq", "dbq", "dWk", "dbk"):
        assert np.abs(g[k]).max() <= 1e-13, k
    valid = valid_mask(d["M"])
    sum_dE = d["dEout"].astype(np.float64)[valid].sum(0)                               # [de]
    We = W["We"].astype(np.float64)
    np.testing.assert_allclose(g["dbf"][p.H:], We @ sum_dE, rtol=0, atol=1e-11)
    np.testing.assert_allclose(g["dWe"], c.astype(np.float64)[:, None] * sum_dE[None, :], rtol=0, atol=1e-11)
    np.testing.assert_array_equal(g["dE"], d["dEout"].astype(np.float64))


def test_variant_backward_finite_differences(oracle_lib):
    """Every gradient of both variants against fp64 central differences of their forward."""
    p, dims, d, W = tiny(seed=9)
    X, E, y = (d[k].astype(np.float64) for k in ("X", "E", "y"))
    Wd = {k: W[k].astype(np.float64) for k in WN}
    dXo, dEo = d["dXout"].astype(np.float64), d["dEout"].astype(np.float64)
    h = 1e-6
    rng = np.random.default_rng(12)
    for variant in ("unnormalised", "light_edge"):
        g = oracle_lib.backward(dims, X, E, y, d["M"], Wd, dXo, dEo, variant=variant)

        def L(X=X, E=E, y=y, W=Wd):
            o = oracle_lib.forward(dims, X, E, y, d["M"], W, variant=variant)
            return float((o["Xout"] * dXo).sum() + (o["Eout"] * dEo).sum())

        def check(name, arr, setter, grad, max_entries=None):
            idx = np.arange(arr.size)
            if max_entries and arr.size > max_entries:
                idx = rng.choice(arr.size, max_entries, replace=False)
            fd = np.empty(len(idx))
            for t, flat in enumerate(idx):
                plus = arr.copy().reshape(-1); plus[flat] += h
                minus = arr.copy().reshape(-1); minus[flat] -= h
                fd[t] = (setter(plus.reshape(arr.shape)) - setter(minus.reshape(arr.shape))) / (2 * h)
            an = grad.reshape(-1)[idx]
            # relative 1e-6, plus an absolute 1e-7 for the difference quotients'
            # own rounding (a gradient that is exactly zero, as dbk of Light Edge)
            assert np.abs(fd - an).max() <= 1e-6 * np.abs(an).max() + 1e-7, f"{variant} {name}"

        check("X", X, lambda a: L(X=a), g["dX"])
        check("E", E, lambda a: L(E=a), g["dE"], max_entries=400)
        check("y", y, lambda a: L(y=a), g["dy"])
        for k in WN:
            if variant == "light_edge" and k == "Wfe":
                continue                       # not a parameter of that layer
            def setk(a, k=k):
                W2 = dict(Wd); W2[k] = a
                return L(W=W2)
            check(k, Wd[k], setk, g["d" + k], max_entries=150)


def test_light_edge_variant_ignores_wfe(oracle_lib):
    """Light Edge ignores Wfe: equal to the layer at Wfe = 0 (pinned above
    against scaled dot-product attention), its dWfe is zero and dE = dE'."""
    p, dims, d, W = tiny(seed=6)
    W0 = dict(W)
    W0["Wfe"] = np.zeros_like(W["Wfe"])
    lv = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W, variant="light_edge")
    l0 = oracle_lib.forward(dims, d["X"], d["E"], d["y"], d["M"], W0)
    for k in ("Xout", "Eout", "O", "LSE"):
        np.testing.assert_array_equal(lv[k], l0[k])
    gv = oracle_lib.backward(dims, d["X"], d["E"], d["y"], d["M"], W, d["dXout"], d["dEout"], variant="light_edge")
    assert np.all(gv["dWfe"] == 0)
    np.testing.assert_array_equal(gv["dE"], d["dEout"].astype(np.float64))
