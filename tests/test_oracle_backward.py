"""Pins of the training-side oracle (oracle/backward.py), CPU only.

- Central finite differences of the layer's loss sum(dy * y) along random
  directions, for every weight, the input and the mean's share in W_up, on
  tiny fp64 layers whose router logits all keep a margin from 0 (so no
  activation decision flips inside the difference); plain and gated.
- A second, independent formulation: the layer written as a dense masked
  torch computation and differentiated by torch.autograd in fp64.
- The entropy regulariser: closed forms (k equal weights give log k; one
  active expert or none give 0) and finite differences of its gradient.
- The controller: its three cases and a run of iterations.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O


def _layer(seed, T=3, D=8, E=5, d_e=6, d_s=4, gated=False, margin=0.15):
    rng = np.random.default_rng(seed)
    L = {
        "W_r": rng.standard_normal((E, D)) / math.sqrt(D),
        "W_up": rng.standard_normal((E, d_e, D)) / math.sqrt(D),
        "W_down": rng.standard_normal((E, D, d_e)) / math.sqrt(d_e),
        "s": rng.uniform(0.5, 2.0, E),
        "W_s_up": rng.standard_normal((d_s, D)) / math.sqrt(D),
        "W_s_down": rng.standard_normal((D, d_s)) / math.sqrt(d_s),
    }
    if gated:
        L["W_val"] = rng.standard_normal((E, d_e, D)) / math.sqrt(D)
    x = rng.standard_normal((T, D))
    # biases that leave every logit at least `margin` away from 0, with a mix
    # of active and inactive experts
    zx = x @ L["W_r"].T
    b = rng.uniform(-0.6, 0.3, E)
    for _ in range(200):
        z = zx + b
        close = np.abs(z) < margin
        if not close.any():
            break
        b = b + np.where(close.any(axis=0), 2.5 * margin, 0.0)
    L["b_r"] = b
    assert np.abs(zx + b).min() >= margin
    dy = rng.standard_normal((T, D))
    return L, x, dy


def _loss(L, x, dy, eps):
    """sum(dy * y) with the mean up-projection recomputed from W_up."""
    LL = dict(L)
    LL["W_bar_up"] = L["W_up"].mean(axis=0)
    y, _, _ = O.layer_forward_tokens(x, LL, eps)
    return float(np.sum(dy * y))


def _grads(L, x, dy, eps, dz_extra=None):
    LL = dict(L)
    LL["W_bar_up"] = L["W_up"].mean(axis=0)
    return O.layer_backward_tokens(x, LL, dy, eps, dz_extra)


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_backward_matches_finite_differences(seed, gated):
    eps = 1e-6
    L, x, dy = _layer(seed, gated=gated)
    G = _grads(L, x, dy, eps)
    rng = np.random.default_rng(100 + seed)
    h = 1e-6
    names = ["W_r", "b_r", "W_up", "W_down", "s", "W_s_up", "W_s_down"] + (["W_val"] if gated else [])
    for name in names + ["x"]:
        base = x if name == "x" else L[name]
        for _ in range(3):
            d = rng.standard_normal(base.shape)
            if name == "x":
                fp = _loss(L, x + h * d, dy, eps)
                fm = _loss(L, x - h * d, dy, eps)
                an = float(np.sum(G["dx"] * d))
            else:
                Lp, Lm = dict(L), dict(L)
                Lp[name], Lm[name] = base + h * d, base - h * d
                fp, fm = _loss(Lp, x, dy, eps), _loss(Lm, x, dy, eps)
                an = float(np.sum(G["d" + name] * d))
            fd = (fp - fm) / (2 * h)
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def _torch_layer(P, x, eps, gated):
    """The layer as a dense masked computation: every expert on every token,
    weighted by ReLU(z) (zero where inactive)."""
    z = x @ P["W_r"].T + P["b_r"]
    r = torch.relu(z)
    W_bar = P["W_up"].mean(dim=0)
    u = x @ W_bar.T                                        # [T, d_e]
    g = torch.einsum("ejd,td->tej", P["W_up"], x)          # [T, E, d_e]
    c = g - u[:, None, :]
    h = c / torch.sqrt((c * c).mean(dim=-1, keepdim=True) + eps)
    a = torch.nn.functional.silu(h)
    if gated:
        a = a * torch.einsum("ejd,td->tej", P["W_val"], x)
    v = torch.einsum("ekj,tej->tek", P["W_down"], a)       # [T, E, D]
    routed = ((P["s"] * r)[:, :, None] * v).sum(dim=1)
    shared = torch.nn.functional.silu(x @ P["W_s_up"].T) @ P["W_s_down"].T
    return shared + routed


@pytest.mark.parametrize("gated", [False, True])
def test_backward_matches_autograd_of_a_dense_formulation(gated):
    eps = 1e-6
    L, x, dy = _layer(7, T=5, D=12, E=6, d_e=8, d_s=6, gated=gated)
    G = _grads(L, x, dy, eps)
    P = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in L.items()}
    xt = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    y = _torch_layer(P, xt, eps, gated)
    (y * torch.tensor(dy)).sum().backward()
    for k in P:
        np.testing.assert_allclose(G["d" + k], P[k].grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=k)
    np.testing.assert_allclose(G["dx"], xt.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_extra_logit_gradient_reaches_the_router_where_active():
    """dz_extra adds to the router logits' gradient on the active set: the
    loss sum(dy * y) + sum(C * ReLU(z)) by finite differences."""
    eps = 1e-6
    L, x, dy = _layer(3)
    C = np.random.default_rng(5).standard_normal((x.shape[0], L["W_r"].shape[0]))

    def loss(LL, xx):
        z = xx @ LL["W_r"].T + LL["b_r"]
        return _loss(LL, xx, dy, eps) + float(np.sum(C * np.maximum(z, 0.0)))

    G = _grads(L, x, dy, eps, dz_extra=C)
    h = 1e-6
    d = np.random.default_rng(6).standard_normal(L["W_r"].shape)
    Lp, Lm = dict(L), dict(L)
    Lp["W_r"], Lm["W_r"] = L["W_r"] + h * d, L["W_r"] - h * d
    fd = (loss(Lp, x) - loss(Lm, x)) / (2 * h)
    assert abs(fd - float(np.sum(G["dW_r"] * d))) <= 1e-6 * max(1.0, abs(fd))
    dd = np.random.default_rng(7).standard_normal(x.shape)
    fd = (loss(L, x + h * dd) - loss(L, x - h * dd)) / (2 * h)
    assert abs(fd - float(np.sum(G["dx"] * dd))) <= 1e-6 * max(1.0, abs(fd))


def test_router_entropy_closed_forms():
    z = np.array([[1.0, 1.0, 1.0, -1.0],      # three equal active weights: log 3
                  [2.0, -0.5, -3.0, -1.0],    # one active expert: 0
                  [-1.0, -2.0, -0.1, -4.0],   # none: 0
                  [3.0, 1.0, -1.0, 0.0]])     # p = (3/4, 1/4); a zero score is inactive
    H, dH = O.router_entropy(z)
    H4 = -(0.75 * math.log(0.75) + 0.25 * math.log(0.25))
    assert H == pytest.approx((math.log(3) + 0.0 + 0.0 + H4) / 4, rel=1e-14)
    assert np.all(dH[:, 3] == 0.0) and np.all(dH[1] == 0.0) and np.all(dH[2] == 0.0)
    # equal weights are a stationary point of the entropy along the active set
    assert np.allclose(dH[0, :3], 0.0, atol=1e-15)


def test_router_entropy_gradient_matches_finite_differences():
    rng = np.random.default_rng(11)
    z = rng.standard_normal((6, 7))
    z[np.abs(z) < 0.1] += 0.3
    H, dH = O.router_entropy(z)
    h = 1e-7
    for _ in range(5):
        d = rng.standard_normal(z.shape)
        fd = (O.router_entropy(z + h * d)[0] - O.router_entropy(z - h * d)[0]) / (2 * h)
        assert abs(fd - float(np.sum(dH * d))) <= 1e-6 * max(1.0, abs(fd))


def test_sparsity_controller():
    assert O.sparsity_controller(1.0, 0.25, 0.2) == pytest.approx(1.002)
    assert O.sparsity_controller(1.0, 0.15, 0.2) == pytest.approx(1 / 1.002)
    assert O.sparsity_controller(0.7, 0.2, 0.2) == 0.7
    lam = 1.0
    for ratio in [0.3] * 100 + [0.1] * 40:
        lam = O.sparsity_controller(lam, ratio, 0.2)
    assert lam == pytest.approx(1.002 ** 60, rel=1e-12)
