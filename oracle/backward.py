"""DECO MoE FFN layer, training side: backward pass, router-entropy
regulariser and adaptive sparsity controller, in fp64 on the CPU (test
infrastructure only).

Sources.  The layer is the one of deco.py ([arXiv] "DECO: Sparse
Mixture-of-Experts with Dense-Comparable Performance on End-Side Devices", §1
and §2; [press] part 2).  The training objective: [press] part 3, adaptive
sparsity regularisation -- a penalty on the router entropy whose coefficient
is multiplied by a small factor (for example 1.002) after every training
iteration in which the activation ratio is above its target and divided by it
when the ratio is below; [arXiv] §2, "Auxiliary training objective" -- an
auto-scaling coefficient as in ReMoE, with the L1 norm replaced by the router
entropy for numerical stability.

Readings where the pages are silent (the paper's §3.3 equations are not on
the pages):
- The gradient of ReLU routing: r_e = z_e on the active set (z_e > 0) and 0
  elsewhere, so dr_e/dz_e = 1 where active and 0 otherwise; a score of exactly
  0 is inactive, with derivative 0.
- The mean up-projection is the function W_bar = (1/E) sum_e W_up[e]: its
  gradient reaches every W_up[e] as dW_bar / E.  The forward pass uses the
  stored W_bar (the rounded mean); the rounding is not differentiated.
- The router entropy of token t is the Shannon entropy of its active routing
  weights normalised to sum to one, p_e = r_e / sum_j r_j over the active e,
  H_t = -sum_e p_e log p_e (0 for a token with no active expert); the
  regulariser is the mean over tokens.  It is higher when more experts share a
  token's weight, as the pages describe.
- The controller compares the iteration's activation ratio with the target
  and leaves the coefficient unchanged when they are equal.

Parity unpinned by the pages: the entropy's form (the pages name the router
entropy but print no formula).  The pins (tests/test_oracle_backward.py) hold
the code to these readings: finite differences, an autograd formulation and
closed forms.

Loops are per token and per active expert in ascending order, as in deco.py.
"""
from __future__ import annotations

import math

import numpy as np

from .deco import router_logits, silu


def sigmoid(h) -> np.ndarray:
    h = np.asarray(h, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-h))


def silu_grad(h) -> np.ndarray:
    """d/dh SiLU(h) = sigma(h) (1 + h (1 - sigma(h)))."""
    s = sigmoid(h)
    return s * (1.0 + np.asarray(h, dtype=np.float64) * (1.0 - s))


def norm_silu_backward(c: np.ndarray, dh: np.ndarray, eps: float) -> np.ndarray:
    """dc for h = c / sqrt(mean(c^2) + eps): with rho = (mean(c^2) + eps)^-1/2,
    dh_i/dc_j = rho delta_ij - rho^3 c_i c_j / d, so
    dc = rho dh - (rho^3 / d) (dh . c) c."""
    d = c.shape[0]
    rho = 1.0 / math.sqrt(float(np.mean(c * c)) + eps)
    return rho * dh - (rho ** 3 / d) * float(dh @ c) * c


def layer_backward_tokens(x: np.ndarray, L: dict, dy: np.ndarray, eps: float, dz_extra=None) -> dict:
    """Gradients of the loss through one DECO MoE layer, given dy = dLoss/dy.

    x [T,D], dy [T,D] and the fp64 weights of deco.layer_forward_tokens.
    dz_extra [T,E], optional: a gradient on the router logits from another
    term of the loss (the entropy regulariser), added where the expert is
    active.  Returns fp64 arrays dx [T,D], dW_r, db_r, dW_up (including the
    mean up-projection's share), dW_down, ds, dW_s_up, dW_s_down, and dW_val
    for gated experts.
    """
    T, D = x.shape
    E, d_e, _ = L["W_up"].shape
    W_val = L.get("W_val")
    g = {k: np.zeros_like(L[k]) for k in ("W_r", "b_r", "W_up", "W_down", "s", "W_s_up", "W_s_down")}
    if W_val is not None:
        g["W_val"] = np.zeros_like(W_val)
    dW_bar = np.zeros_like(L["W_bar_up"])
    dx = np.zeros_like(x)
    for t in range(T):
        x_t, dy_t = x[t], dy[t]
        z = router_logits(x_t, L["W_r"], L["b_r"])
        u = L["W_bar_up"] @ x_t
        # shared expert: y += W_s_down SiLU(hs), hs = W_s_up x
        hs = L["W_s_up"] @ x_t
        g["W_s_down"] += np.outer(dy_t, silu(hs))
        dhs = (L["W_s_down"].T @ dy_t) * silu_grad(hs)
        g["W_s_up"] += np.outer(dhs, x_t)
        dx[t] += L["W_s_up"].T @ dhs
        du = np.zeros(d_e)
        for e in range(E):
            if not z[e] > 0.0:
                continue
            # forward of the pair
            c = L["W_up"][e] @ x_t - u
            rho = 1.0 / math.sqrt(float(np.mean(c * c)) + eps)
            h = rho * c
            act = silu(h)
            q = None if W_val is None else W_val[e] @ x_t
            a = act if q is None else act * q
            v = L["W_down"][e] @ a
            # y += s_e r_e v
            w = float(dy_t @ v)
            g["s"][e] += z[e] * w
            dz = L["s"][e] * w + (0.0 if dz_extra is None else dz_extra[t, e])
            dv = (L["s"][e] * z[e]) * dy_t
            g["W_down"][e] += np.outer(dv, a)
            da = L["W_down"][e].T @ dv
            if q is None:
                dh = da * silu_grad(h)
            else:
                dh = da * q * silu_grad(h)
                dq = da * act
                g["W_val"][e] += np.outer(dq, x_t)
                dx[t] += W_val[e].T @ dq
            dc = norm_silu_backward(c, dh, eps)
            g["W_up"][e] += np.outer(dc, x_t)
            dx[t] += L["W_up"][e].T @ dc
            du -= dc
            # router: z = W_r[e] x + b_r[e]
            g["W_r"][e] += dz * x_t
            g["b_r"][e] += dz
            dx[t] += dz * L["W_r"][e]
        dW_bar += np.outer(du, x_t)
        dx[t] += L["W_bar_up"].T @ du
    g["W_up"] += dW_bar[None, :, :] / E
    out = {"dx": dx}
    out.update({"d" + k: v for k, v in g.items()})
    return out


def router_entropy(z: np.ndarray):
    """Mean router entropy over tokens and its gradient on the logits.

    For token t, over its active experts (z > 0): r = z, R = sum r,
    p = r / R, H_t = -sum p log p (0 with no active expert).  Returns
    (mean_t H_t, dH [T,E]) with dH = d(mean_t H_t)/dz:
    dH_t/dr_e = -(log p_e + H_t) / R on the active set, 0 elsewhere.
    """
    T, E = z.shape
    H = np.zeros(T)
    dH = np.zeros((T, E))
    for t in range(T):
        act = [e for e in range(E) if z[t, e] > 0.0]
        if not act:
            continue
        r = np.array([z[t, e] for e in act])
        R = float(r.sum())
        p = r / R
        H[t] = -float(np.sum(p * np.log(p)))
        for i, e in enumerate(act):
            dH[t, e] = -(math.log(p[i]) + H[t]) / R / T
    return float(H.mean()), dH


def sparsity_controller(lam: float, ratio: float, target: float, factor: float = 1.002) -> float:
    """One step of the adaptive coefficient: x factor above the target
    activation ratio, / factor below it, unchanged at it."""
    if ratio > target:
        return lam * factor
    if ratio < target:
        return lam / factor
    return lam
