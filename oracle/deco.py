"""DECO MoE FFN layer, fp64 CPU oracle (test infrastructure only).

See the package docstring for the sources ([arXiv], [press]) and the readings.
Every function takes numpy float64 arrays that hold the stored values exactly
(bf16 / fp32 widened to fp64) and computes in fp64.  Loops are per token and
per active expert, in ascending expert order, so the code can be checked
against the method's description step by step.
"""
from __future__ import annotations

import math

import numpy as np


# --------------------------------------------------------------------------
# storage helpers

def to_f64(t) -> np.ndarray:
    """A torch tensor (any float dtype) or array as an fp64 numpy array."""
    if hasattr(t, "detach"):
        import torch
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def round_bf16(a) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 value, ties to even.

    bfloat16 has fp32's exponent range and 8 significant bits.  A finite value
    with frexp exponent e (|a| in [2^(e-1), 2^e)) has spacing 2^(e-8) when it
    is normal (e-1 >= -126) and 2^-133 below that (subnormals), so the value
    is rint(a / q) * q with q that spacing; rint rounds halves to even.
    Results of magnitude 2^128 or more overflow to infinity.
    """
    a = np.asarray(a, dtype=np.float64)
    out = np.array(a, copy=True)
    fin = np.isfinite(a) & (a != 0.0)
    _, e = np.frexp(a[fin])
    q = np.ldexp(1.0, np.maximum(e, -125) - 8)
    r = np.rint(a[fin] / q) * q
    r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, r), r)
    out[fin] = r
    return out


def round_storage(a, dtype: str) -> np.ndarray:
    """Round fp64 values once to the storage dtype ("f32" or "bf16")."""
    if dtype == "f32":
        return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        return round_bf16(a)
    raise ValueError(dtype)


def silu(h) -> np.ndarray:
    """SiLU(h) = h * sigmoid(h) = h / (1 + exp(-h))."""
    h = np.asarray(h, dtype=np.float64)
    with np.errstate(over="ignore"):
        return h / (1.0 + np.exp(-h))


# --------------------------------------------------------------------------
# router: [press] part 2 router paragraph; [arXiv] §1, §2 "Router design"

def router_logits(x_t: np.ndarray, W_r: np.ndarray, b_r: np.ndarray) -> np.ndarray:
    """Router logits of one token, each the correctly rounded exact sum.

    z_e = b_r[e] + sum_k x_t[k] * W_r[e, k].  The products are exact in fp64
    for bf16 or fp32 operands and math.fsum rounds the exact sum once, so the
    sign of z_e is exact.
    """
    E = W_r.shape[0]
    z = np.empty(E)
    for e in range(E):
        products = (x_t * W_r[e]).tolist()
        z[e] = math.fsum(products + [float(b_r[e])])
    return z


def route(x: np.ndarray, W_r: np.ndarray, b_r: np.ndarray):
    """ReLU routing for a batch: returns (z [T,E], active [T,E] bool, r [T,E]).

    Expert e is active for token t iff z[t,e] > 0 -- a zero or negative score
    is ignored -- and r = ReLU(z) is the raw routing weight.
    """
    T = x.shape[0]
    z = np.stack([router_logits(x[t], W_r, b_r) for t in range(T)]) if T else \
        np.zeros((0, W_r.shape[0]))
    active = z > 0.0
    r = np.where(active, z, 0.0)
    return z, active, r


def exact_logit(x_t: np.ndarray, w: np.ndarray, b: float):
    """The exact rational value of b + sum_k x_t[k] w[k] (a Fraction)."""
    from fractions import Fraction
    total = Fraction(float(b))
    for xv, wv in zip(x_t.tolist(), w.tolist()):
        total += Fraction(xv) * Fraction(wv)
    return total


def topk_route(x: np.ndarray, W_r: np.ndarray, b_r: np.ndarray, k: int):
    """TopK routing baseline at a fixed k: the k largest logits per token
    (ties to the lower expert index), weights ReLU(z) of the chosen ones.

    The comparison point of [arXiv] §5 ("TopK ... conventional TopK" at the
    same average activation ratio).  Returns (z, active, r) like `route`.

    Ranking is by the exact logit.  The correctly rounded sums of
    `router_logits` keep the order of distinct exact values except that two
    of them may round to the same fp64 number; such ties are settled on the
    exact rational values, and only exactly equal logits go to the lower
    index.
    """
    from functools import cmp_to_key
    T = x.shape[0]
    E = W_r.shape[0]
    z = np.stack([router_logits(x[t], W_r, b_r) for t in range(T)]) if T else \
        np.zeros((0, E))
    active = np.zeros((T, E), dtype=bool)
    for t in range(T):
        exact = {}

        def value(e):
            if e not in exact:
                exact[e] = exact_logit(x[t], W_r[e], b_r[e])
            return exact[e]

        def cmp(e, f):   # negative: e ranks above f
            if z[t, e] != z[t, f]:
                return -1 if z[t, e] > z[t, f] else 1
            ve, vf = value(e), value(f)
            if ve != vf:
                return -1 if ve > vf else 1
            return -1 if e < f else (1 if e > f else 0)

        order = sorted(range(E), key=cmp_to_key(cmp))
        for e in order[:k]:
            active[t, e] = True
    r = np.where(active, np.maximum(z, 0.0), 0.0)
    return z, active, r


def routing_tables(active: np.ndarray):
    """Token -> expert tables of a routing decision.

    counts[e]   number of tokens routed to e
    offsets[e]  exclusive prefix sum of counts (offsets[E] = P, the pair count)
    perm[p]     token of pair p, pairs ordered by expert then token (ascending)
    n_tok[t]    number of experts token t activates
    """
    T, E = active.shape
    counts = active.sum(axis=0).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    perm = []
    for e in range(E):
        for t in range(T):
            if active[t, e]:
                perm.append(t)
    n_tok = active.sum(axis=1).astype(np.int64)
    return counts, offsets, np.asarray(perm, dtype=np.int64), n_tok


# --------------------------------------------------------------------------
# experts: [press] NormSiLU paragraph; [arXiv] §1, §2 "Expert design"

def mean_up(W_up: np.ndarray, dtype: str) -> np.ndarray:
    """The precomputed mean up-projection W_bar_up = (1/E) sum_e W_up[e].

    Summed in fp64 over e ascending, divided by E in fp64, rounded once to the
    storage dtype (the stored W_bar_up the layer then consumes).
    """
    E = W_up.shape[0]
    acc = np.zeros(W_up.shape[1:], dtype=np.float64)
    for e in range(E):
        acc = acc + W_up[e]
    return round_storage(acc / float(E), dtype)


def norm_silu(g: np.ndarray, u: np.ndarray, eps: float):
    """NormSiLU of one (token, expert) pair: returns (c, h, a).

    c = g - u                         inter-expert mean normalisation
    h = c / sqrt(mean(c^2) + eps)     intra-expert RMS normalisation (no gain)
    a = SiLU(h)
    """
    c = g - u
    ms = float(np.mean(c * c))
    h = c / math.sqrt(ms + eps)
    return c, h, silu(h)


def expert_output(x_t, W_up_e, W_down_e, u_t, eps, W_val_e=None):
    """Routed expert e on token t: v = W_down[e] NormSiLU(W_up[e] x_t).

    Gated variant ("DECO (gated)", the ablation of [press] part 2 and [arXiv]
    §2 "Expert design"), when W_val_e is given: the NormSiLU output is
    multiplied element-wise by a linear value branch,
    v = W_down[e] (NormSiLU(W_up[e] x_t) * (W_val[e] x_t)).
    """
    g = W_up_e @ x_t
    _, _, a = norm_silu(g, u_t, eps)
    if W_val_e is not None:
        a = a * (W_val_e @ x_t)
    return W_down_e @ a


def shared_expert(x_t, W_s_up, W_s_down):
    """Always-on shared expert: S = W_s_down SiLU(W_s_up x_t)."""
    return W_s_down @ silu(W_s_up @ x_t)


# --------------------------------------------------------------------------
# the layer

def layer_forward_tokens(x: np.ndarray, L: dict, eps: float, tokens=None):
    """Forward pass of one DECO MoE layer for the listed tokens (default all).

    L holds fp64 arrays W_r [E,D], b_r [E], W_up [E,d_e,D], W_bar_up [d_e,D],
    W_down [E,D,d_e], s [E], W_s_up [d_s,D], W_s_down [D,d_s], and for the
    gated variant W_val [E,d_e,D].
    Returns (y [n,D] fp64 before rounding, z [n,E], active [n,E]).
    """
    if tokens is None:
        tokens = range(x.shape[0])
    tokens = list(tokens)
    D = x.shape[1]
    E = L["W_r"].shape[0]
    y = np.zeros((len(tokens), D))
    zs = np.zeros((len(tokens), E))
    acts = np.zeros((len(tokens), E), dtype=bool)
    for i, t in enumerate(tokens):
        x_t = x[t]
        z = router_logits(x_t, L["W_r"], L["b_r"])
        u = L["W_bar_up"] @ x_t
        routed = np.zeros(D)
        W_val = L.get("W_val")
        for e in range(E):
            if z[e] > 0.0:
                v = expert_output(x_t, L["W_up"][e], L["W_down"][e], u, eps,
                                  None if W_val is None else W_val[e])
                routed = routed + (L["s"][e] * z[e]) * v
        y[i] = shared_expert(x_t, L["W_s_up"], L["W_s_down"]) + routed
        zs[i] = z
        acts[i] = z > 0.0
    return y, zs, acts


def layer_forward(x: np.ndarray, L: dict, eps: float) -> np.ndarray:
    """y for every token of x (fp64, unrounded)."""
    return layer_forward_tokens(x, L, eps)[0]


def stack_forward(x: np.ndarray, layers: list, eps: float, dtype: str, tokens=None):
    """Stacked layers with residual adds: x_{l+1} = round(x_l + MoE_l(x_l)).

    Each layer's output is rounded once to the storage dtype, as the layer
    writes it.  Tokens are independent, so a token subset is exact.
    """
    if tokens is not None:
        x = x[list(tokens)]
    for L in layers:
        x = round_storage(x + layer_forward(x, L, eps), dtype)
    return x


def dense_ffn(x: np.ndarray, W1: np.ndarray, W2: np.ndarray) -> np.ndarray:
    """Equal-parameter dense non-gated FFN baseline: y = W2 SiLU(W1 x).

    The "Dense" comparison of [arXiv] §5, with the same non-gated SiLU MLP
    form as the shared expert and d_ff = d_s + E d_e.
    """
    out = np.zeros((x.shape[0], W2.shape[0]))
    for t in range(x.shape[0]):
        out[t] = W2 @ silu(W1 @ x[t])
    return out
