"""Pins of the CPU oracle against facts the DECO pages and mathematics fix.

None of these tests needs a GPU.  Each pin is chosen so that a plausible slip
in the oracle (a dropped term, a wrong sign or index, sum instead of mean,
scaling in the wrong place, a naive rounding) fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from synth import LayerShape, make_layer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _layer64(shape, seed=0, **kw):
    L = make_layer(shape, seed, **kw)
    L64 = {k: O.to_f64(v) for k, v in L.items()}
    L64["W_bar_up"] = O.mean_up(L64["W_up"], shape.dtype)
    return L64


# --------------------------------------------------------------------------
# storage rounding

def test_round_bf16_matches_torch_single_rounding():
    # fp32 inputs: torch's fp32 -> bf16 cast is one RNE rounding, as is ours.
    g = torch.Generator().manual_seed(5)
    vals = torch.cat([
        torch.randn(20000, generator=g),
        torch.randn(2000, generator=g) * 1e-38,          # subnormal range
        torch.randn(2000, generator=g) * 3e38,           # overflow edge
        torch.tensor([0.0, -0.0, 1.0, -1.0, 2.0 ** -133, 3.3895e38]),
    ]).to(torch.float32)
    ref = vals.to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(vals.to(torch.float64).numpy())
    np.testing.assert_array_equal(got, ref)


def test_round_bf16_ties_to_even():
    u = 2.0 ** -7                      # spacing of bf16 on [1, 2)
    got = O.round_bf16(np.array([1 + u / 2, 1 + 3 * u / 2, -(1 + u / 2), 1 + u / 2 + 2.0 ** -30]))
    np.testing.assert_array_equal(got, [1.0, 1 + 2 * u, -1.0, 1 + u])


# --------------------------------------------------------------------------
# SiLU closed forms

def test_silu_closed_forms():
    assert O.silu(0.0) == 0.0
    # sigmoid(ln 3) = 3/4
    assert O.silu(math.log(3.0)) == pytest.approx(0.75 * math.log(3.0), rel=1e-15)
    h = np.linspace(-30, 30, 601)
    # SiLU(h) - SiLU(-h) = h  (sigmoid(h) + sigmoid(-h) = 1)
    np.testing.assert_allclose(O.silu(h) - O.silu(-h), h, rtol=1e-14, atol=1e-14)
    assert O.silu(60.0) == pytest.approx(60.0, rel=1e-15)
    assert O.silu(-60.0) == pytest.approx(-60.0 * math.exp(-60.0), rel=1e-12)
    assert O.silu(-800.0) == 0.0        # exp overflow handled, limit 0
    # library routine
    t = torch.linspace(-12, 12, 241, dtype=torch.float64)
    np.testing.assert_allclose(O.silu(t.numpy()), torch.nn.functional.silu(t).numpy(),
                               rtol=1e-15, atol=1e-300)


# --------------------------------------------------------------------------
# router: exact sign, strict > 0

def test_router_sign_is_exact_where_naive_sum_fails():
    # products in order 1, 2^-100, -1: a left-to-right fp64 sum gives 0,
    # the exact value is 2^-100 > 0 (active); the mirrored case is inactive.
    x = np.array([[1.0, 2.0 ** -50, 1.0]])
    W = np.array([[1.0, 2.0 ** -50, -1.0],       # +2^-100
                  [1.0, -(2.0 ** -50), -1.0],    # -2^-100
                  [1.0, 0.0, -1.0]])             # exactly 0 -> ignored
    z, active, r = O.route(x, W, np.zeros(3))
    assert active.tolist() == [[True, False, False]]
    assert z[0, 0] == 2.0 ** -100 and z[0, 1] == -(2.0 ** -100) and z[0, 2] == 0.0
    assert r[0].tolist() == [2.0 ** -100, 0.0, 0.0]


def test_router_matches_exact_rational_arithmetic():
    # bf16 operands, bias chosen so that many logits are exactly zero or tiny.
    g = torch.Generator().manual_seed(11)
    T, E, D = 12, 16, 24
    x = torch.randn(T, D, generator=g).to(torch.bfloat16).double().numpy()
    W = (torch.randn(E, D, generator=g) / 5).to(torch.bfloat16).double().numpy()
    b = np.zeros(E)
    # make expert e's logit for token e%T exactly zero (bias = -exact dot, fp32-exact)
    for e in range(E):
        exact = sum(Fraction(float(a)) * Fraction(float(w)) for a, w in zip(x[e % T], W[e]))
        b[e] = float(np.float32(-float(exact)))
    z, active, _ = O.route(x, W, b)
    for t in range(T):
        for e in range(E):
            exact = Fraction(float(b[e])) + sum(
                Fraction(float(a)) * Fraction(float(w)) for a, w in zip(x[t], W[e]))
            assert active[t, e] == (exact > 0)
            assert z[t, e] == float(exact)          # correctly rounded
    assert (~active).sum() > 0 and active.sum() > 0


def test_routing_tables_against_lexicographic_nonzero():
    rng = np.random.default_rng(3)
    for T, E in [(1, 4), (7, 8), (50, 64), (0, 5)]:
        active = rng.random((T, E)) < 0.3
        counts, offsets, perm, n_tok = O.routing_tables(active)
        e_idx, t_idx = np.nonzero(active.T)        # sorted by e, then t
        np.testing.assert_array_equal(perm, t_idx)
        np.testing.assert_array_equal(counts, np.bincount(e_idx, minlength=E))
        assert offsets[0] == 0 and offsets[-1] == active.sum()
        np.testing.assert_array_equal(np.diff(offsets), counts)
        np.testing.assert_array_equal(n_tok, active.sum(axis=1))


# --------------------------------------------------------------------------
# NormSiLU pins

def test_centred_activations_sum_to_zero_over_experts():
    # With the exact (unrounded) fp64 mean, sum_e (g_e - u) = 0 for every token.
    shape = LayerShape(8, 64, 6, 32, 16, "bf16")
    L = {k: O.to_f64(v) for k, v in make_layer(shape, 4).items()}
    Wbar = L["W_up"].mean(axis=0)
    for t in range(shape.T):
        u = Wbar @ L["x"][t]
        cs = np.stack([O.norm_silu(L["W_up"][e] @ L["x"][t], u, 1e-6)[0]
                       for e in range(shape.E)])
        scale = np.abs(cs).sum(axis=0).max()
        assert np.abs(cs.sum(axis=0)).max() <= 1e-13 * scale


def test_rms_normalised_activation_has_unit_rms():
    rng = np.random.default_rng(1)
    for eps in [0.0, 1e-6, 0.5]:
        g = rng.normal(size=256) * 3.0
        u = rng.normal(size=256)
        c, h, a = O.norm_silu(g, u, eps)
        ms = np.mean((g - u) ** 2)
        assert np.sqrt(np.mean(h * h)) == pytest.approx(math.sqrt(ms / (ms + eps)), rel=1e-14)
        np.testing.assert_allclose(c, g - u, rtol=0, atol=0)
        np.testing.assert_allclose(a, O.silu(h), rtol=0, atol=0)


def test_identical_experts_reduce_to_shared_expert():
    # all W_up[e] equal => mean equals each => c = 0 => h = 0 => SiLU = 0
    shape = LayerShape(6, 32, 4, 16, 8, "f32")
    L = _layer64(shape, ratio=0.6)
    L["W_up"][:] = L["W_up"][0]
    L["W_bar_up"] = O.mean_up(L["W_up"], "f32")
    y, _, act = O.layer_forward_tokens(L["x"], L, 1e-6)
    assert act.sum() > 0
    for t in range(shape.T):
        np.testing.assert_array_equal(y[t], O.shared_expert(L["x"][t], L["W_s_up"], L["W_s_down"]))


def test_single_expert_layer_is_shared_only():
    shape = LayerShape(5, 32, 1, 16, 8, "f32")
    L = _layer64(shape, ratio=1.0)
    y, _, act = O.layer_forward_tokens(L["x"], L, 1e-6)
    assert act.all()
    S = np.stack([O.shared_expert(L["x"][t], L["W_s_up"], L["W_s_down"]) for t in range(5)])
    np.testing.assert_array_equal(y, S)


# --------------------------------------------------------------------------
# whole-layer pins

def _shared_torch(x, L):
    X = torch.from_numpy(x)
    return (torch.nn.functional.silu(X @ torch.from_numpy(L["W_s_up"]).T)
            @ torch.from_numpy(L["W_s_down"]).T).numpy()


def test_zero_expert_tokens_get_only_the_shared_expert():
    shape = LayerShape(10, 48, 8, 16, 24, "bf16")
    L = _layer64(shape)
    L["b_r"][:] = -100.0                       # every logit negative
    y, _, act = O.layer_forward_tokens(L["x"], L, 1e-6)
    assert not act.any()
    np.testing.assert_allclose(y, _shared_torch(L["x"], L), rtol=1e-13, atol=1e-13)


def _dense_masked(L, eps):
    """Every expert on every token, each weighted by ReLU(router logit)."""
    x = L["x"]
    Z = np.stack([O.router_logits(x[t], L["W_r"], L["b_r"]) for t in range(x.shape[0])])
    X = torch.from_numpy(x)
    G = torch.einsum("edk,tk->ted", torch.from_numpy(L["W_up"]), X)
    U = X @ torch.from_numpy(L["W_bar_up"]).T
    C = G - U[:, None, :]
    H = C / torch.sqrt((C * C).mean(dim=-1, keepdim=True) + eps)
    A = torch.nn.functional.silu(H)
    V = torch.einsum("ekd,ted->tek", torch.from_numpy(L["W_down"]), A)
    w = torch.from_numpy(L["s"])[None, :] * torch.relu(torch.from_numpy(Z))
    return _shared_torch(x, L) + (w[:, :, None] * V).sum(dim=1).numpy()


@pytest.mark.parametrize("dtype,ratio", [("f32", 0.2), ("bf16", 0.2), ("bf16", 0.6), ("f32", 1.0)])
def test_sparse_equals_dense_evaluation_masked_by_relu(dtype, ratio):
    shape = LayerShape(24, 64, 8, 32, 16, dtype)
    L = _layer64(shape, seed=7, ratio=ratio)
    y, _, act = O.layer_forward_tokens(L["x"], L, 1e-6)
    if ratio == 1.0:
        assert act.all()
    ref = _dense_masked(L, 1e-6)
    scale = np.sqrt(np.mean(ref * ref))
    assert np.abs(y - ref).max() <= 1e-12 * scale


def test_routed_part_is_linear_in_router_scale():
    # Scaling W_r and b_r by 2 (exact) keeps the active set and doubles r.
    shape = LayerShape(16, 64, 8, 32, 16, "f32")
    L = _layer64(shape, seed=2)
    y1, _, a1 = O.layer_forward_tokens(L["x"], L, 1e-6)
    L2 = dict(L, W_r=2 * L["W_r"], b_r=2 * L["b_r"])
    y2, _, a2 = O.layer_forward_tokens(L["x"], L2, 1e-6)
    S = _shared_torch(L["x"], L)
    assert (a1 == a2).all() and a1.any()
    np.testing.assert_allclose(y2 - S, 2 * (y1 - S), rtol=1e-12, atol=1e-12)


def test_expert_scale_multiplies_only_its_own_term():
    shape = LayerShape(16, 64, 8, 32, 16, "f32")
    L = _layer64(shape, seed=9, ratio=0.5)
    e = 3
    ys = []
    for f in (0.0, 1.0, 2.0):
        s = L["s"].copy()
        s[e] *= f
        ys.append(O.layer_forward_tokens(L["x"], dict(L, s=s), 1e-6)[0])
    _, act = O.route(L["x"], L["W_r"], L["b_r"])[:2]
    assert act[:, e].any() and (~act[:, e]).any()
    np.testing.assert_allclose(ys[2] - ys[1], ys[1] - ys[0], rtol=1e-12, atol=1e-12)
    # tokens that do not route to e are unchanged
    np.testing.assert_array_equal(ys[0][~act[:, e]], ys[2][~act[:, e]])


def test_expert_permutation_invariance():
    shape = LayerShape(12, 64, 8, 32, 16, "bf16")
    L = _layer64(shape, seed=5, ratio=0.5)
    y = O.layer_forward(L["x"], L, 1e-6)
    p = np.array([5, 2, 7, 0, 1, 6, 3, 4])
    Lp = dict(L, W_r=L["W_r"][p], b_r=L["b_r"][p], W_up=L["W_up"][p],
              W_down=L["W_down"][p], s=L["s"][p])
    yp = O.layer_forward(L["x"], Lp, 1e-6)
    np.testing.assert_allclose(yp, y, rtol=1e-12, atol=1e-12)


def test_hand_worked_example():
    """A five-token worked example derived by hand (tests/golden)."""
    with open(os.path.join(GOLDEN, "hand_worked_example.json")) as f:
        ex = json.load(f)
    L = {k: np.array(v, dtype=np.float64) for k, v in ex["layer"].items()}
    x = np.array(ex["x"], dtype=np.float64)
    y, z, act = O.layer_forward_tokens(x, L, ex["eps"])
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))   # noqa: E731
    env = dict(sig=sig, sqrt=math.sqrt, silu=lambda v: v * sig(v))
    expect = [[eval(c, env) for c in row] for row in ex["expected_y"]]
    np.testing.assert_allclose(y, expect, rtol=1e-13, atol=1e-13)
    assert act.tolist() == ex["expected_active"]


def test_mean_up_against_library_mean():
    # values on a 2^-12 grid in [-1, 1]: the fp64 sum is exact and the mean is
    # fp32-exact, so torch's fp64 mean -> fp32 -> bf16 is a single rounding.
    g = torch.Generator().manual_seed(8)
    W = (torch.randint(-4096, 4097, (64, 8, 16), generator=g).double() / 4096).to(torch.bfloat16)
    ref = W.double().mean(dim=0).float().to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O.mean_up(O.to_f64(W), "bf16"), ref)
    W32 = (torch.randint(-4096, 4097, (7, 8, 16), generator=g).double() / 4096).float()
    ref32 = W32.double().mean(dim=0).float().double().numpy()
    np.testing.assert_array_equal(O.mean_up(O.to_f64(W32), "f32"), ref32)


def test_dense_ffn_against_library():
    g = torch.Generator().manual_seed(2)
    x = torch.randn(5, 32, generator=g, dtype=torch.float64)
    W1 = torch.randn(48, 32, generator=g, dtype=torch.float64)
    W2 = torch.randn(32, 48, generator=g, dtype=torch.float64)
    ref = (torch.nn.functional.silu(x @ W1.T) @ W2.T).numpy()
    np.testing.assert_allclose(O.dense_ffn(x.numpy(), W1.numpy(), W2.numpy()), ref,
                               rtol=1e-13, atol=1e-13)


def test_stack_residual_and_token_subset():
    shape = LayerShape(6, 32, 4, 16, 8, "bf16")
    layers = [_layer64(shape, seed=1, layer=l) for l in range(3)]
    x = layers[0]["x"]
    full = O.stack_forward(x, layers, 1e-6, "bf16")
    sub = O.stack_forward(x, layers, 1e-6, "bf16", tokens=[4, 1])
    np.testing.assert_array_equal(full[[4, 1]], sub)
    # a layer whose routed and shared outputs vanish is the identity
    Z = dict(layers[0], W_s_down=0 * layers[0]["W_s_down"], b_r=-100 + 0 * layers[0]["b_r"])
    np.testing.assert_array_equal(O.stack_forward(x, [Z], 1e-6, "bf16"), x)


def test_topk_route_picks_k_largest():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(9, 16))
    W = rng.normal(size=(8, 16))
    z, active, r = O.topk_route(x, W, np.zeros(8), 3)
    assert (active.sum(axis=1) == 3).all()
    for t in range(9):
        chosen = np.sort(np.nonzero(active[t])[0])
        np.testing.assert_array_equal(chosen, np.sort(np.argsort(-z[t], kind="stable")[:3]))


def test_topk_route_ranks_by_exact_value():
    # logits 1 and 1 + 2^-60 round to the same fp64 number; the exact order
    # decides (expert 1 is larger although its index is higher), and an exact
    # tie (experts 2 and 3) goes to the lower index
    x = np.zeros((1, 4))
    x[0, 0], x[0, 1] = 1.0, 2.0 ** -30
    W = np.zeros((4, 4))
    W[0, 0] = 1.0
    W[1, 0], W[1, 1] = 1.0, 2.0 ** -30
    W[2, 0], W[2, 2] = 0.5, 1.0
    W[3, 0], W[3, 3] = 0.5, 2.0
    x[0, 2], x[0, 3] = 0.25, 0.125
    b = np.zeros(4)
    z, act, r = O.topk_route(x, W, b, 1)
    assert z[0, 0] == z[0, 1] == 1.0                     # tie in fp64
    assert act[0].tolist() == [False, True, False, False]
    z, act, r = O.topk_route(x, W, b, 3)
    assert z[0, 2] == z[0, 3] == 0.75                    # an exact tie
    assert act[0].tolist() == [True, True, True, False]
    assert r[0, 1] == 1.0 and r[0, 3] == 0.0


def test_topk_route_matches_brute_force_exact_ranking():
    # small-integer operands: every logit is an exact integer, many tie
    from fractions import Fraction
    rng = np.random.default_rng(3)
    x = rng.integers(-3, 4, size=(12, 6)).astype(float)
    W = rng.integers(-2, 3, size=(9, 6)).astype(float)
    b = rng.integers(-2, 3, size=9).astype(float)
    for k in (1, 3, 9):
        _, act, r = O.topk_route(x, W, b, k)
        for t in range(12):
            vals = [sum(Fraction(a) * Fraction(c) for a, c in zip(x[t], W[e])) + Fraction(b[e])
                    for e in range(9)]
            want = sorted(range(9), key=lambda e: (-vals[e], e))[:k]
            assert sorted(np.nonzero(act[t])[0].tolist()) == sorted(want)
            for e in range(9):
                assert r[t, e] == (max(float(vals[e]), 0.0) if e in want else 0.0)


# --------------------------------------------------------------------------
# gated experts ("DECO (gated)"): a = NormSiLU(W_up x) * (W_val x)

def test_gated_value_of_one_is_the_non_gated_layer():
    # W_val[e] = ones (x) x_t / (x_t . x_t) makes every value feature of token t
    # equal to 1, so the gated layer on t equals the non-gated one
    shape = LayerShape(3, 32, 4, 16, 8, "f32")
    L = _layer64(shape, 3, ratio=0.6)
    t = 1
    x_t = L["x"][t]
    Lg = dict(L, W_val=np.stack([np.outer(np.ones(16), x_t) / float(x_t @ x_t)] * 4))
    y, _, act = O.layer_forward_tokens(L["x"], L, 1e-6, [t])
    yg, _, _ = O.layer_forward_tokens(L["x"], Lg, 1e-6, [t])
    assert act.any()
    np.testing.assert_allclose(yg, y, rtol=1e-12, atol=1e-12)


def test_gated_zero_value_leaves_only_the_shared_expert():
    shape = LayerShape(5, 32, 4, 16, 8, "f32")
    L = _layer64(shape, 4, ratio=0.6)
    Lg = dict(L, W_val=np.zeros((4, 16, 32)))
    y, _, act = O.layer_forward_tokens(L["x"], Lg, 1e-6)
    assert act.any()
    shared = np.stack([O.shared_expert(L["x"][t], L["W_s_up"], L["W_s_down"]) for t in range(5)])
    np.testing.assert_allclose(y, shared, rtol=0, atol=1e-14)


def test_gated_routed_part_is_linear_in_the_value_branch():
    shape = LayerShape(6, 32, 4, 16, 8, "f32")
    L = _layer64(shape, 5, ratio=0.5)
    W_val = np.random.default_rng(0).normal(size=(4, 16, 32)) / math.sqrt(32)
    shared = np.stack([O.shared_expert(L["x"][t], L["W_s_up"], L["W_s_down"]) for t in range(6)])
    y1, _, act = O.layer_forward_tokens(L["x"], dict(L, W_val=W_val), 1e-6)
    y3, _, _ = O.layer_forward_tokens(L["x"], dict(L, W_val=-3.0 * W_val), 1e-6)
    assert act.any()
    np.testing.assert_allclose(y3 - shared, -3.0 * (y1 - shared), rtol=1e-12, atol=1e-12)


def test_gated_sparse_equals_dense_evaluation_masked_by_relu():
    # every expert evaluated for every token, multiplied by ReLU(z): the
    # inactive ones drop out
    shape = LayerShape(7, 32, 5, 16, 8, "bf16")
    L = _layer64(shape, 6, ratio=0.4)
    L["W_val"] = O.to_f64(make_layer(shape, 6, gated=True)["W_val"])
    y = O.layer_forward(L["x"], L, 1e-6)
    for t in range(7):
        x_t = L["x"][t]
        z = O.router_logits(x_t, L["W_r"], L["b_r"])
        u = L["W_bar_up"] @ x_t
        ref = O.shared_expert(x_t, L["W_s_up"], L["W_s_down"])
        for e in range(5):
            c = L["W_up"][e] @ x_t - u
            h = c / math.sqrt(float(np.mean(c * c)) + 1e-6)
            a = h / (1.0 + np.exp(-h)) * (L["W_val"][e] @ x_t)
            ref = ref + L["s"][e] * max(z[e], 0.0) * (L["W_down"][e] @ a)
        np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-12)
