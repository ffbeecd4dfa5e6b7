"""GPU parity of the training side (deco_moe_backward, deco_moe_router_entropy)
against the fp64 oracle (oracle/backward.py), through the C ABI.

Tolerance: the backward kernels compute in fp32 from the exactly stored
operands (no reduced-precision intermediates), so each gradient is held to
the forward pass's fp32 bar, max|err| <= 1e-4 * RMS of the oracle's gradient,
for bf16 storage too.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity_util import case, to_gpu, to_oracle
from synth import LayerShape, make_layer

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _dy(shape, seed):
    g = torch.Generator().manual_seed(seed)
    dy = torch.randn(shape.T, shape.D, generator=g)
    return dy.to(torch.float32 if shape.dtype == "f32" else torch.bfloat16)


def _check(grads, ref, what):
    assert set(grads) == set(ref), (sorted(grads), sorted(ref))
    for k, v in ref.items():
        got = grads[k].double().cpu().numpy()
        assert got.shape == v.shape, (k, got.shape, v.shape)
        rms = float(np.sqrt(np.mean(v * v))) if v.size else 0.0
        err = float(np.abs(got - v).max()) if v.size else 0.0
        assert err <= TOL * rms + 1e-30, f"{what} {k}: max err {err:.3e} vs rms {rms:.3e}"


def _run(lib, shape, L, dy, eps, dz_extra=None, residual=False):
    G = to_gpu(L, lib)
    dz_dev = None if dz_extra is None else torch.tensor(dz_extra, dtype=torch.float32).cuda()
    grads = lib.backward(G["x"], G, dy.cuda(), dz_extra=dz_dev, eps=eps, residual=residual)
    torch.cuda.synchronize()
    L64 = to_oracle(L, shape.dtype)
    ref = O.layer_backward_tokens(O.to_f64(L["x"]), L64, O.to_f64(dy), eps, dz_extra)
    if residual:
        ref["dx"] = ref["dx"] + O.to_f64(dy)
    return grads, ref, G


@pytest.mark.parametrize("name", ["tiny_f32"])
def test_backward_parity_fp32(lib, name):
    shape, L = case(name)
    grads, ref, _ = _run(lib, shape, L, _dy(shape, 5), shape.eps)
    _check(grads, ref, name)


@pytest.mark.parametrize("gated", [False, True])
def test_backward_parity_bf16(lib, gated):
    shape = LayerShape(16, 512, 16, 128, 256, "bf16")
    L = make_layer(shape, 41, gated=gated)
    grads, ref, _ = _run(lib, shape, L, _dy(shape, 6), shape.eps)
    _check(grads, ref, f"bf16 gated={gated}")


def test_backward_with_logit_gradient_and_residual(lib):
    shape = LayerShape(24, 256, 8, 64, 128, "bf16")
    L = make_layer(shape, 43)
    dz = np.random.default_rng(3).standard_normal((shape.T, shape.E)).astype(np.float32).astype(np.float64)
    grads, ref, _ = _run(lib, shape, L, _dy(shape, 7), shape.eps, dz_extra=dz, residual=True)
    _check(grads, ref, "dz_extra + residual")


def test_backward_is_deterministic(lib):
    shape = LayerShape(16, 512, 16, 128, 256, "bf16")
    L = make_layer(shape, 45)
    G = to_gpu(L, lib)
    dy = _dy(shape, 8).cuda()
    a = lib.backward(G["x"], G, dy, eps=shape.eps)
    b = lib.backward(G["x"], G, dy, eps=shape.eps)
    torch.cuda.synchronize()
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_router_entropy_matches_oracle(lib):
    shape, L = case("edge_decode_t16")
    G = to_gpu(L, lib)
    res = lib.routing(G["x"], G)
    lam = 0.37
    H, dz = lib.router_entropy(res["r"], res["active"], lam)
    torch.cuda.synchronize()
    z = O.to_f64(L["x"]) @ O.to_f64(L["W_r"]).T + O.to_f64(L["b_r"])
    # the oracle on the same active set (the GPU's decisions are exact)
    act = res["active"].cpu().numpy().astype(bool)
    assert np.array_equal(act, z > 0)
    Hm, dH = O.router_entropy(np.where(act, z, -1.0))
    Hg = H.cpu().numpy().astype(np.float64)
    assert abs(Hg[-1] - Hm) <= 1e-5 * max(1.0, Hm)
    np.testing.assert_allclose(dz.cpu().numpy(), lam * dH, rtol=1e-4, atol=1e-6 * np.abs(lam * dH).max())
