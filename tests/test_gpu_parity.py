"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Routing (active sets, counts, offsets, permutation,
per-token counts) must match bit for bit; outputs within max|err| <= 1e-4 *
RMS (fp32) or 2e-2 * RMS (bf16) of the oracle's fp64 output."""
import numpy as np
import pytest
import torch

import oracle as O
from parity_util import (case, check_close, oracle_forward, oracle_logits, to_gpu, to_oracle)
from synth import LayerShape, make_layer

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().numpy()


def _routing_check(deco, shape, L, G, z_exact=None, tokens=None):
    x64 = O.to_f64(L["x"])
    W_r64, b_r64 = O.to_f64(L["W_r"]), O.to_f64(L["b_r"])
    res = deco.routing(G["x"], G)
    torch.cuda.synchronize()
    act_gpu = _np(res["active"]).astype(bool)
    if tokens is None:
        z = oracle_logits(x64, W_r64, b_r64) if z_exact is None else z_exact
        act = z > 0
        np.testing.assert_array_equal(act_gpu, act)
        counts, offsets, perm, n_tok = O.routing_tables(act)
        np.testing.assert_array_equal(_np(res["counts"]), counts)
        np.testing.assert_array_equal(_np(res["offsets"]), offsets)
        np.testing.assert_array_equal(_np(res["perm"])[: offsets[-1]], perm)
        np.testing.assert_array_equal(_np(res["n_tok"])[: shape.T], n_tok)
        r = _np(res["r"])
        scale = np.abs(z).max()
        assert np.abs(r - np.where(act, z, 0.0)).max() <= 1e-5 * scale
        return act
    # full-size case: exact active sets on sampled tokens, table properties on all
    z = oracle_logits(x64[tokens], W_r64, b_r64)
    np.testing.assert_array_equal(act_gpu[tokens], z > 0)
    counts, offsets, perm, n_tok = O.routing_tables(act_gpu)
    np.testing.assert_array_equal(_np(res["counts"]), counts)
    np.testing.assert_array_equal(_np(res["offsets"]), offsets)
    np.testing.assert_array_equal(_np(res["perm"])[: offsets[-1]], perm)
    np.testing.assert_array_equal(_np(res["n_tok"])[: shape.T], n_tok)
    return act_gpu


# --------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny_f32", "edge_decode_t1", "large_t16"])
def test_mean_up_bit_exact(lib, name):
    shape, L = case(name)
    G = to_gpu(L, lib)
    ref = O.mean_up(O.to_f64(L["W_up"]), shape.dtype)
    np.testing.assert_array_equal(G["W_bar_up"].double().cpu().numpy(), ref)


@pytest.mark.parametrize("name", ["tiny_f32", "edge_decode_t1", "edge_decode_t4",
                                  "edge_decode_t16", "large_t16", "edge_prefill_t4096"])
def test_routing_bit_exact(lib, name):
    shape, L = case(name)
    G = to_gpu(L, lib)
    act = _routing_check(lib, shape, L, G)
    if name == "edge_prefill_t4096":
        assert not act[::64].any()          # planted zero-expert tokens
        ratio = act.mean()
        assert 0.1 < ratio < 0.3


def test_routing_full_size_large_layer(lib):
    shape, L = case("large_t16384")
    G = to_gpu(L, lib)
    toks = np.random.default_rng(0).choice(shape.T, 48, replace=False)
    # and the tokens whose logits come closest to zero, where a decision is
    # easiest to get wrong (picked from an fp64 product of the inputs)
    z64 = O.to_f64(L["x"]) @ O.to_f64(L["W_r"]).T + O.to_f64(L["b_r"])
    near = np.argsort(np.abs(z64).min(axis=1))[:16]
    _routing_check(lib, shape, L, G, tokens=np.unique(np.concatenate([toks, near])))


@pytest.mark.parametrize("name", ["tiny_f32", "edge_decode_t1", "edge_decode_t4",
                                  "edge_decode_t16", "large_t16"])
def test_forward_parity_full(lib, name):
    shape, L = case(name)
    G = to_gpu(L, lib)
    out = lib.forward(G["x"], G, eps=shape.eps)
    torch.cuda.synchronize()
    ref = oracle_forward(O.to_f64(L["x"]), to_oracle(L, shape.dtype), shape.eps, range(shape.T))
    check_close(out.double().cpu().numpy(), ref, shape.dtype, name)


@pytest.mark.parametrize("name,n", [("edge_prefill_t4096", 96), ("large_t16384", 24)])
def test_forward_parity_full_size_sampled(lib, name, n):
    shape, L = case(name)
    G = to_gpu(L, lib)
    out = lib.forward(G["x"], G, eps=shape.eps)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    toks = np.sort(np.concatenate([rng.choice(shape.T, n, replace=False), [0, 64, shape.T - 1]]))
    ref = oracle_forward(O.to_f64(L["x"]), to_oracle(L, shape.dtype), shape.eps, toks)
    check_close(out.double().cpu().numpy()[toks], ref, shape.dtype, name)


# --------------------------------------------------------------------------
# edge cases: ragged batches, degenerate routing, residual, dtypes

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,ratio", [(1, 0.2), (37, 0.2), (70, 0.05), (19, 1.0), (23, 0.0)])
def test_forward_edge_cases(lib, dtype, T, ratio):
    shape = LayerShape(T, 256, 8, 128, 192, dtype)
    L = make_layer(shape, 21, ratio=ratio if ratio > 0 else 0.2)
    if ratio == 0.0:
        L["b_r"] = torch.full_like(L["b_r"], -1e4)       # no token routes anywhere
    G = to_gpu(L, lib)
    out = lib.forward(G["x"], G, eps=shape.eps)
    torch.cuda.synchronize()
    L64 = to_oracle(L, dtype)
    ref, z, act = O.layer_forward_tokens(O.to_f64(L["x"]), L64, shape.eps)
    if ratio == 1.0:
        assert act.all()
    if ratio == 0.0:
        assert not act.any()
    check_close(out.double().cpu().numpy(), ref, dtype, f"T={T} ratio={ratio}")


def test_single_expert_and_wide_expert(lib):
    for shape in [LayerShape(9, 128, 1, 64, 64, "f32"), LayerShape(12, 192, 5, 512, 64, "bf16")]:
        L = make_layer(shape, 3, ratio=0.7)
        G = to_gpu(L, lib)
        out = lib.forward(G["x"], G, eps=shape.eps)
        torch.cuda.synchronize()
        ref = O.layer_forward(O.to_f64(L["x"]), to_oracle(L, shape.dtype), shape.eps)
        check_close(out.double().cpu().numpy(), ref, shape.dtype, str(shape))


def test_residual_stack_of_eight_layers(lib):
    """The 8-layer residual stack of the larger layer shape.

    Each layer is checked on the oracle's own input to that layer (its stack
    state, a bf16 tensor) at the stated tolerance.  Without a normalisation
    between layers the stack's activations grow ~3.6x per layer (x_{l+1} =
    x_l + layer(x_l), with the layer's output scaling with |x|), so small
    per-layer differences compound; the GPU's own 8-layer stack is therefore
    compared end to end in norm, not element-wise."""
    base = case("large_t16")[0]
    layers = [make_layer(base, 3, layer=l) for l in range(8)]
    x = O.to_f64(layers[0]["x"])
    xg = layers[0]["x"].cuda()
    for l, L in enumerate(layers):
        W = {k: v for k, v in L.items() if k != "x"}
        G = to_gpu(W, lib)
        L64 = to_oracle(W, "bf16")
        xin = torch.from_numpy(x).to(torch.bfloat16).cuda()      # exact: x is bf16-valued
        out = lib.forward(xin, G, eps=base.eps, residual=True)
        xg = lib.forward(xg, G, eps=base.eps, residual=True)
        torch.cuda.synchronize()
        ref = x + O.layer_forward(x, L64, base.eps)
        check_close(out.double().cpu().numpy(), ref, "bf16", f"stack layer {l}")
        x = O.round_storage(ref, "bf16")
    d = xg.double().cpu().numpy() - x
    rel = float(np.linalg.norm(d) / np.linalg.norm(x))
    assert rel <= 0.1, rel


def test_forward_is_deterministic(lib):
    shape, L = case("edge_prefill_t4096")
    G = to_gpu(L, lib)
    a = lib.forward(G["x"], G).clone()
    b = lib.forward(G["x"], G)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_dense_ffn_parity(lib):
    for dtype, (T, D, d_ff) in [("f32", (13, 256, 1152)), ("bf16", (16, 2048, 17408))]:
        from synth import make_dense
        Dn = make_dense(T, D, d_ff, dtype, 4)
        out = lib.dense_ffn(Dn["x"].cuda(), Dn["W1"].cuda(), Dn["W2"].cuda())
        torch.cuda.synchronize()
        ref = O.dense_ffn(O.to_f64(Dn["x"]), O.to_f64(Dn["W1"]), O.to_f64(Dn["W2"]))
        check_close(out.double().cpu().numpy(), ref, dtype, f"dense {dtype}")


def test_nonfinite_router_input_sets_device_error(lib):
    shape = LayerShape(4, 256, 8, 128, 128, "f32")
    L = make_layer(shape, 2)
    L["x"][1, 3] = float("nan")
    G = to_gpu(L, lib)
    ws = lib.alloc_workspace(lib.layer_shape(G["x"], G))
    lib.forward(G["x"], G, workspace=ws)
    assert lib.device_error(ws) == 1
    assert lib.device_error(ws) == 0          # cleared
    L["x"][1, 3] = 0.0
    G["x"] = L["x"].cuda()
    lib.forward(G["x"], G, workspace=ws)
    assert lib.device_error(ws) == 0


@pytest.mark.parametrize("T,ratio", [(1, 0.0), (1, 1.0), (5, 0.2), (16, 0.0), (16, 1.0), (11, 0.4)])
def test_decode_path_edge_cases(lib, T, ratio):
    # bf16, T <= 16, d_model a multiple of 256: the weight-streaming decode kernels
    shape = LayerShape(T, 512, 16, 256, 256, "bf16")
    L = make_layer(shape, 31, ratio=ratio if ratio > 0 else 0.2)
    if ratio == 0.0:
        L["b_r"] = torch.full_like(L["b_r"], -1e4)
    G = to_gpu(L, lib)
    out = lib.forward(G["x"], G, eps=shape.eps)
    torch.cuda.synchronize()
    ref, z, act = O.layer_forward_tokens(O.to_f64(L["x"]), to_oracle(L, "bf16"), shape.eps)
    assert act.all() if ratio == 1.0 else True
    check_close(out.double().cpu().numpy(), ref, "bf16", f"decode T={T} ratio={ratio}")
    # repeated calls reuse the workspace (counters, activations) and agree bitwise
    out2 = lib.forward(G["x"], G, eps=shape.eps)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


@pytest.mark.parametrize("shape,ratio,residual", [
    (LayerShape(300, 320, 5, 192, 320, "bf16"), 0.3, False),    # ragged rows, columns and K
    (LayerShape(129, 256, 3, 256, 64, "bf16"), 1.0, True),      # every pair active, residual
    (LayerShape(17, 512, 16, 64, 576, "bf16"), 0.2, False),     # smallest prefill batch
    (LayerShape(600, 1024, 12, 128, 1024, "bf16"), 0.0, False), # no pair active
])
def test_prefill_path_shapes(lib, shape, ratio, residual):
    # bf16, T > 16: the tensor-core prefill kernels
    L = make_layer(shape, 41, ratio=ratio if ratio > 0 else 0.2)
    if ratio == 0.0:
        L["b_r"] = torch.full_like(L["b_r"], -1e4)
    G = to_gpu(L, lib)
    out = lib.forward(G["x"], G, eps=shape.eps, residual=residual)
    torch.cuda.synchronize()
    ref, z, act = O.layer_forward_tokens(O.to_f64(L["x"]), to_oracle(L, "bf16"), shape.eps)
    if ratio == 1.0:
        assert act.all()
    if residual:
        ref = ref + O.to_f64(L["x"])
    check_close(out.double().cpu().numpy(), ref, "bf16", f"prefill {shape} ratio={ratio}")
    out2 = lib.forward(G["x"], G, eps=shape.eps, residual=residual)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_dense_ffn_tensor_core_path(lib):
    from synth import make_dense
    Dn = make_dense(300, 512, 1216, "bf16", 5)      # T > 16, ragged rows and columns
    out = lib.dense_ffn(Dn["x"].cuda(), Dn["W1"].cuda(), Dn["W2"].cuda())
    torch.cuda.synchronize()
    ref = O.dense_ffn(O.to_f64(Dn["x"]), O.to_f64(Dn["W1"]), O.to_f64(Dn["W2"]))
    check_close(out.double().cpu().numpy(), ref, "bf16", "dense bf16 T=300")


@pytest.mark.parametrize("T,dtype", [(40, "bf16"), (300, "bf16"), (8, "bf16"), (40, "f32")])
def test_routing_exact_on_cancelling_logits(lib, T, dtype):
    """Router rows 0-2 see logits whose products cancel exactly (features come
    in equal pairs, the weights in opposite pairs), so the exact logit is the
    bias: +2^-30 (active), -2^-30 and 0 (inactive).  An fp32 evaluation lands
    near zero with either sign; the decision must still be exact."""
    shape = LayerShape(T, 256, 8, 64, 64, dtype)
    L = make_layer(shape, 51)
    x = L["x"].float()
    x[:, 1::2] = x[:, 0::2]
    W = L["W_r"].float()
    W[:3, 1::2] = -W[:3, 0::2]
    L["x"] = x.to(L["x"].dtype)
    L["W_r"] = W.to(L["W_r"].dtype)
    L["b_r"][0] = 2.0 ** -30
    L["b_r"][1] = -(2.0 ** -30)
    L["b_r"][2] = 0.0
    G = to_gpu(L, lib)
    act = _routing_check(lib, shape, L, G)
    assert act[:, 0].all() and not act[:, 1].any() and not act[:, 2].any()
    out = lib.forward(G["x"], G, eps=shape.eps)
    torch.cuda.synchronize()
    ref = O.layer_forward(O.to_f64(L["x"]), to_oracle(L, dtype), shape.eps)
    check_close(out.double().cpu().numpy(), ref, dtype, f"cancelling logits T={T} {dtype}")


@pytest.mark.parametrize("T,dtype", [(40, "bf16"), (8, "bf16"), (40, "f32")])
def test_routing_exact_wide_exponent_range(lib, T, dtype):
    """Even tokens carry two features of 2^120 that cancel in router rows 0-3
    (rows 0-2 as in the cancelling test, row 3 with weights +1, -1), so the
    exact logit of those rows is decided by products more than 128 bits below
    the largest one: the general fixed-point accumulation, not the register
    window.  Routing only (the other rows' logits are ~2^116)."""
    shape = LayerShape(T, 256, 8, 64, 64, dtype)
    L = make_layer(shape, 53)
    x = L["x"].float()
    x[:, 1::2] = x[:, 0::2]
    x[0::2, 0] = 2.0 ** 120
    x[0::2, 1] = 2.0 ** 120
    W = L["W_r"].float()
    W[:3, 1::2] = -W[:3, 0::2]
    W[3, 0], W[3, 1] = 1.0, -1.0
    L["x"] = x.to(L["x"].dtype)
    L["W_r"] = W.to(L["W_r"].dtype)
    L["b_r"][0] = 2.0 ** -30
    L["b_r"][1] = -(2.0 ** -30)
    L["b_r"][2] = 0.0
    G = to_gpu(L, lib)
    act = _routing_check(lib, shape, L, G)
    assert act[:, 0].all() and not act[:, 1].any() and not act[:, 2].any()


def _plant_near_zero_logits(L, pairs):
    """Set b_r[e] = -fl32(x_t . W_r[e]) for each (t, e): the exact logit of t
    at e is then the fp32 rounding residual of its dot product (|z| below half
    an fp32 ulp of the sum, either sign, or exactly 0 when the sum is an fp32
    value), the hardest case for a sign decision made from an fp32 sum."""
    import math
    x64, W64 = O.to_f64(L["x"]), O.to_f64(L["W_r"])
    for t, e in pairs:
        dot = math.fsum((x64[t] * W64[e]).tolist())     # products exact in fp64
        L["b_r"][e] = -float(np.float32(dot))
    return L


@pytest.mark.parametrize("name", ["edge_decode_t1", "edge_decode_t16", "large_t16",
                                  "edge_prefill_t4096"])
def test_routing_exact_on_planted_near_zero_logits(lib, name):
    """The router each forward path runs (the decode kernels' router for bf16
    batches of up to 16 tokens, the tiled router above) decides logits whose
    exact value is a rounding residual or exactly zero like the oracle does."""
    shape, L = case(name)
    T, E = shape.T, shape.E
    rng = np.random.default_rng(7)
    es = rng.choice(E, min(E, 24), replace=False)
    pairs = [(int(rng.integers(T)), int(e)) for e in es]
    L = _plant_near_zero_logits(L, pairs)
    G = to_gpu(L, lib)
    if T <= 16:
        act = _routing_check(lib, shape, L, G)
    else:
        toks = np.unique(np.array([t for t, _ in pairs] + [0, T - 1]))
        act = _routing_check(lib, shape, L, G, tokens=toks)
    # the forward pass of the same batch uses the same decisions
    out = lib.forward(G["x"], G, eps=shape.eps)
    torch.cuda.synchronize()
    toks = sorted({t for t, _ in pairs} | {0, T - 1})
    ref = oracle_forward(O.to_f64(L["x"]), to_oracle(L, shape.dtype), shape.eps, toks)
    check_close(out.double().cpu().numpy()[toks], ref, shape.dtype, f"planted {name}")


@pytest.mark.parametrize("T", [1, 5, 16])
def test_dense_ffn_decode_path(lib, T):
    # bf16, T <= 16: the weight-streaming kernel with no routed experts
    from synth import make_dense
    Dn = make_dense(T, 2048, 17408, "bf16", 6)
    out = lib.dense_ffn(Dn["x"].cuda(), Dn["W1"].cuda(), Dn["W2"].cuda())
    torch.cuda.synchronize()
    ref = O.dense_ffn(O.to_f64(Dn["x"]), O.to_f64(Dn["W1"]), O.to_f64(Dn["W2"]))
    check_close(out.double().cpu().numpy(), ref, "bf16", f"dense decode T={T}")
    out2 = lib.dense_ffn(Dn["x"].cuda(), Dn["W1"].cuda(), Dn["W2"].cuda())
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


@pytest.mark.parametrize("shape", [LayerShape(16, 512, 16, 256, 256, "bf16"),      # decode kernel
                                   LayerShape(300, 320, 5, 192, 320, "bf16")])     # tensor-core kernels
def test_timeout_path_reports_and_recovers(lib, shape):
    """With the wait limit lowered to a few hundred cycles the kernels give up
    their waits for data: they set bit 2 of the device error word, wait for
    the copies and tensor-core operations they already issued, and return.
    The next call with the default limit is correct."""
    L = make_layer(shape, 61)
    G = to_gpu(L, lib)
    ws = lib.alloc_workspace(lib.layer_shape(G["x"], G))
    ref = O.layer_forward(O.to_f64(L["x"]), to_oracle(L, "bf16"), shape.eps)
    lib.set_wait_limit(300)
    try:
        for _ in range(3):
            lib.forward(G["x"], G, workspace=ws, eps=shape.eps)
            assert lib.device_error(ws) & 2
    finally:
        lib.set_wait_limit(0)
    out = lib.forward(G["x"], G, workspace=ws, eps=shape.eps)
    assert lib.device_error(ws) == 0
    check_close(out.double().cpu().numpy(), ref, "bf16", f"after timeouts {shape}")


# --------------------------------------------------------------------------
# TopK routing (the baseline of the paper's §5 comparison)

def _topk_k(E):
    return max(1, int(round(0.2 * E)))


def _topk_check(lib, shape, L, G, k, tokens=None):
    res = lib.routing(G["x"], G, topk=k)
    torch.cuda.synchronize()
    act_gpu = _np(res["active"]).astype(bool)
    x64 = O.to_f64(L["x"])
    toks = np.arange(shape.T) if tokens is None else np.asarray(tokens)
    z, act, r = O.topk_route(x64[toks], O.to_f64(L["W_r"]), O.to_f64(L["b_r"]), k)
    np.testing.assert_array_equal(act_gpu[toks], act)
    assert (act_gpu.sum(axis=1) == k).all()
    counts, offsets, perm, n_tok = O.routing_tables(act_gpu)
    np.testing.assert_array_equal(_np(res["counts"]), counts)
    np.testing.assert_array_equal(_np(res["offsets"]), offsets)
    np.testing.assert_array_equal(_np(res["perm"])[: offsets[-1]], perm)
    scale = np.abs(z).max()
    assert np.abs(_np(res["r"])[toks] - r).max() <= 1e-5 * scale
    return act_gpu


@pytest.mark.parametrize("name", ["tiny_f32", "edge_decode_t1", "edge_decode_t16", "large_t16",
                                  "edge_prefill_t4096"])
def test_topk_routing_bit_exact(lib, name):
    shape, L = case(name)
    G = to_gpu(L, lib)
    k = _topk_k(shape.E)
    toks = None
    if shape.T > 64:
        toks = np.sort(np.random.default_rng(2).choice(shape.T, 64, replace=False))
    _topk_check(lib, shape, L, G, k, toks)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_topk_routing_exact_ties(lib, dtype):
    """Rows 1 and 3 of W_r copy row 0 (same bias): exact ties, which go to
    the lower index.  Row 5 is row 4 with one weight moved by one unit in the
    last place of the storage format, so the two logits differ by x_t[7]
    times that unit: inside the fp32 sums' error bounds, where the exact
    comparison decides."""
    import math
    shape = LayerShape(40, 256, 8, 64, 64, dtype)
    L = make_layer(shape, 71)
    W = L["W_r"].float()
    W[1] = W[0]
    W[3] = W[0]
    W[5] = W[4]
    w47 = float(W[4, 7])
    W[5, 7] = w47 + 2.0 ** (math.floor(math.log2(abs(w47))) - (7 if dtype == "bf16" else 23))
    b = L["b_r"]
    b[1] = b[0]
    b[3] = b[0]
    b[5] = b[4]
    # make rows 0, 4 sit at the boundary of a k = 2 selection for many tokens
    b[0] += 2.0
    b[4] += 2.0
    L["W_r"] = W.to(L["W_r"].dtype)
    G = to_gpu(L, lib)
    for k in (1, 2, 3, 4):
        _topk_check(lib, shape, L, G, k)


@pytest.mark.parametrize("shape", [LayerShape(16, 2048, 64, 256, 1024, "bf16"),   # decode kernel
                                   LayerShape(300, 320, 5, 192, 320, "bf16"),     # tensor-core kernels
                                   LayerShape(37, 256, 8, 128, 192, "f32")])      # general kernels
def test_topk_forward_parity(lib, shape):
    L = make_layer(shape, 73)
    G = to_gpu(L, lib)
    k = _topk_k(shape.E)
    out = lib.forward(G["x"], G, eps=shape.eps, topk=k)
    torch.cuda.synchronize()
    L64 = to_oracle(L, shape.dtype)
    x64 = O.to_f64(L["x"])
    _, act, r = O.topk_route(x64, L64["W_r"], L64["b_r"], k)
    # the layer with the TopK decisions: the oracle's per-expert terms
    ref = np.zeros((shape.T, shape.D))
    for t in range(shape.T):
        u = L64["W_bar_up"] @ x64[t]
        y = O.shared_expert(x64[t], L64["W_s_up"], L64["W_s_down"])
        for e in range(shape.E):
            if act[t, e]:
                y = y + (L64["s"][e] * r[t, e]) * O.expert_output(x64[t], L64["W_up"][e], L64["W_down"][e], u,
                                                                 shape.eps)
        ref[t] = y
    check_close(out.double().cpu().numpy(), ref, shape.dtype, f"topk forward {shape}")


def test_residual_stack_prefill_t16384(lib):
    """The 8-layer residual stack of the larger layer (d_model 4096, 128
    experts) at T = 16384 tokens: the tensor-core path, whose routed outputs
    are staged in fp16.  Activations grow several-fold per layer without a
    normalisation between layers, which once pushed the staged values out of
    the fp16 range; they are now staged before the s_e r_e scaling.  Each
    layer is checked on the GPU's own input to it (teacher forcing) on
    sampled tokens: random ones, the last one, and per layer the token with
    the fewest active experts and the token with the logit closest to zero."""
    base = case("large_t16384")[0]
    T = base.T
    x = make_layer(base, 3, layer=0)["x"].cuda()
    ws = None
    rng = np.random.default_rng(5)
    for l in range(8):
        W = make_layer(base, 3, layer=l, with_x=False)
        G = to_gpu(W, lib)
        if ws is None:
            ws = lib.alloc_workspace(lib.layer_shape(x, G, residual=True))
        out = lib.forward(x, G, workspace=ws, eps=base.eps, residual=True)
        assert lib.device_error(ws) == 0
        rt = lib.routing(x, G)
        n_act = rt["n_tok"].cpu().numpy()
        r = rt["r"]
        zmin = torch.where(r > 0, r, torch.full_like(r, float("inf"))).min(dim=1).values
        toks = set(rng.choice(T, 8, replace=False).tolist()) | {T - 1, int(np.argmin(n_act)),
                                                                  int(torch.argmin(zmin).item())}
        toks = sorted(toks)
        x64 = x[toks].double().cpu().numpy()
        L64 = to_oracle(W, "bf16")
        ref = x64 + oracle_forward(x64, L64, base.eps, range(len(toks)), parallel=False)
        check_close(out.double().cpu().numpy()[toks], ref, "bf16", f"stack T=16384 layer {l}")
        x = out
        del G, rt
    assert torch.isfinite(x.float()).all()


@pytest.mark.parametrize("shape,topk", [
    (LayerShape(40, 256, 8, 512, 64, "bf16"), 0),      # tiled router, general expert kernels (d_e 512)
    (LayerShape(300, 320, 5, 192, 320, "bf16"), 0),    # tensor-core kernels
    (LayerShape(16, 512, 16, 256, 256, "bf16"), 0),    # decode kernel
    (LayerShape(37, 256, 8, 128, 192, "f32"), 0),      # general kernels
    (LayerShape(300, 320, 5, 192, 320, "bf16"), 2),    # TopK routing, tensor-core kernels
    (LayerShape(16, 512, 16, 256, 256, "bf16"), 3),    # TopK routing, decode kernel
])
def test_workspace_size_covers_every_write(lib, shape, topk):
    """The kernels write only inside deco_moe_workspace_size bytes: a guard
    region after the workspace keeps its byte pattern through a forward and a
    routing call, and the output still matches the oracle's routing."""
    L = make_layer(shape, 81)
    G = to_gpu(L, lib)
    n = lib.workspace_size(lib.layer_shape(G["x"], G, topk=topk))
    buf = torch.full((n + 65536,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = buf[:n]
    lib.forward(G["x"], G, workspace=ws, eps=shape.eps, topk=topk)
    lib.routing(G["x"], G, workspace=ws, topk=topk)
    torch.cuda.synchronize()
    assert bool((buf[n:] == 0xA5).all())


# --------------------------------------------------------------------------
# gated experts ("DECO (gated)"): a = NormSiLU(x W_up^T - u) * (x W_val^T)

@pytest.mark.parametrize("shape,topk", [
    (LayerShape(16, 2048, 64, 256, 1024, "bf16"), 0),   # decode kernel
    (LayerShape(5, 512, 16, 256, 256, "bf16"), 0),      # decode kernel, ragged batch
    (LayerShape(300, 320, 5, 192, 320, "bf16"), 0),     # tensor-core kernels, ragged tiles
    (LayerShape(37, 256, 8, 128, 192, "f32"), 0),       # general kernels
    (LayerShape(40, 256, 8, 512, 64, "bf16"), 0),       # tiled router, general expert kernels
    (LayerShape(16, 512, 16, 256, 256, "bf16"), 3),     # gated with TopK routing
])
def test_gated_forward_parity(lib, shape, topk):
    L = make_layer(shape, 91, gated=True, ratio=0.3)
    G = to_gpu(L, lib)
    out = lib.forward(G["x"], G, eps=shape.eps, topk=topk)
    torch.cuda.synchronize()
    L64 = to_oracle(L, shape.dtype)
    x64 = O.to_f64(L["x"])
    if topk == 0:
        ref = O.layer_forward(x64, L64, shape.eps)
    else:
        _, act, r = O.topk_route(x64, L64["W_r"], L64["b_r"], topk)
        ref = np.zeros((shape.T, shape.D))
        for t in range(shape.T):
            u = L64["W_bar_up"] @ x64[t]
            y = O.shared_expert(x64[t], L64["W_s_up"], L64["W_s_down"])
            for e in range(shape.E):
                if act[t, e]:
                    y = y + (L64["s"][e] * r[t, e]) * O.expert_output(
                        x64[t], L64["W_up"][e], L64["W_down"][e], u, shape.eps, L64["W_val"][e])
            ref[t] = y
    check_close(out.double().cpu().numpy(), ref, shape.dtype, f"gated {shape} topk={topk}")
    out2 = lib.forward(G["x"], G, eps=shape.eps, topk=topk)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_gated_prefill_full_size_sampled(lib):
    shape, L = case("edge_prefill_t4096")
    L["W_val"] = make_layer(shape, 2, gated=True, with_x=False)["W_val"]
    G = to_gpu(L, lib)
    ws = lib.alloc_workspace(lib.layer_shape(G["x"], G))
    n = ws.numel()
    guard = torch.full((n + 65536,), 0xA5, dtype=torch.uint8, device="cuda")
    out = lib.forward(G["x"], G, workspace=guard[:n], eps=shape.eps)
    torch.cuda.synchronize()
    assert bool((guard[n:] == 0xA5).all())
    toks = [0, 1, 64, 1000, 2047, shape.T - 1]
    ref = oracle_forward(O.to_f64(L["x"]), to_oracle(L, "bf16"), shape.eps, toks)
    check_close(out.double().cpu().numpy()[toks], ref, "bf16", "gated prefill T=4096")


def test_gated_requires_the_value_branch(lib):
    shape = LayerShape(4, 256, 8, 64, 64, "bf16")
    L = make_layer(shape, 92)
    G = to_gpu(L, lib)
    sh = lib.layer_shape(G["x"], G)
    sh.gated = 1                                  # gated shape, no W_val pointer
    w = lib._weights(G)
    ws = lib.alloc_workspace(sh)
    out = torch.empty_like(G["x"])
    import ctypes
    rc = lib._lib.deco_moe_forward(ctypes.byref(sh), G["x"].data_ptr(), ctypes.byref(w), out.data_ptr(),
                                   ws.data_ptr(), ws.numel(), lib._stream(None))
    assert rc == 1


# --------------------------------------------------------------------------
# routed experts held in pinned host memory (offloaded parameters)

def _host_experts(G):
    """The routed experts' matrices moved to pinned host memory, which the
    device reads through its own address space."""
    H = dict(G)
    for n in ("W_up", "W_down", "W_val"):
        if n in H:
            H[n] = H[n].cpu().pin_memory()
    return H


@pytest.mark.parametrize("name", ["tiny_f32", "edge_decode_t4"])
def test_experts_in_host_memory(lib, name):
    shape, L = case(name)
    G = to_gpu(L, lib)
    H = _host_experts(G)
    assert lib.layer_shape(G["x"], H).experts_on_host == 1
    out = lib.forward(G["x"], H, eps=shape.eps)
    torch.cuda.synchronize()
    ref = oracle_forward(O.to_f64(L["x"]), to_oracle(L, shape.dtype), shape.eps, range(shape.T))
    check_close(out.double().cpu().numpy(), ref, shape.dtype, name + " experts on host")
    if shape.dtype == "f32":   # the same general kernels as device-resident weights: bitwise equal
        assert torch.equal(out, lib.forward(G["x"], G, eps=shape.eps))


def test_experts_in_host_memory_prefill_batch_and_gated(lib):
    shape = LayerShape(40, 512, 16, 128, 256, "bf16")
    for gated in (False, True):
        L = make_layer(shape, 31, gated=gated)
        G = to_gpu(L, lib)
        out = lib.forward(G["x"], _host_experts(G), eps=shape.eps)
        torch.cuda.synchronize()
        ref = oracle_forward(O.to_f64(L["x"]), to_oracle(L, shape.dtype), shape.eps, range(shape.T))
        check_close(out.double().cpu().numpy(), ref, shape.dtype, f"host experts T=40 gated={gated}")


def test_experts_on_host_must_be_mapped(lib):
    shape, L = case("edge_decode_t4")
    G = to_gpu(L, lib)
    H = dict(G)
    H["W_up"], H["W_down"] = G["W_up"].cpu(), G["W_down"].cpu()   # pageable: not reachable
    with pytest.raises(lib.DecoError) as ei:
        lib.forward(G["x"], H, eps=shape.eps)
    assert ei.value.code == 1
