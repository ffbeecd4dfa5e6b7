"""C-ABI tests that need no GPU: the library loads, exports every function
include/deco_moe.h declares, and rejects bad arguments on the host before
launching anything (none of these calls reaches the device)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def deco():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "deco_build", os.path.join(ROOT, "sparse_moe_ffn_relu_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import sparse_moe_ffn_relu_b200 as d
    return d


def _declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(deco_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(deco):
    names = _declared("deco_moe.h")
    assert "deco_moe_forward" in names and len(names) >= 8
    lib = ctypes.CDLL(deco.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(deco.EXPORTS)


def test_status_strings(deco):
    for code in range(6):
        assert deco._lib.deco_status_string(code)
    assert deco._lib.deco_status_string(99) == b"unknown status"


def _shape(deco, **kw):
    base = dict(T=16, D=2048, E=64, d_e=256, d_s=1024, dtype=deco.DECO_BF16)
    base.update(kw)
    return deco.make_shape(base["T"], base["D"], base["E"], base["d_e"], base["d_s"], base["dtype"])


def _ws(deco, shape):
    n = ctypes.c_size_t(0)
    rc = deco._lib.deco_moe_workspace_size(ctypes.byref(shape), ctypes.byref(n))
    return rc, n.value


def test_workspace_size_and_shape_checks(deco):
    rc, n = _ws(deco, _shape(deco))
    assert rc == 0 and n > 0 and n % 256 == 0
    rc2, n2 = _ws(deco, _shape(deco, T=4096))
    assert rc2 == 0 and n2 > n
    assert _ws(deco, _shape(deco, T=0)) [0] == 0
    bad = [dict(T=-1), dict(D=0), dict(E=0), dict(d_e=0), dict(d_s=0), dict(dtype=7)]
    for kw in bad:
        assert _ws(deco, _shape(deco, **kw))[0] == 1, kw
    unsupported = [dict(D=2000), dict(E=257), dict(d_e=96), dict(d_e=1024), dict(d_s=100)]
    for kw in unsupported:
        assert _ws(deco, _shape(deco, **kw))[0] == 2, kw
    s = _shape(deco)
    s.rms_eps = float("nan")
    assert _ws(deco, s)[0] == 1
    assert deco._lib.deco_moe_workspace_size(ctypes.byref(s), None) == 1


def _fake_weights(deco, **override):
    w = deco.Weights(*[0x10000 + 0x1000 * i for i in range(8)])
    for k, v in override.items():
        setattr(w, k, v)
    return w


def test_forward_rejects_bad_arguments_without_launching(deco):
    lib = deco._lib
    s = _shape(deco)
    _, need = _ws(deco, s)
    w = _fake_weights(deco)
    X, OUT, WS = 0x100000, 0x200000, 0x300000
    fwd = lambda sh, x, ww, out, ws, n: lib.deco_moe_forward(  # noqa: E731
        ctypes.byref(sh), x, ctypes.byref(ww) if ww is not None else None, out, ws, n, None)
    assert fwd(s, X, None, OUT, WS, need) == 1                       # no weights
    assert fwd(s, X, _fake_weights(deco, W_up=None), OUT, WS, need) == 1
    assert fwd(s, X, _fake_weights(deco, s=0x10004), OUT, WS, need) == 1   # misaligned
    assert fwd(s, None, w, OUT, WS, need) == 1                       # no x
    assert fwd(s, X, w, X, WS, need) == 1                            # x aliases out
    assert fwd(s, X + 8, w, OUT, WS, need) == 1                      # misaligned x
    assert fwd(s, X, w, OUT, None, need) == 3                        # no workspace
    assert fwd(s, X, w, OUT, WS, need - 1) == 3                      # too small
    assert fwd(s, X, w, OUT, WS + 16, need) == 3                     # misaligned workspace
    assert fwd(_shape(deco, E=300), X, w, OUT, WS, need) == 2
    assert fwd(_shape(deco, T=0), X, w, OUT, WS, 0) == 0             # empty batch: no-op


def test_routing_mean_dense_reject_bad_arguments(deco):
    lib = deco._lib
    s = _shape(deco)
    _, need = _ws(deco, s)
    w = _fake_weights(deco)
    r = deco.Routing(*[0x400000 + 0x1000 * i for i in range(6)])
    assert lib.deco_moe_routing(ctypes.byref(s), 0x100000, ctypes.byref(w), None, 0x300000,
                                need, None) == 1
    assert lib.deco_moe_routing(ctypes.byref(s), 0x100000, ctypes.byref(w), ctypes.byref(r),
                                0x300000, 16, None) == 3
    assert lib.deco_moe_mean_up(0, 256, 2048, 1, 0x1000, 0x2000, None) == 1
    assert lib.deco_moe_mean_up(4, 256, 2048, 1, 0x1000, 0x1000, None) == 1
    assert lib.deco_moe_mean_up(4, 256, 2048, 3, 0x1000, 0x2000, None) == 1
    n = ctypes.c_size_t(0)
    assert lib.deco_dense_ffn_workspace_size(16, 2048, 17408, 1, ctypes.byref(n)) == 0 and n.value > 0
    assert lib.deco_dense_ffn_workspace_size(16, 2000, 17408, 1, ctypes.byref(n)) == 2
    assert lib.deco_dense_ffn_forward(16, 2048, 17408, 1, 0x1000, 0x2000, 0x3000, 0x1000,
                                      0x5000, n.value, None) == 1    # x aliases out
    assert lib.deco_dense_ffn_forward(16, 2048, 17408, 1, 0x1000, 0x2000, 0x3000, 0x4000,
                                      0x5000, 8, None) == 3
    code = ctypes.c_int(0)
    assert lib.deco_moe_device_error(None, ctypes.byref(code), None) == 1


def test_workspace_follows_the_kernel_path(deco):
    """Host-side path choice seen through the workspace plan: a bf16 batch of
    more than 16 tokens with d_e <= 256 takes the tensor-core path, whose
    workspace holds an fp16 row of D values per possible (token, expert) pair;
    fp32 batches and d_e = 512 take the general kernels, which do not."""
    T, D, E = 32, 2048, 64
    rc, n_bf16 = _ws(deco, _shape(deco, T=T))
    rc2, n_f32 = _ws(deco, _shape(deco, T=T, dtype=deco.DECO_F32))
    rc3, n_wide = _ws(deco, _shape(deco, T=T, d_e=512))
    assert rc == rc2 == rc3 == 0
    assert n_bf16 >= T * E * D * 2
    assert n_f32 < T * E * D * 2 and n_wide < T * E * D * 2 + T * E * 512 * 4


def test_decode_workspaces_fit_the_static_scratch(deco):
    """Every decode batch of the two bench layers fits the built-in scratch of
    deco_moe_forward_static, whose size the header and the binding agree on."""
    text = open(os.path.join(ROOT, "include", "deco_moe.h")).read()
    m = re.search(r"#define DECO_STATIC_SCRATCH_BYTES \((\d+)u << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == deco.STATIC_SCRATCH_BYTES
    for T in (1, 4, 16):
        for D, E, d_s in ((2048, 64, 1024), (4096, 128, 2048)):
            rc, n = _ws(deco, _shape(deco, T=T, D=D, E=E, d_s=d_s))
            assert rc == 0 and n <= deco.STATIC_SCRATCH_BYTES, (T, D, E, n)


def test_experts_on_host_is_checked_before_launching(deco):
    """Host-resident experts: the flag is 0 or 1, such a batch takes the
    general kernels (no per-pair rows in its workspace), and weight pointers
    that are not mapped host memory are rejected before any launch."""
    T, D, E = 32, 2048, 64
    s = _shape(deco, T=T)
    s.experts_on_host = 2
    assert _ws(deco, s)[0] == 1
    s.experts_on_host = 1
    rc, n = _ws(deco, s)
    assert rc == 0 and n < T * E * D * 2
    w = _fake_weights(deco)
    assert deco._lib.deco_moe_forward(ctypes.byref(s), 0x100000, ctypes.byref(w), 0x200000, 0x300000,
                                      n, None) == 1
    assert deco._lib.deco_moe_forward_static(ctypes.byref(s), 0x100000, ctypes.byref(w), 0x200000,
                                             None) == 1


def test_training_side_host_checks(deco):
    """The sparsity controller against the oracle's, and the backward's
    argument checks (no launch)."""
    import oracle as O
    for lam, ratio, target in [(1.0, 0.25, 0.2), (0.5, 0.1, 0.2), (2.0, 0.2, 0.2)]:
        assert deco.sparsity_controller(lam, ratio, target) == O.sparsity_controller(lam, ratio, target)
    v = ctypes.c_double(1.0)
    assert deco._lib.deco_sparsity_controller(ctypes.byref(v), 0.3, 0.2, 1.0) == 1   # factor must exceed 1
    lib = deco._lib
    s = _shape(deco)
    n = ctypes.c_size_t(0)
    assert lib.deco_moe_backward_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0 and n.value > 0
    st = _shape(deco)
    st.topk = 13
    assert lib.deco_moe_backward_workspace_size(ctypes.byref(st), ctypes.byref(n)) == 2
    w = _fake_weights(deco)
    g = deco.Grads(*[0x500000 + 0x1000 * i for i in range(8)])
    bw = lambda sh, gg, ws, nb: lib.deco_moe_backward(  # noqa: E731
        ctypes.byref(sh), 0x100000, ctypes.byref(w), 0x180000, None, gg, ws, nb, None)
    assert lib.deco_moe_backward_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0
    assert bw(s, None, 0x300000, n.value) == 1                              # no gradients
    assert bw(s, ctypes.byref(deco.Grads(*([0] * 9))), 0x300000, n.value) == 1
    assert bw(s, ctypes.byref(g), 0x300000, n.value - 1) == 3               # workspace too small
    assert bw(st, ctypes.byref(g), 0x300000, n.value) == 2                  # TopK
    assert lib.deco_moe_router_entropy(4, 0, 0x1000, 0x2000, 1.0, 0x3000, 0x4000, None) == 1
